// SIMT (fp32 FFMA) chunked lightning attention forward.
//
// Tiling after "MiniMax-01: Scaling Foundation Models with Lightning
// Attention | Summary", section 2.2: the sequence is cut into tiles of C
// tokens; inside a tile a masked, decayed score matrix is applied to V; the
// tiles before it enter through the carried d x d state; the state is then
// decayed by lam^L and the tile's keys and values are added. Section 3.3 of
// the same page lists tile sizes 32, 64, 128 next to 256; this kernel takes
// C = 32, 64 or 128 and its result must not depend on C beyond rounding.
//
// Decay exponents are never negative: lam^(r-c) in the mask, lam^(r+1) on the
// carried-state term of local row r, lam^(L-1-c) on key c of the update and
// lam^L on the state (lam^-j factors would overflow fp32 for strong decay).
//
// One CTA per (problem, slice of DV value columns); the state slice S[d][DV]
// stays in shared memory for the whole sequence. This is the fp32 path
// (tolerance 1e-4 of rms is beyond tf32 tensor cores) and a reference-grade
// GPU path for shapes the tensor-core kernel does not cover.
#include <algorithm>

#include "kernels.h"

namespace la {
namespace {

struct SimtArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* slopes;
    void* o;
    float* state_out;
    Problems P;
    int reverse;
    const float* state_in;  // [problems][D][D] state before the first token, or null
    int state_only;         // final states only (o is not written)
};

template <int D, int DV, int C>
constexpr size_t simt_smem_floats()
{
    return 2 * C * (D + 1) + C * DV + C * (C + 1) + D * DV + (C + 1);
}

template <typename Tin, typename Tout, int D, int DV, int C>
__global__ void __launch_bounds__(256) simt_forward_kernel(SimtArgs a)
{
    extern __shared__ float sm[];
    float* Qs = sm;                  // [C][D+1]
    float* Ks = Qs + C * (D + 1);    // [C][D+1]
    float* Vs = Ks + C * (D + 1);    // [C][DV]
    float* As = Vs + C * DV;         // [C][C+1] decayed, masked scores
    float* Ss = As + C * (C + 1);    // [D][DV] carried state slice
    float* pw = Ss + D * DV;         // [C+1]   lam^m

    const long long prob = blockIdx.x;
    const int c0 = blockIdx.y * DV;
    const int H = a.P.H;
    const int h = (int)(prob % H);
    long long row0, len, st_idx;
    if (a.P.cu_seqlens) {
        const long long s = prob / H;
        const long long b = a.P.cu_seqlens[s], e = a.P.cu_seqlens[s + 1];
        row0 = (long long)h * a.P.total + b;
        len = e - b;
        if (len > 0 && len < a.P.min_len) return;  // served by another kernel
        st_idx = prob;  // s * H + h
    } else {
        row0 = prob * a.P.N;
        len = a.P.N;
        st_idx = prob;
    }
    const float slope = a.slopes[h];
    for (int m = threadIdx.x; m <= C; m += blockDim.x) pw[m] = expf(-slope * (float)m);
    // The carried state starts as the caller's incoming state (or zero); this
    // CTA reads its own column slice before it writes that slice of state_out.
    const float* s_in = a.state_in ? a.state_in + st_idx * D * D : nullptr;
    for (int e = threadIdx.x; e < D * DV; e += blockDim.x)
        Ss[e] = s_in ? s_in[(e / DV) * D + c0 + e % DV] : 0.f;

    const Tin* q = (const Tin*)a.q + row0 * D;
    const Tin* k = (const Tin*)a.k + row0 * D;
    const Tin* v = (const Tin*)a.v + row0 * D;
    Tout* o = (Tout*)a.o + row0 * D;
    const bool rev = a.reverse != 0;
    const long long ntiles = (len + C - 1) / C;
    __syncthreads();

    for (long long it = 0; it < ntiles; ++it) {
        const long long t0 = (rev ? (ntiles - 1 - it) : it) * C;
        const int L = (int)min((long long)C, len - t0);
        for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
            const int r = e / D, c = e % D;
            float qv = 0.f, kv = 0.f;
            if (r < L) {
                qv = to_f32(q[(t0 + r) * D + c]);
                kv = to_f32(k[(t0 + r) * D + c]);
            }
            Qs[r * (D + 1) + c] = qv;
            Ks[r * (D + 1) + c] = kv;
        }
        for (int e = threadIdx.x; e < C * DV; e += blockDim.x) {
            const int r = e / DV, c = e % DV;
            Vs[e] = (r < L) ? to_f32(v[(t0 + r) * D + c0 + c]) : 0.f;
        }
        __syncthreads();
        if (!a.state_only) {  // the outputs of this tile
            // Intra-tile scores: As[r][c] = lam^|r-c| (q_r . k_c) on the causal side.
            for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
                const int r = e / C, c = e % C;
                float w = 0.f;
                const bool keep = r < L && c < L && (rev ? (c >= r) : (c <= r));
                if (keep) {
                    float s = 0.f;
#pragma unroll 8
                    for (int x = 0; x < D; ++x) s = fmaf(Qs[r * (D + 1) + x], Ks[c * (D + 1) + x], s);
                    w = s * pw[rev ? (c - r) : (r - c)];
                }
                As[r * (C + 1) + c] = w;
            }
            __syncthreads();
            // Outputs: intra product plus the decayed carried-state product.
            for (int e = threadIdx.x; e < C * DV; e += blockDim.x) {
                const int r = e / DV, b = e % DV;
                if (r >= L) continue;
                float intra = 0.f;
                for (int c = 0; c < L; ++c) intra = fmaf(As[r * (C + 1) + c], Vs[c * DV + b], intra);
                float inter = 0.f;
#pragma unroll 8
                for (int x = 0; x < D; ++x) inter = fmaf(Qs[r * (D + 1) + x], Ss[x * DV + b], inter);
                const float sc = pw[rev ? (L - r) : (r + 1)];
                o[(t0 + r) * D + c0 + b] = from_f32<Tout>(fmaf(sc, inter, intra));
            }
            __syncthreads();
        }
        // State update: S <- lam^L S + sum_c lam^(L-1-c) k_c^T v_c (reverse: lam^c).
        for (int e = threadIdx.x; e < D * DV; e += blockDim.x) {
            const int x = e / DV, b = e % DV;
            float acc = pw[L] * Ss[e];
            for (int c = 0; c < L; ++c)
                acc = fmaf(Ks[c * (D + 1) + x] * pw[rev ? c : (L - 1 - c)], Vs[c * DV + b], acc);
            Ss[e] = acc;
        }
        __syncthreads();
    }
    if (a.state_out) {
        float* st = a.state_out + st_idx * D * D;
        for (int e = threadIdx.x; e < D * DV; e += blockDim.x) {
            const int x = e / DV, b = e % DV;
            st[x * D + c0 + b] = Ss[e];
        }
    }
}

template <typename Tin, typename Tout, int D, int DV, int C>
cudaError_t launch_one(const SimtArgs& a, cudaStream_t stream)
{
    const size_t smem = simt_smem_floats<D, DV, C>() * sizeof(float);
    auto kern = simt_forward_kernel<Tin, Tout, D, DV, C>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const long long nprob = a.P.count();
    if (nprob == 0) return cudaSuccess;
    dim3 grid((unsigned)nprob, D / DV);
    kern<<<grid, 256, smem, stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename Tin, typename Tout, int D>
cudaError_t launch_d(const SimtArgs& a, int block, cudaStream_t stream)
{
    switch (block) {
    case 32: return launch_one<Tin, Tout, D, 64, 32>(a, stream);
    case 64: return launch_one<Tin, Tout, D, 64, 64>(a, stream);
    case 128:
        // Keep the largest instantiation within 227 KB of shared memory.
        if (D == 128) return launch_one<Tin, Tout, D, 32, 128>(a, stream);
        return launch_one<Tin, Tout, D, 64, 128>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename Tin, typename Tout>
cudaError_t launch_t(const SimtArgs& a, int d, int block, cudaStream_t stream)
{
    if (d == 64) return launch_d<Tin, Tout, 64>(a, block, stream);
    if (d == 128) return launch_d<Tin, Tout, 128>(a, block, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_forward(const Problems& P, const void* q, const void* k, const void* v,
                                const float* slopes, void* o, float* state_out, int d,
                                int in_t, int out_t, int block, int reverse,
                                cudaStream_t stream, const float* state_in, int state_only)
{
    SimtArgs a{q, k, v, slopes, o, state_out, P, reverse, reverse ? nullptr : state_in,
               state_only};
    if (in_t == LA_F32 && out_t == LA_F32) return launch_t<float, float>(a, d, block, stream);
    if (in_t == LA_BF16 && out_t == LA_F32)
        return launch_t<__nv_bfloat16, float>(a, d, block, stream);
    if (in_t == LA_BF16 && out_t == LA_BF16)
        return launch_t<__nv_bfloat16, __nv_bfloat16>(a, d, block, stream);
    return cudaErrorInvalidValue;
}

}  // namespace la
