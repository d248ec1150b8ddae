// Fused single-token decode step of lightning attention.
//
// "MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
// section 3.3 (Batched Kernel Fusion): the memory-bound decode operations are
// fused into one kernel. For each (sequence b, head h):
//     S <- lam_h S + k^T v        (S[a][c] += k_a v_c after the decay)
//     o  = q S                    (with the updated state)
// The fp32 state is the only large operand: it is read once and written once,
// so the kernel is a pure HBM stream of 2 * 4 * d * d bytes per (b, h).
//
// The packed form (PACKED = 1) serves a batch of mixed lengths: the CTA of
// (sequence s, head h) handles the single token of s when s has exactly one
// token in the packed [H][total][d] inputs, and exits otherwise (longer
// sequences go to the prefill kernel, on another stream).
//
// Layout: one CTA of 4 warps per (b, h). A warp owns rows a = w, w+4, ...;
// lane l owns columns [VEC*l, VEC*l + VEC) of every row, so each row is one
// fully coalesced 32 * VEC * 4-byte access. Rows are processed in batches of
// ROWS loads in flight per thread before any store. The partial products
// q_a S[a][:] are reduced across the 4 warps through shared memory.
#include "kernels.h"

namespace la {
namespace {

template <int VEC> struct VecF;
template <> struct VecF<4> {
    using T = float4;
};
template <> struct VecF<2> {
    using T = float2;
};

__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ float2 ld_stream(const float2* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4* p, float4 x) { __stcs(p, x); }
__device__ __forceinline__ void st_stream(float2* p, float2 x) { __stcs(p, x); }

template <int VEC>
__device__ __forceinline__ void update(typename VecF<VEC>::T& s, float lam, float ka,
                                       const float* vv, float qa, float* acc)
{
    float* e = reinterpret_cast<float*>(&s);
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        e[i] = fmaf(lam, e[i], ka * vv[i]);
        acc[i] = fmaf(qa, e[i], acc[i]);
    }
}

template <typename Tin, typename Tout, int D, int PACKED>
__global__ void __launch_bounds__(128) decode_kernel(const Tin* __restrict__ q,
                                                     const Tin* __restrict__ k,
                                                     const Tin* __restrict__ v,
                                                     const float* __restrict__ slopes,
                                                     float* __restrict__ state, Tout* __restrict__ o,
                                                     int H, const int* __restrict__ cu,
                                                     long long total)
{
    constexpr int VEC = D / 32;
    constexpr int ROWS = 8;  // loads in flight per thread
    using V = typename VecF<VEC>::T;
    __shared__ float qs[D], ks[D];
    __shared__ float red[4][D];

    const long long p = blockIdx.x;  // b * H + h: the state's index
    long long row = p;                // the token's row in q, k, v, o
    if (PACKED) {
        const long long sq = p / H;
        if (cu[sq + 1] - cu[sq] != 1) return;
        row = (p % H) * total + cu[sq];
    }
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const float lam = expf(-slopes[p % H]);
    if (tid < D) {
        qs[tid] = to_f32(q[row * D + tid]);
        ks[tid] = to_f32(k[row * D + tid]);
    }
    float vv[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) vv[i] = to_f32(v[row * D + lane * VEC + i]);
    __syncthreads();

    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    V* S = reinterpret_cast<V*>(state + p * D * D) + lane;
    constexpr int rows_per_warp = D / 4;
#pragma unroll
    for (int r0 = 0; r0 < rows_per_warp; r0 += ROWS) {
        V s[ROWS];
#pragma unroll
        for (int j = 0; j < ROWS; ++j) s[j] = ld_stream(S + (w + 4 * (r0 + j)) * (D / VEC));
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const int a = w + 4 * (r0 + j);
            update<VEC>(s[j], lam, ks[a], vv, qs[a], acc);
            st_stream(S + a * (D / VEC), s[j]);
        }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[w][lane * VEC + i] = acc[i];
    __syncthreads();
    if (tid < D)
        o[row * D + tid] = from_f32<Tout>(red[0][tid] + red[1][tid] + red[2][tid] + red[3][tid]);
}

template <typename Tin, typename Tout, int PACKED>
cudaError_t launch(const void* q, const void* k, const void* v, const float* slopes, float* state,
                   void* o, int B, int H, int d, const int* cu, long long total,
                   cudaStream_t stream)
{
    const long long n = (long long)B * H;
    if (n == 0) return cudaSuccess;
    if (d == 128)
        decode_kernel<Tin, Tout, 128, PACKED><<<(unsigned)n, 128, 0, stream>>>(
            (const Tin*)q, (const Tin*)k, (const Tin*)v, slopes, state, (Tout*)o, H, cu, total);
    else
        decode_kernel<Tin, Tout, 64, PACKED><<<(unsigned)n, 128, 0, stream>>>(
            (const Tin*)q, (const Tin*)k, (const Tin*)v, slopes, state, (Tout*)o, H, cu, total);
    count_launch();
    return cudaGetLastError();
}

template <int PACKED>
cudaError_t dispatch(const void* q, const void* k, const void* v, const float* slopes,
                     float* state, void* o, int B, int H, int d, int in_t, int out_t,
                     const int* cu, long long total, cudaStream_t stream)
{
    if (in_t == LA_F32 && out_t == LA_F32)
        return launch<float, float, PACKED>(q, k, v, slopes, state, o, B, H, d, cu, total, stream);
    if (in_t == LA_BF16 && out_t == LA_F32)
        return launch<__nv_bfloat16, float, PACKED>(q, k, v, slopes, state, o, B, H, d, cu, total,
                                                    stream);
    if (in_t == LA_BF16 && out_t == LA_BF16)
        return launch<__nv_bfloat16, __nv_bfloat16, PACKED>(q, k, v, slopes, state, o, B, H, d, cu,
                                                            total, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* slopes,
                          float* state, void* o, int B, int H, int d, int in_t, int out_t,
                          cudaStream_t stream)
{
    return dispatch<0>(q, k, v, slopes, state, o, B, H, d, in_t, out_t, nullptr, 0, stream);
}

cudaError_t launch_decode_packed(const int* cu_seqlens, int num_seqs, const void* q,
                                 const void* k, const void* v, const float* slopes,
                                 float* states, void* o, int H, long long total, int d, int in_t,
                                 int out_t, cudaStream_t stream)
{
    return dispatch<1>(q, k, v, slopes, states, o, num_seqs, H, d, in_t, out_t, cu_seqlens, total,
                       stream);
}

}  // namespace la
