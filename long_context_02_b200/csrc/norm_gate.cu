// Output normalization and gate after lightning attention.
//
// "MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
// section 2.2: the linear-attention output passes through a normalization,
// and the blocks gate it; the page gives neither form. This library reads
// them as an RMS normalization over all H*d features of a token followed by a
// sigmoid gate:
//
//     r_{b,n}          = 1 / sqrt( mean_{h,c} O[b][h][n][c]^2 + eps )
//     Y[b][n][h d + c] = w[h d + c] * O[b][h][n][c] * r_{b,n} * sigmoid(G[b][n][h d + c])
//
// O is head-major (as the prefill writes it); G, w and Y are token-major, the
// layout of the projection that follows. The reduction of a token spans all
// H heads, which the prefill produces in H different CTAs at different times,
// so it runs as its own streaming pass rather than in the prefill's epilogue.
//
// One CTA of NT threads takes T consecutive tokens. Thread t owns the
// 8-element chunks t, t + NT, ... (MAXC of them) of each token's H*d
// features; a chunk never crosses a head row, since d is a multiple of 8.
// T * MAXC = 4 keeps the registers per thread fixed. CTAs are kept small
// (NT = 256 up to H*d = 8192, with T = 4, 2, 1 as H*d grows; NT = 512 and
// T = 1 up to 16384) so that five of them share an SM: each CTA waits at
// its one barrier at a different time, and the SM always has loads in
// flight. All loads are issued, with streaming hints, before the reduction;
// the block reduces the T sums of squares in a fixed order under one
// barrier, then every thread scales, gates and stores its chunks. Bytes per
// token: H*d*(|O| + 2|Y|) plus w, which stays in L2. The gate uses the fast
// exponential and division intrinsics, so the arithmetic stays well under
// the memory time.
#include "kernels.h"

namespace la {
namespace {

constexpr int NG_THREADS_MAX = 512;
constexpr int NG_SLOTS = 4;  // T * MAXC: H*d <= NT * 8 * 4 / T

// Eight consecutive elements held in their storage type.
template <typename T> struct Chunk8;
template <> struct Chunk8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p)
    {
        u = __ldcs(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ float get(int e) const
    {
        const uint32_t w = (&u.x)[e >> 1];
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* x)
    {
        uint4 o;
        uint32_t* ow = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            ow[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        __stcs(reinterpret_cast<uint4*>(p), o);
    }
};
template <> struct Chunk8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p)
    {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ float get(int e) const
    {
        return e < 4 ? (&a.x)[e] : (&b.x)[e - 4];
    }
    __device__ __forceinline__ static void store(float* p, const float* x)
    {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
        __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
    }
};

// sigmoid(x) = 1 / (1 + e^-x) with the fast exponential and division
// intrinsics (a few ulp; a large negative x gives e^-x = inf and a gate of 0).
__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

template <typename To, typename Tg, int NT, int T>
__global__ void __launch_bounds__(NT) norm_gate_kernel(const To* __restrict__ o,
                                                               const Tg* __restrict__ g,
                                                               const float* __restrict__ w,
                                                               float eps, Tg* __restrict__ y,
                                                               int H, long long N, int d,
                                                               long long tokens)
{
    constexpr int MAXC = NG_SLOTS / T;
    __shared__ float red[T][NT / 32];
    const long long t0 = (long long)blockIdx.x * T;
    const int F = H * d, nchunks = F / 8, cpr = d / 8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    Chunk8<To> xo[T][MAXC];
    Chunk8<Tg> xg[T][MAXC];
#pragma unroll
    for (int j = 0; j < T; ++j) {
        const long long t = t0 + j;
        if (t >= tokens) continue;
        const long long b = t / N, n = t % N;
#pragma unroll
        for (int m = 0; m < MAXC; ++m) {
            const int c = tid + NT * m;
            if (c < nchunks) {
                const int h = c / cpr, col = (c - h * cpr) * 8;
                xo[j][m].load(o + ((b * H + h) * N + n) * d + col);
                xg[j][m].load(g + t * F + 8 * c);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < T; ++j) {
        float ss = 0.f;
        if (t0 + j < tokens) {
#pragma unroll
            for (int m = 0; m < MAXC; ++m) {
                if (tid + NT * m < nchunks) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(xo[j][m].get(e), xo[j][m].get(e), ss);
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (lane == 0) red[j][warp] = ss;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < T; ++j) {
        const long long t = t0 + j;
        if (t >= tokens) continue;
        float tot = 0.f;
#pragma unroll
        for (int i = 0; i < NT / 32; ++i) tot += red[j][i];
        const float r = rsqrtf(tot / (float)F + eps);
#pragma unroll
        for (int m = 0; m < MAXC; ++m) {
            const int c = tid + NT * m;
            if (c < nchunks) {
                const float4 w0 = __ldg(reinterpret_cast<const float4*>(w + 8 * c));
                const float4 w1 = __ldg(reinterpret_cast<const float4*>(w + 8 * c) + 1);
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float out[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    out[e] = wv[e] * xo[j][m].get(e) * r * sigmoid(xg[j][m].get(e));
                Chunk8<Tg>::store(y + t * F + 8 * c, out);
            }
        }
    }
}

template <typename To, typename Tg, int NT, int T>
cudaError_t launch_t(const void* o, const void* g, const float* w, float eps, void* y,
                     long long tokens, int H, long long N, int d, cudaStream_t stream)
{
    const long long grid = (tokens + T - 1) / T;
    norm_gate_kernel<To, Tg, NT, T><<<(unsigned)grid, NT, 0, stream>>>(
        (const To*)o, (const Tg*)g, w, eps, (Tg*)y, H, N, d, tokens);
    count_launch();
    return cudaGetLastError();
}

template <typename To, typename Tg>
cudaError_t launch(const void* o, const void* g, const float* w, float eps, void* y, int B, int H,
                   long long N, int d, cudaStream_t stream)
{
    const long long tokens = (long long)B * N;
    if (tokens == 0) return cudaSuccess;
    const long long F = (long long)H * d;
    if (F <= 256 * 8) return launch_t<To, Tg, 256, 4>(o, g, w, eps, y, tokens, H, N, d, stream);
    if (F <= 256 * 16) return launch_t<To, Tg, 256, 2>(o, g, w, eps, y, tokens, H, N, d, stream);
    if (F <= 256 * 32) return launch_t<To, Tg, 256, 1>(o, g, w, eps, y, tokens, H, N, d, stream);
    return launch_t<To, Tg, 512, 1>(o, g, w, eps, y, tokens, H, N, d, stream);
}

}  // namespace

bool norm_gate_supported(int H, int d)
{
    return (long long)H * d <= (long long)NG_THREADS_MAX * NG_SLOTS * 8;
}

cudaError_t launch_norm_gate(const void* o, const void* g, const float* w, float eps, void* y,
                             int B, int H, long long N, int d, int o_t, int g_t,
                             cudaStream_t stream)
{
    if (o_t == LA_BF16 && g_t == LA_BF16)
        return launch<__nv_bfloat16, __nv_bfloat16>(o, g, w, eps, y, B, H, N, d, stream);
    if (o_t == LA_BF16 && g_t == LA_F32)
        return launch<__nv_bfloat16, float>(o, g, w, eps, y, B, H, N, d, stream);
    if (o_t == LA_F32 && g_t == LA_BF16)
        return launch<float, __nv_bfloat16>(o, g, w, eps, y, B, H, N, d, stream);
    if (o_t == LA_F32 && g_t == LA_F32)
        return launch<float, float>(o, g, w, eps, y, B, H, N, d, stream);
    return cudaErrorInvalidValue;
}

}  // namespace la
