// Global prefix of a sequence-parallel prefill (LASP+).
//
// "MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
// section 3.2: with the sequence cut into R consecutive chunks, one per rank,
// every rank summarizes its chunk locally (the chunk's own state S_p, from a
// prefill of the chunk alone), the summaries are gathered, and each rank
// builds the state before its chunk from them:
//
//     S_in(r) = sum_{p<r} ( prod_{p<q<r} alpha_q ) S_p,    alpha_q = lam^(n_q)
//
// evaluated as the recurrence acc <- alpha_p acc + S_p over p = 0..r-1. One
// thread per four consecutive state entries; the gathered states are read
// once, coalesced.
#include "kernels.h"

namespace la {
namespace {

struct PrefixArgs {
    const float* states;  // [R][P][d][d]
    const float* slopes;  // [H]
    float* out;           // [P][d][d]
    long long lens[LA_MAX_CHUNKS];
    int r, H, d;
    long long P;
};

__global__ void __launch_bounds__(256) state_prefix_kernel(const PrefixArgs a)
{
    const long long dd = (long long)a.d * a.d;
    const long long n4 = a.P * dd / 4;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const long long x = (4 * i) / dd;  // problem b * H + h
        const float slope = a.slopes[x % a.H];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p = 0; p < a.r; ++p) {
            const float al = expf(-slope * (float)a.lens[p]);
            const float4 s = reinterpret_cast<const float4*>(a.states + p * a.P * dd)[i];
            acc = make_float4(fmaf(al, acc.x, s.x), fmaf(al, acc.y, s.y), fmaf(al, acc.z, s.z),
                              fmaf(al, acc.w, s.w));
        }
        reinterpret_cast<float4*>(a.out)[i] = acc;
    }
}

}  // namespace

cudaError_t launch_state_prefix(const float* states, const float* slopes, const long long* lens,
                                int R, int r, int B, int H, int d, float* out,
                                cudaStream_t stream)
{
    PrefixArgs a{};
    a.states = states;
    a.slopes = slopes;
    a.out = out;
    for (int p = 0; p < R; ++p) a.lens[p] = lens[p];
    a.r = r;
    a.H = H;
    a.d = d;
    a.P = (long long)B * H;
    const long long n4 = a.P * d * d / 4;
    const int grid = (int)((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
    state_prefix_kernel<<<grid, 256, 0, stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace la
