// Internal launchers of liblightning (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace la {

// One (sequence, head) problem list, either dense [B][H][N][d] or packed
// varlen [H][total][d] with device cu_seqlens.
struct Problems {
    int H = 0;
    long long N = 0;                // dense: tokens per sequence
    int num_seqs = 0;               // dense: B; varlen: number of sequences
    const int* cu_seqlens = nullptr;  // varlen when not null
    long long total = 0;            // varlen: packed length
    int min_len = 1;                // varlen: sequences shorter than this (but not empty)
                                    // are left alone (outputs and states untouched)
    long long count() const { return (long long)num_seqs * H; }
};

// SIMT chunked forward (fp32 FFMA): the fp32 path, and the bf16 path for
// head dims the tensor-core kernel does not take. reverse != 0 runs the
// time-reversed operator O_i = sum_{j >= i} lam^(j-i) (q_i . k_j) v_j.
// state_in (may be null or equal to state_out) is the state before the first
// token of each (sequence, head).
cudaError_t launch_simt_forward(const Problems& P, const void* q, const void* k, const void* v,
                                const float* slopes, void* o, float* state_out, int d,
                                int in_t, int out_t, int block, int reverse,
                                cudaStream_t stream, const float* state_in = nullptr,
                                int state_only = 0);

// Fused single-token decode step.
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* slopes,
                          float* state, void* o, int B, int H, int d, int in_t, int out_t,
                          cudaStream_t stream);

// Incoming state of chunk r of a sequence-parallel prefill from the chunks'
// gathered local states [R][B][H][d][d] (R <= LA_MAX_CHUNKS).
cudaError_t launch_state_prefix(const float* states, const float* slopes, const long long* lens,
                                int R, int r, int B, int H, int d, float* out,
                                cudaStream_t stream);

// Output normalization and gate (RMS over each token's H*d features, then a
// sigmoid gate); O head-major [B][H][N][d], G and Y token-major [B][N][H*d].
bool norm_gate_supported(int H, int d);
cudaError_t launch_norm_gate(const void* o, const void* g, const float* w, float eps, void* y,
                             int B, int H, long long N, int d, int o_t, int g_t,
                             cudaStream_t stream);

// The decode step for the one-token sequences of a packed [H][total][d]
// batch (states [num_seqs][H][d][d]); every other sequence is left alone.
cudaError_t launch_decode_packed(const int* cu_seqlens, int num_seqs, const void* q,
                                 const void* k, const void* v, const float* slopes,
                                 float* states, void* o, int H, long long total, int d, int in_t,
                                 int out_t, cudaStream_t stream);

}  // namespace la
