// Tensor-core (tcgen05 / TMEM / TMA) lightning attention kernels for bf16
// inputs with head dim 128 on sm_100a.
#pragma once

#include <cuda_runtime.h>

#include "kernels.h"

namespace la {

// Test-only fault injection (set through la_set_fault_injection).
struct FaultInjection {
    int skip_publish = 0;   // segments never publish their prefix: successors time out
    int wait_limit_us = 0;  // bound of the inter-CTA wait (0 = default, 2 s)
};
extern FaultInjection g_fault;

// Workspace bytes after the header: per-chain flags, two inclusive-prefix
// state slots per chain, and (varlen) the planned work items.
size_t tc_workspace_bytes(const Problems& P, int d, int seg_tuning, bool varlen);

// Forward prefill (dense or varlen). reverse != 0 runs the time-reversed
// operator (used by the backward pass). state_in (forward only, may be null or
// equal to state_out): per (sequence, head) state before the first token.
// state_only != 0 writes the final states alone (o is not written; q unused).
cudaError_t launch_tc_forward(const Problems& P, const void* q, const void* k, const void* v,
                              const float* slopes, void* o, float* state_out, int d, int out_t,
                              int seg_tuning, void* workspace, cudaStream_t stream,
                              int reverse = 0, const float* state_in = nullptr,
                              int state_only = 0);

// Backward: dQ by the forward operator on (dO, V, K); dK and dV by the
// time-reversed operator on (V, dO, Q) and (K, Q, dO).
cudaError_t launch_tc_backward(const Problems& P, const void* dO, const void* q, const void* k,
                               const void* v, const float* slopes, void* dq, void* dk, void* dv,
                               int d, int out_t, int seg_tuning, void* workspace,
                               cudaStream_t stream);

}  // namespace la
