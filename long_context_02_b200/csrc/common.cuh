// Shared device/host helpers of liblightning (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lightning.h"

namespace la {

// Element loads/stores with conversion to and from fp32.
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x)
{
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

// Workspace header shared by every kernel that takes a workspace. It sits at
// the start of the caller's workspace; the host clears it before each call.
struct WsHeader {
    int status;        // la_status of device-side failures (0 = ok)
    int ticket;        // dynamic work-item counter of persistent kernels
    int num_items;     // number of work items (written by the varlen planner)
    int timeout_item;  // first item whose bounded wait gave up (-1 if none)
    int pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte line");

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch accounting (per host thread), reported by la_last_launch_count().
void count_launch(int n = 1);

}  // namespace la
