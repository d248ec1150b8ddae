// la_prefill_noalloc: the prefill for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: a plain C or embedded host
// program that has no device-memory allocator of its own, a plugin whose host
// application forbids allocations after start-up, or a latency-critical loop
// that must not call cudaMalloc (it can synchronize the whole device). This
// entry point serves them with scratch memory that the library itself owns: a
// fixed-size array in device global memory, created when the library's device
// code is loaded on a GPU and held by that GPU until the process exits.
//
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library
// routine. The work is the ordinary la_prefill, pointed at the built-in array.
#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = LA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The built-in scratch. In host code this name is only a stand-in for the
// symbol, not a device address; the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the built-in scratch on the current device, looked up
// once per device (with that device current). Returns nullptr on failure.
void* scratch_on_current_device(int* status)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        *status = LA_ERR_CUDA;
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *status = LA_ERR_UNSUPPORTED;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || ptr == nullptr) {
            *status = LA_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev] = ptr;
    }
    *status = LA_OK;
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" LA_API int la_prefill_noalloc(const void* q, const void* k, const void* v,
                                         const float* slopes, void* o, float* state_out, int B,
                                         int H, long long N, int d, int in_t, int out_t,
                                         la_stream_t stream)
{
    // Size check first, on the host: requests that need more scratch than the
    // built-in array holds are refused before anything touches the GPU.
    const size_t need = la_workspace_bytes(LA_OP_PREFILL, B, H, N, d, 0, in_t);
    if (need > kScratchBytes) return LA_ERR_WORKSPACE;
    int status = LA_OK;
    void* scratch = scratch_on_current_device(&status);
    if (scratch == nullptr) return status;
    // la_prefill clears the parts of the workspace that must start at zero
    // (status word, work ticket, per-chain scan counters) on `stream` before
    // its kernel runs; everything else is written before it is read.
    return la_prefill(q, k, v, slopes, o, state_out, B, H, N, d, in_t, out_t, scratch,
                      kScratchBytes, stream);
}

extern "C" LA_API int la_noalloc_device_status(la_stream_t stream)
{
    // The status word sits at the start of the built-in scratch, where
    // la_prefill writes device-side errors (a bounded wait that gave up). It is
    // read into a host int with a plain copy: nothing is allocated here either.
    int status = LA_OK;
    void* scratch = scratch_on_current_device(&status);
    if (scratch == nullptr) return status;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LA_ERR_CUDA;
    return word;
}
