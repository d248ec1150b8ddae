// C ABI of liblightning: argument checks, workspace layout, dispatch.
// The public contract of every entry point is documented in include/lightning.h.
#include <cstdint>
#include <cstring>

#include "kernels.h"
#include "tc_forward.h"

namespace la {

static thread_local int g_launches = 0;
void count_launch(int n) { g_launches += n; }

static int g_block = 0;    // fp32-path tile length, 0 = default
static int g_segment = 0;  // bf16-path scan segment length, 0 = automatic

static int default_block() { return g_block ? g_block : 64; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_dtypes(int in_t, int out_t)
{
    if (in_t != LA_BF16 && in_t != LA_F32) return LA_ERR_INVALID_ARG;
    if (out_t != LA_BF16 && out_t != LA_F32) return LA_ERR_INVALID_ARG;
    if (in_t == LA_F32 && out_t != LA_F32) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

static int check_d(int d)
{
    if (d <= 0) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

static int status_of(cudaError_t e) { return e == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

// Size limits: token coordinates reach the TMA engine as 32-bit integers and
// (sequence, head) problems are counted in 32-bit work items.
static int check_sizes(long long B_or_seqs, int H, long long tokens)
{
    if (tokens > LA_MAX_TOKENS || B_or_seqs * (long long)H > LA_MAX_PROBLEMS) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

// Whether the tcgen05 tensor-core kernel takes this request.
static bool use_tensor_cores(int in_t, int d) { return in_t == LA_BF16 && d == 128; }

static size_t workspace_for(const Problems& P, int d, int in_t, bool varlen)
{
    size_t bytes = sizeof(WsHeader);
    if (use_tensor_cores(in_t, d)) bytes += tc_workspace_bytes(P, d, g_segment, varlen);
    return bytes;
}

static int check_workspace(const void* ws, size_t ws_bytes, size_t need)
{
    if (ws == nullptr || ws_bytes < need) return LA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

// Clear the header (status, tickets) before a call that uses the workspace.
static cudaError_t clear_header(void* ws, cudaStream_t s)
{
    return cudaMemsetAsync(ws, 0, sizeof(WsHeader), s);
}

}  // namespace la

using namespace la;

extern "C" {

LA_API size_t la_workspace_bytes(int op, int B, int H, long long N_or_total, int d, int num_seqs,
                                 int in_t)
{
    if (check_d(d) != LA_OK || H <= 0 || N_or_total < 0) return 0;
    if (in_t != LA_BF16 && in_t != LA_F32) return 0;
    Problems P;
    P.H = H;
    switch (op) {
    case LA_OP_PREFILL:
    case LA_OP_BACKWARD:
        if (B <= 0) return 0;
        P.num_seqs = B;
        P.N = N_or_total;
        return workspace_for(P, d, in_t, false);
    case LA_OP_PREFILL_VARLEN:
        if (num_seqs < 0) return 0;
        P.num_seqs = num_seqs;
        P.total = N_or_total;
        P.cu_seqlens = reinterpret_cast<const int*>(16);  // marks varlen; never read here
        return workspace_for(P, d, in_t, true);
    case LA_OP_DECODE: return 0;
    default: return 0;
    }
}

namespace {

// Dense prefill, optionally continued from per-(sequence, head) states.
int prefill_dense(const void* q, const void* k, const void* v, const float* slopes,
                  const float* state_in, void* o, float* state_out, int B, int H, long long N,
                  int d, int in_t, int out_t, void* workspace, size_t ws_bytes, la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0 || N < 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(B, H, N) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((st = check_dtypes(in_t, out_t)) != LA_OK) return st;
    // With N == 0 the token tensors are empty and may be NULL.
    if (!slopes || (N > 0 && (!q || !k || !v || !o))) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(slopes) ||
        (state_out && !aligned16(state_out)) || !aligned16(state_in))
        return LA_ERR_INVALID_ARG;
    Problems P;
    P.H = H;
    P.num_seqs = B;
    P.N = N;
    if ((st = check_workspace(workspace, ws_bytes, workspace_for(P, d, in_t, false))) != LA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = status_of(clear_header(workspace, s))) != LA_OK) return st;
    if (use_tensor_cores(in_t, d))
        return status_of(launch_tc_forward(P, q, k, v, slopes, o, state_out, d, out_t, g_segment,
                                           workspace, s, 0, state_in));
    return status_of(launch_simt_forward(P, q, k, v, slopes, o, state_out, d, in_t, out_t,
                                         default_block(), 0, s, state_in));
}

// Packed variable-length prefill, optionally continued from per-(sequence, head) states.
int prefill_varlen(const int* cu_seqlens, int num_seqs, const void* q, const void* k,
                   const void* v, const float* slopes, const float* state_in, void* o,
                   float* state_out, int H, long long total, int d, int in_t, int out_t,
                   void* workspace, size_t ws_bytes, la_stream_t stream)
{
    g_launches = 0;
    if (num_seqs < 0 || H <= 0 || total < 0) return LA_ERR_INVALID_ARG;
    // Tokens without sequences would be left unwritten: the arguments disagree.
    if (num_seqs == 0 && total > 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(num_seqs, H, total) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((st = check_dtypes(in_t, out_t)) != LA_OK) return st;
    if (!cu_seqlens || !slopes || (total > 0 && (!q || !k || !v || !o)))
        return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(slopes) ||
        (state_out && !aligned16(state_out)) || !aligned16(state_in) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return LA_ERR_INVALID_ARG;
    Problems P;
    P.H = H;
    P.num_seqs = num_seqs;
    P.cu_seqlens = cu_seqlens;
    P.total = total;
    if ((st = check_workspace(workspace, ws_bytes, workspace_for(P, d, in_t, true))) != LA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = status_of(clear_header(workspace, s))) != LA_OK) return st;
    if (num_seqs == 0) return LA_OK;
    if (use_tensor_cores(in_t, d))
        return status_of(launch_tc_forward(P, q, k, v, slopes, o, state_out, d, out_t, g_segment,
                                           workspace, s, 0, state_in));
    return status_of(launch_simt_forward(P, q, k, v, slopes, o, state_out, d, in_t, out_t,
                                         default_block(), 0, s, state_in));
}

}  // namespace

LA_API int la_prefill(const void* q, const void* k, const void* v, const float* slopes, void* o,
                      float* state_out, int B, int H, long long N, int d, int in_t, int out_t,
                      void* workspace, size_t ws_bytes, la_stream_t stream)
{
    return prefill_dense(q, k, v, slopes, nullptr, o, state_out, B, H, N, d, in_t, out_t,
                         workspace, ws_bytes, stream);
}

LA_API int la_prefill_with_state(const void* q, const void* k, const void* v,
                                 const float* slopes, const float* state_in, void* o,
                                 float* state_out, int B, int H, long long N, int d, int in_t,
                                 int out_t, void* workspace, size_t ws_bytes, la_stream_t stream)
{
    if (!state_in) {
        g_launches = 0;
        return LA_ERR_INVALID_ARG;
    }
    return prefill_dense(q, k, v, slopes, state_in, o, state_out, B, H, N, d, in_t, out_t,
                         workspace, ws_bytes, stream);
}

LA_API int la_prefill_state(const void* k, const void* v, const float* slopes,
                            const float* state_in, float* state_out, int B, int H, long long N,
                            int d, int in_t, void* workspace, size_t ws_bytes, la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0 || N < 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(B, H, N) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if (in_t != LA_BF16 && in_t != LA_F32) return LA_ERR_INVALID_ARG;
    if (!slopes || !state_out || (N > 0 && (!k || !v))) return LA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(slopes) || !aligned16(state_out) ||
        !aligned16(state_in))
        return LA_ERR_INVALID_ARG;
    Problems P;
    P.H = H;
    P.num_seqs = B;
    P.N = N;
    if ((st = check_workspace(workspace, ws_bytes, workspace_for(P, d, in_t, false))) != LA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = status_of(clear_header(workspace, s))) != LA_OK) return st;
    // No query is read and no output written: k stands in for q.
    if (use_tensor_cores(in_t, d))
        return status_of(launch_tc_forward(P, k, k, v, slopes, nullptr, state_out, d, LA_F32,
                                           g_segment, workspace, s, 0, state_in, 1));
    return status_of(launch_simt_forward(P, k, k, v, slopes, nullptr, state_out, d, in_t, LA_F32,
                                         default_block(), 0, s, state_in, 1));
}

LA_API int la_prefill_varlen(const int* cu_seqlens, int num_seqs, const void* q, const void* k,
                             const void* v, const float* slopes, void* o, float* state_out, int H,
                             long long total, int d, int in_t, int out_t, void* workspace,
                             size_t ws_bytes, la_stream_t stream)
{
    return prefill_varlen(cu_seqlens, num_seqs, q, k, v, slopes, nullptr, o, state_out, H, total,
                          d, in_t, out_t, workspace, ws_bytes, stream);
}

LA_API int la_prefill_varlen_with_state(const int* cu_seqlens, int num_seqs, const void* q,
                                        const void* k, const void* v, const float* slopes,
                                        const float* state_in, void* o, float* state_out, int H,
                                        long long total, int d, int in_t, int out_t,
                                        void* workspace, size_t ws_bytes, la_stream_t stream)
{
    if (!state_in && num_seqs > 0) {  // an empty batch has no states
        g_launches = 0;
        return LA_ERR_INVALID_ARG;
    }
    return prefill_varlen(cu_seqlens, num_seqs, q, k, v, slopes, state_in, o, state_out, H, total,
                          d, in_t, out_t, workspace, ws_bytes, stream);
}

LA_API int la_mixed_step(const int* cu_seqlens, int num_seqs, const void* q, const void* k,
                         const void* v, const float* slopes, float* states, void* o, int H,
                         long long total, int d, int in_t, int out_t, void* workspace,
                         size_t ws_bytes, la_stream_t prefill_stream, la_stream_t decode_stream)
{
    g_launches = 0;
    if (num_seqs < 0 || H <= 0 || total < 0) return LA_ERR_INVALID_ARG;
    // Tokens without sequences would be left unwritten: the arguments disagree.
    if (num_seqs == 0 && total > 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(num_seqs, H, total) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((st = check_dtypes(in_t, out_t)) != LA_OK) return st;
    // An empty batch (num_seqs == 0) has no states and may pass NULL.
    if (!cu_seqlens || !slopes || (num_seqs > 0 && !states) ||
        (total > 0 && (!q || !k || !v || !o)))
        return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(slopes) ||
        !aligned16(states) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return LA_ERR_INVALID_ARG;
    Problems P;
    P.H = H;
    P.num_seqs = num_seqs;
    P.cu_seqlens = cu_seqlens;
    P.total = total;
    P.min_len = 2;  // one-token sequences go to the decode kernel
    if ((st = check_workspace(workspace, ws_bytes, workspace_for(P, d, in_t, true))) != LA_OK)
        return st;
    cudaStream_t ps = reinterpret_cast<cudaStream_t>(prefill_stream);
    cudaStream_t ds = reinterpret_cast<cudaStream_t>(decode_stream);
    if ((st = status_of(clear_header(workspace, ps))) != LA_OK) return st;
    if (num_seqs == 0) return LA_OK;
    cudaError_t e = use_tensor_cores(in_t, d)
                        ? launch_tc_forward(P, q, k, v, slopes, o, states, d, out_t, g_segment,
                                            workspace, ps, 0, states)
                        : launch_simt_forward(P, q, k, v, slopes, o, states, d, in_t, out_t,
                                              default_block(), 0, ps, states);
    if (e != cudaSuccess) return LA_ERR_CUDA;
    return status_of(launch_decode_packed(cu_seqlens, num_seqs, q, k, v, slopes, states, o, H,
                                          total, d, in_t, out_t, ds));
}

LA_API int la_output_norm_gate(const void* o, const void* gate, const float* weight, float eps,
                               void* y, int B, int H, long long N, int d, int o_t, int y_t,
                               la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0 || N < 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(B, H, N) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((o_t != LA_BF16 && o_t != LA_F32) || (y_t != LA_BF16 && y_t != LA_F32))
        return LA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 3.0e38f) return LA_ERR_INVALID_ARG;  // also rejects NaN
    if (!norm_gate_supported(H, d)) return LA_ERR_UNSUPPORTED;
    if ((long long)B * N > LA_MAX_TOKENS) return LA_ERR_UNSUPPORTED;  // one CTA per token
    if (N > 0 && (!o || !gate || !weight || !y)) return LA_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(gate) || !aligned16(weight) || !aligned16(y))
        return LA_ERR_INVALID_ARG;
    return status_of(launch_norm_gate(o, gate, weight, eps, y, B, H, N, d, o_t, y_t,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

LA_API int la_state_prefix(const float* states, const float* slopes, const long long* lens, int R,
                           int r, int B, int H, int d, float* out, la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0 || R < 1 || R > LA_MAX_CHUNKS || r < 0 || r > R) return LA_ERR_INVALID_ARG;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if (!states || !slopes || !lens || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(states) || !aligned16(slopes) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    for (int p = 0; p < R; ++p)
        if (lens[p] < 0) return LA_ERR_INVALID_ARG;
    return status_of(launch_state_prefix(states, slopes, lens, R, r, B, H, d, out,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

LA_API int la_decode(const void* q, const void* k, const void* v, const float* slopes,
                     float* state_inout, void* o, int B, int H, int d, int in_t, int out_t,
                     la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0) return LA_ERR_INVALID_ARG;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((st = check_dtypes(in_t, out_t)) != LA_OK) return st;
    if (!q || !k || !v || !slopes || !state_inout || !o) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(slopes) ||
        !aligned16(state_inout))
        return LA_ERR_INVALID_ARG;
    return status_of(launch_decode(q, k, v, slopes, state_inout, o, B, H, d, in_t, out_t,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

LA_API int la_backward(const void* dO, const void* q, const void* k, const void* v,
                       const float* slopes, void* dq, void* dk, void* dv, int B, int H,
                       long long N, int d, int in_t, int out_t, void* workspace, size_t ws_bytes,
                       la_stream_t stream)
{
    g_launches = 0;
    if (B <= 0 || H <= 0 || N < 0) return LA_ERR_INVALID_ARG;
    if (check_sizes(B, H, N) != LA_OK) return LA_ERR_UNSUPPORTED;
    int st = check_d(d);
    if (st != LA_OK) return st;
    if ((st = check_dtypes(in_t, out_t)) != LA_OK) return st;
    if (!slopes || (N > 0 && (!dO || !q || !k || !v || !dq || !dk || !dv)))
        return LA_ERR_INVALID_ARG;
    if (!aligned16(dO) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(slopes) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return LA_ERR_INVALID_ARG;
    Problems P;
    P.H = H;
    P.num_seqs = B;
    P.N = N;
    if ((st = check_workspace(workspace, ws_bytes, workspace_for(P, d, in_t, false))) != LA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = status_of(clear_header(workspace, s))) != LA_OK) return st;
    if (N == 0) return LA_OK;
    if (use_tensor_cores(in_t, d))
        return status_of(launch_tc_backward(P, dO, q, k, v, slopes, dq, dk, dv, d, out_t,
                                            g_segment, workspace, s));
    // The three gradients are the operator itself with permuted operands:
    //   dQ = forward  (q,k,v) <- (dO, V, K)
    //   dK = reversed (q,k,v) <- (V, dO, Q)
    //   dV = reversed (q,k,v) <- (K, Q, dO)
    const int blk = default_block();
    cudaError_t e = launch_simt_forward(P, dO, v, k, slopes, dq, nullptr, d, in_t, out_t, blk, 0, s);
    if (e == cudaSuccess)
        e = launch_simt_forward(P, v, dO, q, slopes, dk, nullptr, d, in_t, out_t, blk, 1, s);
    if (e == cudaSuccess)
        e = launch_simt_forward(P, k, q, dO, slopes, dv, nullptr, d, in_t, out_t, blk, 1, s);
    return status_of(e);
}

LA_API const char* la_status_string(int status)
{
    switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: unsupported request";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA error";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: device-side bounded wait gave up";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown status";
    }
}

LA_API int la_read_device_status(const void* workspace, la_stream_t stream)
{
    if (!workspace) return LA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LA_ERR_CUDA;
    int status = 0;
    if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LA_ERR_CUDA;
    return status;
}

LA_API int la_set_tuning(int block_tokens, int segment_tokens)
{
    if (block_tokens != 0 && block_tokens != 32 && block_tokens != 64 && block_tokens != 128)
        return LA_ERR_INVALID_ARG;
    if (segment_tokens < 0 || segment_tokens % 128 != 0) return LA_ERR_INVALID_ARG;
    g_block = block_tokens;
    g_segment = segment_tokens;
    return LA_OK;
}

LA_API int la_get_tuning(int* block_tokens, int* segment_tokens)
{
    if (block_tokens) *block_tokens = g_block;
    if (segment_tokens) *segment_tokens = g_segment;
    return LA_OK;
}

LA_API int la_last_launch_count(void) { return g_launches; }

LA_API int la_set_fault_injection(int skip_publish, int wait_limit_us)
{
    if (wait_limit_us < 0) return LA_ERR_INVALID_ARG;
    g_fault.skip_publish = skip_publish ? 1 : 0;
    g_fault.wait_limit_us = wait_limit_us;
    return LA_OK;
}

}  // extern "C"
