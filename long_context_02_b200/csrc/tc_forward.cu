// Lightning attention on the sm_100a tensor cores: tcgen05 MMAs with TMEM
// accumulators, TMA-staged bf16 tiles, a chunk-parallel scan of the state
// across segments, head dim 128.
//
// What is computed (per (sequence, head) "chain", decay lam = exp(-slope)):
//   O_i = sum_{j<=i} lam^(i-j) (q_i . k_j) v_j,   final state sum_j lam^(N-1-j) k_j^T v_j.
// "MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary":
//   section 2.2 - tiles: a masked intra-tile product plus the product with the
//                 accumulated key-value state, which is then updated;
//   section 3.2 - LASP+: each partition summarizes its keys/values locally and
//                 the summaries combine into prefixes, so partitions need not
//                 wait for the serial pass before them;
//   section 3.3 - tiled prefill on batched matmuls (here tcgen05).
//
// Work decomposition. The value dimension is split in two halves of 64
// columns: O[:, half] and state[:, half] need only V[:, half], so each
// (chain, half) is an independent problem with its own 128 x 64 state. A
// chain is also cut into segments of SEG tokens (a multiple of the 128-token
// block; one segment when there are enough chains to fill the GPU). A work
// item is one (chain, half, segment). Persistent CTAs (one per SM) take items
// from an atomic ticket in segment-major order, so an item's predecessor in
// its chain always holds a smaller ticket and is already running or done.
// For each item:
//   phase A (only if a later segment needs it): the segment's local state
//     S_loc = sum_j lam^(len-1-j) k_j^T v_j, accumulated in TMEM over the
//     segment's blocks; then a bounded wait for the predecessor's inclusive
//     prefix S_prev and a publish of lam^len S_prev + S_loc: the scan combine
//     (a1, S1) o (a2, S2) = (a1 a2, a2 S1 + S2).
//   phase C: the segment's blocks from S = S_prev. Per 128-token block:
//     MMA1  SP  = Q K^T                    (fp32, TMEM)
//     E_P   P   = SP * lam^(i-j) [j<=i]     written back into TMEM as bf16 hi + lo
//     MMA2  OI  = P_hi V + P_lo V           (A operand from TMEM)
//     MMA3  [OE_hi | OE_lo] = Q [S_hi | S_lo]   (bf16 hi + lo copies of the fp32 state,
//                                              side by side: one N = 128 MMA per k-step)
//     E_O   O   = OI + lam^(i+1) (OE_hi + OE_lo)  -> global (bf16 or fp32)
//     E_V   Vd  = lam^(L-1-j) v_j           (bf16 hi + lo, shared memory)
//     MMA4  DS  = K^T Vd_hi + K^T Vd_lo
//     E_S   S   = lam^L S + DS              (fp32 in registers; hi + lo copies for MMA3)
// Only non-negative decay exponents appear, so nothing overflows; terms that
// underflow are below fp32 resolution of the result.
//
// Precision. Q, K and V enter the MMAs exactly as given (bf16). Every operand
// the kernel forms itself (P, the state copy, the decayed values) is split as
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): a relative error of about
// 2^-16, with fp32's exponent range, so no scaling is needed anywhere. One
// bf16 rounding of any of those three operands would cost about 1e-2 of the
// output's rms; the split costs a second MMA for each.
//
// Warp roles (16 warps, 4 warpgroups): warp 0 TMA producer, warp 1 MMA issuer
// (also owns TMEM); warps 4-7 "P" (E_P); warps 8-11 "VO" (E_V, E_O); warps
// 12-15 "S" (E_S and the scan; the fp32 state lives in their registers, one
// key row a per thread). TMEM: 512 columns = SP[2] | OI | DS | OE, with OE
// holding [OE_hi | OE_lo].
//
// Shared memory is the resource every step competes for: the MMAs' operand
// reads (both operands of the smem-operand forms), the TMA writes and the
// epilogues' loads and stores all share its 128 bytes per clock, and an
// mbarrier probe queues behind them. Hence MMA3 reads Q once for both state
// copies (N = 128), and the MMA warp probes every barrier a group needs at
// once (wait_multi), so that MMA4 and MMA3 issue back to back.
// Shared memory: two slots each for Q, K (128 x 128) and V (128 x 64), the
// decayed values (hi, lo) and the state copies (hi, lo), all in the 128-byte
// swizzled layout TMA writes.
//
// The kernel has three modes (template MODE): general (0), the state-only
// pass (1), and one segment per chain (2: no phase A, no scan, used by dense
// problems whose chains fill the GPU). Each is its own instantiation, so no
// mode carries another's code. The state-only pass (final states, no
// outputs) runs phase A alone: it keeps three K and V stages (using the
// Q slot and state-copy buffer it leaves idle), two decayed-value buffers,
// and one N = 128 MMA4 per k-step over [Vd_hi | Vd_lo] whose halves
// accumulate apart in the idle score columns. The phase A of a segmented
// chain does the same with two stages (its Q slot 0 holds the second
// decayed-value buffer until phase A's MMAs are done, then phase C's Q).
// Phase A prefetches its K and V tiles into L2 a few blocks ahead.
//
// Every wait is bounded: an mbarrier wait gives up after 4 s, the inter-CTA
// wait after 2 s; either records LA_ERR_TIMEOUT in the workspace header and
// the CTA winds down (waiting, bounded, for its own copies and MMAs in
// flight, then freeing TMEM).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tc_forward.h"

namespace la {
namespace tc {

constexpr int D = 128;                           // head dim (d_k = d_v)
constexpr int DV = 64;                           // value columns per work item
constexpr int C = 128;                           // tokens per block
constexpr int NUM_THREADS = 512;                 // 4 warpgroups
// Register split (setmaxnreg, which ptxas also uses to allocate each role):
// launched at 65536 / 512 = 128 per thread. 128 * (104 + 120 + 128 + 152) =
// 64512 <= 65536.
constexpr int REGS_CTRL = 104, REGS_P = 120, REGS_VO = 128, REGS_S = 152;
static_assert(128 * (REGS_CTRL + REGS_P + REGS_VO + REGS_S) <= 65536, "register split");
constexpr uint32_t BOX_BYTES = 128 * 64 * 2;     // one TMA box: 128 rows x 64 bf16
constexpr uint32_t TILE_BYTES = 2 * BOX_BYTES;   // 128 x 128 bf16
// Tile region (1024-aligned).
constexpr uint32_t OFF_Q = 0;                          // 2 x 32 KB
constexpr uint32_t OFF_K = OFF_Q + 2 * TILE_BYTES;     // 2 x 32 KB
constexpr uint32_t OFF_V = OFF_K + 2 * TILE_BYTES;     // 2 x 16 KB
constexpr uint32_t OFF_VH = OFF_V + 2 * BOX_BYTES;     // decayed values, hi
constexpr uint32_t OFF_VL = OFF_VH + BOX_BYTES;        // decayed values, lo
constexpr uint32_t OFF_SH = OFF_VL + BOX_BYTES;        // state copy, hi
constexpr uint32_t OFF_SL = OFF_SH + BOX_BYTES;        // state copy, lo
constexpr uint32_t SMEM_TILES = OFF_SL + BOX_BYTES;    // 224 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_SP = 0, COL_OI = 256, COL_DS = 320, COL_OE = 384;  // OE: 128 columns
constexpr int PREFETCH_AHEAD = 3;  // phase A: blocks between an L2 prefetch and its load
constexpr unsigned long long WAIT_LIMIT_NS = 4000000000ull;
constexpr unsigned long long FLAG_LIMIT_NS = 2000000000ull;
constexpr unsigned long long DRAIN_LIMIT_NS = 200000000ull;

// Barriers. A waiter must never fall two phases behind its barrier (a parity
// wait would then return at once or hang), so every resource that can be
// two uses ahead of its consumer has one barrier per buffer.
enum {
    B_QF0, B_QF1, B_QE0, B_QE1,      // Q slots: loaded / released (after MMA3)
    B_KF0, B_KF1, B_KE0, B_KE1,      // K slots: loaded / released (after MMA4)
    B_VF0, B_VF1, B_VE0, B_VE1,      // V slots: loaded / released (after MMA2)
    B_SP_FULL0, B_SP_FULL1,          // MMA1 done -> E_P
    B_P_READY0, B_P_READY1,          // E_P done -> MMA2
    B_VH_FREE, B_VH_READY,           // decayed values: MMA4 done / E_V done
    B_VHA_READY,                     // phase A: E_V done by the VO, P and S groups together
    B_VH_FREE1, B_VHA_READY1,        // the second decayed-value buffer (phase A)
    B_DS_FULL, B_DS_EMPTY,           // DS: MMA4 done / E_S read it
    B_S_FREE, B_S_READY,             // state copy: MMA3 done / E_S wrote it
    B_O_FULL, B_O_EMPTY,             // OI: MMA2 done / E_O read it
    B_OE_FREE,                       // OE: E_O read it (MMA3 may write it)
    B_ITEM_FULL0, B_ITEM_FULL1, B_ITEM_EMPTY0, B_ITEM_EMPTY1,
    B_FIN, B_P_SYNC, B_S_SYNC,
    B_KF2, B_KE2, B_VF2, B_VE2,      // third K and V stage (state-only pass)
    B_A_DONE,                        // a segment's phase A MMAs done: Q slot 0 is free again
    NUM_BARS
};

// tcgen05 instruction descriptors (kind::f16): D fp32, M = 128, A and B bf16.
// bits: [4,6) D format (1 = f32), [7,10) A format and [10,13) B format
// (1 = bf16), 15 A major, 16 B major (0 = K-major, 1 = MN-major),
// [17,23) N >> 3, [24,29) M >> 4.
constexpr uint32_t idesc(uint32_t n, uint32_t a_mn_major, uint32_t b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
           ((n >> 3) << 17) | ((128u >> 4) << 24);
}
constexpr uint32_t IDESC_QK = idesc(128, 0, 0);  // Q K^T: both K-major
constexpr uint32_t IDESC_PV = idesc(64, 0, 1);   // P (TMEM) V: V MN-major
constexpr uint32_t IDESC_QS = idesc(128, 0, 1);  // Q [S_hi | S_lo]: rows = key dim, MN-major
constexpr uint32_t IDESC_KV = idesc(64, 1, 1);   // K^T Vd: both MN-major
constexpr uint32_t IDESC_KV2 = idesc(128, 1, 1);  // K^T [Vd_hi | Vd_lo] (state-only pass)

struct Params {
    int H;
    int nchains;        // dense: B*H
    int nseg;           // dense: segments per chain
    int seg_tokens;
    long long N;        // dense: tokens per chain
    const int* cu_seqlens;  // varlen when not null
    long long total;
    const int4* items;  // varlen: planned (chain, p_ord, nseg) per (chain, segment)
    int num_items_dense;
    const float* slopes;
    void* o;
    float* state_out;
    const float* state_in;  // [chains][D][D] state before token 0 (null: zero), forward only
    int reverse;
    WsHeader* hdr;
    int* chain_flags;   // per (chain, half): segments published so far
    float* incl;        // [chains][2 halves][2 slots][D][DV] inclusive prefixes
    unsigned long long flag_limit_ns;  // bound of the inter-CTA wait
    int skip_publish;   // fault injection (tests): never raise the chain counters
};

struct Item {
    int valid;
    int chain;
    int half;           // value columns [64 half, 64 half + 64)
    int head;
    int p_ord;          // position in the chain's processing order
    int nseg;
    int len;            // tokens in the segment
    int z;              // TMA coordinate 2
    int y0;             // TMA coordinate 1 of the segment's first token
    long long out_row0; // flat [rows][D] row of the segment's first token
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait. Gives up (returning false) when another role aborted, or
// after `limit` ns, in which case it records the timeout and raises the
// CTA-wide abort flag.
__device__ __forceinline__ bool mbar_wait_slow(uint64_t* b, uint32_t parity, volatile int* abort,
                                            WsHeader* hdr, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 63) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit) {
                *abort = 1;
                atomicExch(&hdr->status, (int)LA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort,
                                          WsHeader* hdr,
                                          unsigned long long limit = WAIT_LIMIT_NS)
{
    if (mbar_try_wait(b, parity)) return true;
    return mbar_wait_slow(b, parity, abort, hdr, limit);
}

// Warp-uniform bounded wait: every lane polls, and the warp proceeds only if
// all lanes saw the phase complete.
__device__ __forceinline__ bool wait_warp(uint64_t* b, uint32_t parity, volatile int* abort,
                                          WsHeader* hdr)
{
    const bool ok = mbar_wait(b, parity, abort, hdr);
    return __all_sync(0xffffffffu, ok);
}

// Warp-uniform bounded wait on up to three barriers at once: lane i probes
// barrier i (lanes past n probe barrier 0), so the probes go out together
// instead of one round trip each.
__device__ __forceinline__ bool wait_multi(int n, uint64_t* b0, uint32_t p0, uint64_t* b1,
                                           uint32_t p1, uint64_t* b2, uint32_t p2, int lane,
                                           volatile int* abort, WsHeader* hdr)
{
    uint64_t* b = (lane == 1 && n > 1) ? b1 : (lane == 2 && n > 2) ? b2 : b0;
    const uint32_t par = (lane == 1 && n > 1) ? p1 : (lane == 2 && n > 2) ? p2 : p0;
    if (__all_sync(0xffffffffu, mbar_try_wait(b, par))) return true;
    return __all_sync(0xffffffffu, mbar_wait_slow(b, par, abort, hdr, WAIT_LIMIT_NS));
}

// Bounded barrier over one 128-thread group (an mbarrier of count 128).
__device__ __forceinline__ bool group_sync(uint64_t* b, uint32_t& n, volatile int* abort,
                                           WsHeader* hdr)
{
    mbar_arrive(b);
    return wait_warp(b, n++ & 1, abort, hdr);
}

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One lane of a converged warp (the lowest active lane: lane 0 here).
__device__ __forceinline__ bool elect_one()
{
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}

// Brings a tile into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z,
                                                uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.prefetch.tensor.3d.L2.global.tile.L2::cache_hint [%0, {%1, %2, %3}], %4;" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Pack two fp32 into bf16x2 (round to nearest even); `lo` goes to the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Pairs of fp32 in one 64-bit register for the packed f32x2 instructions.
__device__ __forceinline__ uint64_t f2(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2u(uint32_t a, uint32_t b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ float f2x(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2y(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// bf16x2 word -> fp32 pair (exact).
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) { return f2u(w << 16, w & 0xffff0000u); }

// Pair x -> (hi, lo) bf16x2 words with x = hi + lo to about 2^-16 relative.
__device__ __forceinline__ void split_pair(uint64_t x, uint32_t& hi, uint32_t& lo)
{
    hi = pack_bf16x2(f2x(x), f2y(x));
    const uint64_t d = sub2(x, bf2_to_f2(hi));
    lo = pack_bf16x2(f2x(d), f2y(d));
}

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 version bit.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ int num_blocks(int len) { return (len + C - 1) / C; }

// Segment offset of the k-th block in processing order.
__device__ __forceinline__ int block_t0(int len, int k, int rev)
{
    const int nb = num_blocks(len);
    return (rev ? nb - 1 - k : k) * C;
}

// Offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)r * 128u + ((uint32_t)((c ^ r) & 7) << 4);
}

// Ordered L2 loads/stores (volatile asm keeps their program order).
__device__ __forceinline__ float4 ld_cg_ordered(const float* p)
{
    float4 w;
    asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(w.x), "=f"(w.y), "=f"(w.z), "=f"(w.w)
                 : "l"(p)
                 : "memory");
    return w;
}
__device__ __forceinline__ void st_cg_ordered(float* p, float4 w)
{
    asm volatile("st.global.cg.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(w.x), "f"(w.y),
                 "f"(w.z), "f"(w.w)
                 : "memory");
}

// ------------------------------------------------------------------ work items

// Ticket t -> (chain, half, segment). Halves of one (chain, segment) take
// adjacent tickets, so they run side by side and share Q and K in L2.
__device__ Item make_item(const Params& p, int t, int num_items)
{
    Item it{};
    it.valid = 0;
    if (t >= num_items) return it;
    const int base = t >> 1;
    it.half = t & 1;
    int chain, p_ord, nseg;
    long long seq_start, seq_len, rowbase;
    if (p.cu_seqlens == nullptr) {
        p_ord = base / p.nchains;
        chain = base % p.nchains;
        nseg = p.nseg;
        it.head = chain % p.H;
        it.z = chain;
        seq_start = 0;
        seq_len = p.N;
        rowbase = (long long)chain * p.N;
    } else {
        const int4 w = p.items[base];
        chain = w.x;
        p_ord = w.y;
        nseg = w.z;
        const int s = chain / p.H;
        it.head = chain % p.H;
        it.z = it.head;
        seq_start = p.cu_seqlens[s];
        seq_len = (long long)p.cu_seqlens[s + 1] - seq_start;
        rowbase = (long long)it.head * p.total;
    }
    const int seg = p.reverse ? nseg - 1 - p_ord : p_ord;
    const long long off = (long long)seg * p.seg_tokens;
    it.valid = 1;
    it.chain = chain;
    it.p_ord = p_ord;
    it.nseg = nseg;
    it.len = (int)min((long long)p.seg_tokens, seq_len - off);
    it.y0 = (int)(seq_start + off);
    it.out_row0 = rowbase + seq_start + off;
    return it;
}

// ------------------------------------------------------------------ roles

struct Smem {
    uint8_t* tiles;  // 1024-aligned tile region
    uint64_t* bars;
    Item* ring;
    volatile int* abort;
    float* pw;       // [C+1] lam^m of the P group's current item
    __device__ uint8_t* q(int s) const { return tiles + OFF_Q + s * TILE_BYTES; }
    __device__ uint8_t* k(int s) const { return tiles + OFF_K + s * TILE_BYTES; }
    __device__ uint8_t* v(int s) const { return tiles + OFF_V + s * BOX_BYTES; }
    // The state-only pass's three K and V stages: stage 2 uses Q slot 1 and the
    // state-copy buffer, which that pass leaves idle.
    __device__ uint8_t* k3(uint32_t s) const { return s < 2 ? k((int)s) : tiles + OFF_Q + TILE_BYTES; }
    __device__ uint8_t* v3(uint32_t s) const { return s < 2 ? v((int)s) : tiles + OFF_SH; }
    __device__ uint8_t* vh() const { return tiles + OFF_VH; }
    __device__ uint8_t* vl() const { return tiles + OFF_VL; }
    __device__ uint8_t* sh() const { return tiles + OFF_SH; }
    __device__ uint8_t* sl() const { return tiles + OFF_SL; }
    // Phase A loads no Q: Q slot 0 holds a second decayed-value buffer (hi,
    // lo), so that E_V of one block overlaps MMA4 of the previous. (A
    // segmented chain's phase C takes the slot back once phase A is done.)
    __device__ uint8_t* vh1() const { return tiles + OFF_Q; }
    __device__ uint8_t* vl1() const { return tiles + OFF_Q + BOX_BYTES; }
};

// Reads the next item from the ring (all roles see the same sequence).
__device__ __forceinline__ bool next_item(const Params& p, const Smem& sm, uint32_t k, Item& it,
                                          bool warp_wide, int lane)
{
    const int slot = k & 1;
    const bool ok = warp_wide ? wait_warp(&sm.bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)
                              : mbar_wait(&sm.bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr);
    if (!ok) return false;
    it = sm.ring[slot];
    if (warp_wide) __syncwarp();
    if (!warp_wide || lane == 0) mbar_arrive(&sm.bars[B_ITEM_EMPTY0 + slot]);
    return it.valid != 0;
}

// K and V stages: two, or three in the state-only pass. Use u of a tile
// goes to stage u % n with phase (u / n) & 1.
template <int SO> __device__ __forceinline__ constexpr uint32_t num_stages() { return SO ? 3u : 2u; }
__device__ __forceinline__ int kf_bar(uint32_t s) { return s < 2 ? B_KF0 + (int)s : B_KF2; }
__device__ __forceinline__ int ke_bar(uint32_t s) { return s < 2 ? B_KE0 + (int)s : B_KE2; }
__device__ __forceinline__ int vf_bar(uint32_t s) { return s < 2 ? B_VF0 + (int)s : B_VF2; }
__device__ __forceinline__ int ve_bar(uint32_t s) { return s < 2 ? B_VE0 + (int)s : B_VE2; }

// Producer warp: TMA loads (one elected lane issues; the warp waits together).
template <int MODE>
__device__ void producer_role(const Params& p, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv, const Smem& sm, int lane)
{
    constexpr bool SO = MODE == 1, ONE = MODE == 2;
    uint64_t* bars = sm.bars;
    const int num_items = 2 * (p.cu_seqlens ? *reinterpret_cast<volatile int*>(&p.hdr->num_items)
                                            : p.num_items_dense);
    // K and V read in phase A are read again in phase C: keep them in L2. Q
    // and K are read by both halves of a chain; V only by its own half.
    const uint64_t keep = l2_policy_evict_last(), normal = l2_policy_evict_normal(),
                   drop = l2_policy_evict_first();
    // nk, nv, nq: K, V and Q loads issued (K and V always come in pairs).
    uint32_t nq = 0, nk = 0, nv = 0, n_a = 0;
    const uint32_t NS = num_stages<SO>();
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
        const int slot = k & 1;
        if (!wait_warp(&bars[B_ITEM_EMPTY0 + slot], ((k >> 1) & 1) ^ 1, sm.abort, p.hdr)) break;
        int t = 0;
        if (lane == 0) t = atomicAdd(&p.hdr->ticket, 1);
        t = __shfl_sync(0xffffffffu, t, 0);
        const Item it = make_item(p, t, num_items);
        if (lane == 0) {
            sm.ring[slot] = it;
            mbar_arrive(&bars[B_ITEM_FULL0 + slot]);
        }
        __syncwarp();
        if (!it.valid) break;
        const int nb = num_blocks(it.len);
        const bool has_succ = !ONE && it.p_ord < it.nseg - 1;
        // Phase A (pass 0) loads K and V; phase C (pass 1) loads Q, K and V.
        const int last_pass = SO ? 1 : 2;
        for (int pass = (has_succ || SO) ? 0 : 1; pass < last_pass && ok; ++pass) {
            // (a state-only pass reads K and V once)
            const bool again = pass == 0 && !SO;
            const uint64_t kpol = again ? keep : normal, vpol = again ? keep : drop;
            for (int kb = 0; kb < nb && ok; ++kb) {
                const int y = it.y0 + block_t0(it.len, kb, p.reverse);
                // Phase A's blocks are short (E_V and MMA4 only), and two slots
                // per tile then cover less than the DRAM latency: bring the
                // tiles of a later block into L2 first. (In phase C the same
                // prefetch costs more than it saves.)
                if (pass == 0 && kb + PREFETCH_AHEAD < nb && elect_one()) {
                    const int yp = it.y0 + block_t0(it.len, kb + PREFETCH_AHEAD, p.reverse);
                    tma_prefetch_3d(tk, 0, yp, it.z, kpol);
                    tma_prefetch_3d(tk, 64, yp, it.z, kpol);
                    tma_prefetch_3d(tv, DV * it.half, yp, it.z, normal);
                }
                __syncwarp();
                if (SO) {
                    // Three K and V stages.
                    const uint32_t s3 = nk % 3, ph = (nk / 3) & 1;
                    ok = wait_warp(&bars[ke_bar(s3)], ph ^ 1, sm.abort, p.hdr) &&
                         wait_warp(&bars[ve_bar(s3)], ph ^ 1, sm.abort, p.hdr);
                    if (!ok) break;
                    if (elect_one()) {
                        mbar_expect_tx(&bars[kf_bar(s3)], TILE_BYTES);
                        tma_load_3d(sm.k3(s3), tk, &bars[kf_bar(s3)], 0, y, it.z, kpol);
                        tma_load_3d(sm.k3(s3) + BOX_BYTES, tk, &bars[kf_bar(s3)], 64, y, it.z, kpol);
                        mbar_expect_tx(&bars[vf_bar(s3)], BOX_BYTES);
                        tma_load_3d(sm.v3(s3), tv, &bars[vf_bar(s3)], DV * it.half, y, it.z, vpol);
                    }
                    __syncwarp();
                    ++nk;
                    ++nv;
                    continue;
                }
                const int s = nk & 1;
                ok = wait_warp(&bars[B_KE0 + s], ((nk >> 1) & 1) ^ 1, sm.abort, p.hdr);
                if (!ok) break;
                if (elect_one()) {
                    mbar_expect_tx(&bars[B_KF0 + s], TILE_BYTES);
                    tma_load_3d(sm.k(s), tk, &bars[B_KF0 + s], 0, y, it.z, kpol);
                    tma_load_3d(sm.k(s) + BOX_BYTES, tk, &bars[B_KF0 + s], 64, y, it.z, kpol);
                }
                __syncwarp();
                ++nk;
                if (pass == 1) {
                    // Phase A kept its second decayed-value buffer in Q slot 0.
                    if (kb == 0 && has_succ) {
                        ok = wait_warp(&bars[B_A_DONE], n_a & 1, sm.abort, p.hdr);
                        ++n_a;
                        if (!ok) break;
                    }
                    const int sq = nq & 1;
                    ok = wait_warp(&bars[B_QE0 + sq], ((nq >> 1) & 1) ^ 1, sm.abort, p.hdr);
                    if (!ok) break;
                    if (elect_one()) {
                        mbar_expect_tx(&bars[B_QF0 + sq], TILE_BYTES);
                        tma_load_3d(sm.q(sq), tq, &bars[B_QF0 + sq], 0, y, it.z, normal);
                        tma_load_3d(sm.q(sq) + BOX_BYTES, tq, &bars[B_QF0 + sq], 64, y, it.z, normal);
                    }
                    __syncwarp();
                    ++nq;
                }
                ok = wait_warp(&bars[B_VE0 + s], ((nv >> 1) & 1) ^ 1, sm.abort, p.hdr);
                if (!ok) break;
                if (elect_one()) {
                    mbar_expect_tx(&bars[B_VF0 + s], BOX_BYTES);
                    tma_load_3d(sm.v(s), tv, &bars[B_VF0 + s], DV * it.half, y, it.z, vpol);
                }
                __syncwarp();
                ++nv;
            }
        }
    }
    if (*sm.abort) {
        // Wind down: let this CTA's copies in flight land before it exits
        // (the last use of each slot; earlier uses completed before it).
        volatile int never = 0;
        for (uint32_t u = (nk > NS ? nk - NS : 0); u < nk; ++u)
            mbar_wait(&bars[kf_bar(u % NS)], (u / NS) & 1, &never, p.hdr, DRAIN_LIMIT_NS);
        for (uint32_t u = (nv > NS ? nv - NS : 0); u < nv; ++u)
            mbar_wait(&bars[vf_bar(u % NS)], (u / NS) & 1, &never, p.hdr, DRAIN_LIMIT_NS);
        for (uint32_t u = (nq > 2 ? nq - 2 : 0); u < nq; ++u)
            mbar_wait(&bars[B_QF0 + (u & 1)], (u >> 1) & 1, &never, p.hdr, DRAIN_LIMIT_NS);
    }
}

// K-step offsets of shared-memory descriptors, in the descriptor's 16-byte
// address units: K-major tiles (two 64-column boxes, 32 bytes per k-step
// inside a box) and MN-major tiles (16 rows of 128 bytes per k-step).
__device__ __forceinline__ uint64_t koff_k(int ks)
{
    return (uint64_t)((ks >> 2) * (BOX_BYTES >> 4) + (ks & 3) * 2);
}
__device__ __forceinline__ uint64_t koff_mn(int ks) { return (uint64_t)(ks * 128); }

// MMA warp: the whole warp waits; one elected lane (lane 0, the warp being
// converged) issues every MMA and commit, so that each commit tracks all
// earlier MMAs. Descriptors are built once; each MMA adds a constant k-step
// offset, which keeps the issue loop short.
template <int MODE>
__device__ void mma_role(const Params& p, const Smem& sm, uint32_t tmem, int lane)
{
    constexpr bool SO = MODE == 1, ONE = MODE == 2;
    uint64_t* bars = sm.bars;
    // Slot s's tile is slot 0's plus a fixed distance, so one base per tensor.
    const uint64_t dq0 = sdesc(smem_u32(sm.q(0)), 16u, 1024u);
    const uint64_t dk0 = sdesc(smem_u32(sm.k(0)), 16u, 1024u);
    const uint64_t dkm0 = sdesc(smem_u32(sm.k(0)), BOX_BYTES, 1024u);
    const uint64_t dv0 = sdesc(smem_u32(sm.v(0)), 16u, 1024u);
    const uint64_t dvh = sdesc(smem_u32(sm.vh()), 16u, 1024u);
    const uint64_t dsh = sdesc(smem_u32(sm.sh()), BOX_BYTES, 1024u);  // [S_hi | S_lo], N = 128
    constexpr uint64_t TILE16 = TILE_BYTES >> 4, BOX16 = BOX_BYTES >> 4;
    // nq, nkv: Q / K-V loads consumed; g: phase-C blocks; n_ds: DS productions;
    // n_vh: decayed-value tiles; n_s: state copies.
    uint32_t nq = 0, nkv = 0, g = 0, n_ds = 0, n_vh = 0, n_s = 0, n_vha = 0, n_vha1 = 0;
    auto commit = [&](int bar) {
        if (elect_one()) mma_commit(&bars[bar]);
        __syncwarp();
    };
    // Phase C: DS = K^T Vd (hi and lo) for the K tile in slot sk. Phase A uses
    // mma4s; keeping this copy separate keeps its descriptors constants in
    // the issue loop.
    auto mma4 = [&](int sk, bool accumulate) {
        const uint64_t a = dkm0 + (uint64_t)sk * TILE16;
        const uint32_t d = tmem + COL_DS;
        const uint32_t acc0 = accumulate ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(d, a + koff_mn(ks), dvh + part * BOX16 + koff_mn(ks), IDESC_KV,
                           (part || ks) ? 1u : acc0);
        }
        __syncwarp();
    };
    // Phase A: K stage sk (of three in the state-only pass, else two) and
    // decayed-value buffer vb, one N = 128 MMA per k-step over
    // [Vd_hi | Vd_lo] (adjacent boxes), so K^T is read once; the two 64-column
    // halves accumulate apart in the score columns, free until phase C's
    // first MMA1, and E_S adds them. (Its descriptors are built here, not kept
    // live through phase C.)
    auto mma4s = [&](uint32_t sk, int vb, bool accumulate) {
        const uint64_t a = sdesc(smem_u32(sm.k3(sk)), BOX_BYTES, 1024u);
        const uint64_t b = sdesc(smem_u32(vb ? sm.vh1() : sm.vh()), BOX_BYTES, 1024u);
        const uint32_t d = tmem + COL_SP;
        const uint32_t acc0 = accumulate ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(d, a + koff_mn(ks), b + koff_mn(ks), IDESC_KV2, ks ? 1u : acc0);
        }
        __syncwarp();
    };
    // SP[g & 1] = Q K^T for phase-C block g (Q slot nq, K slot nkv).
    auto mma1 = [&](uint32_t gg, uint32_t q_use, uint32_t kv_use) -> bool {
        const int sq = q_use & 1, sk = kv_use & 1;
        if (!wait_multi(2, &bars[B_QF0 + sq], (q_use >> 1) & 1, &bars[B_KF0 + sk],
                        (kv_use >> 1) & 1, nullptr, 0, lane, sm.abort, p.hdr))
            return false;
        tc_fence_after();
        const uint64_t a = dq0 + (uint64_t)sq * TILE16, b = dk0 + (uint64_t)sk * TILE16;
        const uint32_t d = tmem + COL_SP + 128u * (gg & 1);
        if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(d, a + koff_k(ks), b + koff_k(ks), IDESC_QK, ks > 0 ? 1u : 0u);
            mma_commit(&bars[B_SP_FULL0 + (gg & 1)]);
        }
        __syncwarp();
        return true;
    };
    Item it;
    for (uint32_t k = 0;; ++k) {
        if (!next_item(p, sm, k, it, true, lane)) break;
        const int nb = num_blocks(it.len);
        const bool has_succ = !ONE && it.p_ord < it.nseg - 1;
        bool ok = true;
        if (has_succ || SO) {
            // Phase A: DS accumulates the segment's local state over its blocks.
            const uint32_t NS = num_stages<SO>();
            // The second decayed-value buffer is Q slot 0, which the previous
            // item's MMA1 and MMA3 may still read: one more phase of its free
            // barrier, completing after every MMA issued so far.
            if (!SO) commit(B_VH_FREE1);
            for (int kb = 0; kb < nb && ok; ++kb) {
                const uint32_t sk = nkv % NS;
                // Phase A alternates the two decayed-value buffers.
                const bool second = (kb & 1) != 0;
                uint32_t& reads = second ? n_vha1 : n_vha;
                ok = wait_warp(&bars[kf_bar(sk)], (nkv / NS) & 1, sm.abort, p.hdr) &&
                     wait_warp(&bars[second ? B_VHA_READY1 : B_VHA_READY], reads & 1, sm.abort,
                               p.hdr) &&
                     (kb > 0 || wait_warp(&bars[B_DS_EMPTY], (n_ds & 1) ^ 1, sm.abort, p.hdr));
                if (!ok) break;
                ++reads;
                tc_fence_after();
                // In phase A, E_V (done: VH_READY) is the V slot's only reader; MMA4
                // reads K and the decayed copy. Release the slot now, so that the
                // next V load overlaps this MMA4.
                if (elect_one()) mbar_arrive(&bars[ve_bar(sk)]);
                __syncwarp();
                mma4s(sk, second ? 1 : 0, kb > 0);
                if (elect_one()) {
                    mma_commit(&bars[second ? B_VH_FREE1 : B_VH_FREE]);
                    mma_commit(&bars[ke_bar(sk)]);
                }
                __syncwarp();
                ++nkv;
            }
            if (!ok) break;
            commit(B_DS_FULL);
            ++n_ds;
            if (!SO) commit(B_A_DONE);  // the producer may load Q into slot 0 again
        }
        if (SO) continue;
        // Phase C.
        const uint32_t q0 = nq, kv0 = nkv, g0 = g;
        // Phase A left the local state in the score columns: MMA1 may
        // overwrite them once E_S has read it.
        if (has_succ && !wait_warp(&bars[B_DS_EMPTY], (n_ds & 1) ^ 1, sm.abort, p.hdr)) break;
        if (!mma1(g0, q0, kv0)) break;
        for (int kb = 0; kb < nb && ok; ++kb) {
            const uint32_t gg = g0 + kb;
            const int sq = (q0 + kb) & 1, skv = (kv0 + kb) & 1;
            // MMA4: this block's DS, once E_V has decayed its values and E_S
            // has read the previous DS.
            // One probe for everything MMA4 and MMA3 need: the decayed values,
            // DS read by E_S, and the state copy (which E_S writes after reading
            // the previous DS), so that the two groups issue back to back. The
            // first block's copy is made from the scan's prefix or the caller's
            // state, which E_S reads from global memory: MMA4 does not wait for it.
            ok = kb > 0 ? wait_multi(3, &bars[B_VH_READY], n_vh & 1, &bars[B_DS_EMPTY],
                                     (n_ds & 1) ^ 1, &bars[B_S_READY], n_s & 1, lane, sm.abort,
                                     p.hdr)
                        : wait_multi(2, &bars[B_VH_READY], n_vh & 1, &bars[B_DS_EMPTY],
                                     (n_ds & 1) ^ 1, nullptr, 0, lane, sm.abort, p.hdr);
            if (!ok) break;
            ++n_vh;
            tc_fence_after();
            mma4(skv, false);
            if (elect_one()) {
                mma_commit(&bars[B_DS_FULL]);
                mma_commit(&bars[B_VH_FREE]);
                mma_commit(&bars[B_KE0 + skv]);
            }
            __syncwarp();
            ++n_ds;
            // MMA3: [OE_hi | OE_lo] = Q [S_hi | S_lo], once E_O of the previous block
            // has read OE (and, for the first block, E_S has written the copy).
            ok = kb > 0 ? wait_warp(&bars[B_OE_FREE], (gg & 1) ^ 1, sm.abort, p.hdr)
                        : wait_multi(2, &bars[B_OE_FREE], (gg & 1) ^ 1, &bars[B_S_READY],
                                     n_s & 1, nullptr, 0, lane, sm.abort, p.hdr);
            ++n_s;
            if (!ok) break;
            tc_fence_after();
            {
                const uint64_t a = dq0 + (uint64_t)sq * TILE16;
                const uint32_t d = tmem + COL_OE;
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ss(d, a + koff_k(ks), dsh + koff_mn(ks), IDESC_QS, ks ? 1u : 0u);
                    mma_commit(&bars[B_S_FREE]);
                    mma_commit(&bars[B_QE0 + sq]);
                }
                __syncwarp();
            }
            // MMA1 of the next block, so that E_P overlaps this block's MMA2.
            if (kb + 1 < nb && !(ok = mma1(gg + 1, q0 + kb + 1, kv0 + kb + 1))) break;
            // MMA2: OI = P V (P hi and lo from TMEM), once E_P is done and
            // E_O has read the previous OI.
            ok = wait_multi(2, &bars[B_P_READY0 + (gg & 1)], (gg >> 1) & 1, &bars[B_O_EMPTY],
                            (gg & 1) ^ 1, nullptr, 0, lane, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
            {
                const uint64_t b = dv0 + (uint64_t)skv * BOX16;
                const uint32_t a = tmem + COL_SP + 128u * (gg & 1);
                // K-step ks (tokens 16ks..16ks+15) sits in chunk ks/2: hi words
                // at column 32(ks/2) + 8(ks%2), lo words 16 columns further.
                if (elect_one()) {
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_ts(tmem + COL_OI, a + 32u * (ks >> 1) + 8u * (ks & 1) + 16u * part,
                                   b + koff_mn(ks), IDESC_PV, (part || ks) ? 1u : 0u);
                    mma_commit(&bars[B_O_FULL]);
                    mma_commit(&bars[B_VE0 + skv]);
                }
                __syncwarp();
            }
        }
        if (!ok) break;
        nq += nb;
        nkv += nb;
        g += nb;
    }
    // Make sure no MMA is in flight before TMEM is released.
    commit(B_FIN);
    volatile int never = 0;
    mbar_wait(&bars[B_FIN], 0, &never, p.hdr, DRAIN_LIMIT_NS);
    __syncwarp();
}

// Phase A (local state of a segment with a successor, or the state-only
// pass): nothing but E_V and MMA4 runs, so the VO, P and S groups share E_V.
// Each takes some of the 16-byte chunks of its row's 64 decayed values (VO
// chunks 0-2, P 3-5, S 6-7) and arrives on the buffer's phase-A barrier (384
// arrivals). Block kb uses buffer kb & 1. nkv counts the V loads the caller
// has seen, n_vh and n_vh1 the phases of buffers 0 and 1's free barriers.
template <int REV, int MODE>
__device__ bool phase_a_ev(const Params& p, const Smem& sm, const Item& it, float slope, int row,
                           int c0, int c1, uint32_t& nkv, uint32_t& n_vh, uint32_t& n_vh1)
{
    constexpr bool SO = MODE == 1;
    uint64_t* bars = sm.bars;
    const int nb = num_blocks(it.len);
    if (!SO) ++n_vh1;  // the MMA warp's extra phase for Q slot 0 (see mma_role)
    for (int kb = 0; kb < nb; ++kb) {
        const int t0 = block_t0(it.len, kb, REV);
        const int L = min(C, it.len - t0);
        const int m = REV ? t0 + row : it.len - 1 - (t0 + row);
        const uint32_t NS = num_stages<SO>(), s = nkv % NS;
        const bool second = (kb & 1) != 0;
        uint32_t& uses = second ? n_vh1 : n_vh;
        if (!wait_warp(&bars[vf_bar(s)], (nkv / NS) & 1, sm.abort, p.hdr)) return false;
        if (!wait_warp(&bars[second ? B_VH_FREE1 : B_VH_FREE], (uses & 1) ^ 1, sm.abort, p.hdr))
            return false;
        uint8_t* vh = second ? sm.vh1() : sm.vh();
        uint8_t* vl = second ? sm.vl1() : sm.vl();
        const float f = row < L ? expf(-slope * (float)m) : 0.f;
        const uint64_t ff = f2(f, f);
        const uint8_t* src = sm.v3(s);
#pragma unroll 1
        for (int c = c0; c < c1; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(src + swz(row, c));
            uint4 h, l;
            split_pair(mul2(bf2_to_f2(u.x), ff), h.x, l.x);
            split_pair(mul2(bf2_to_f2(u.y), ff), h.y, l.y);
            split_pair(mul2(bf2_to_f2(u.z), ff), h.z, l.z);
            split_pair(mul2(bf2_to_f2(u.w), ff), h.w, l.w);
            *reinterpret_cast<uint4*>(vh + swz(row, c)) = h;
            *reinterpret_cast<uint4*>(vl + swz(row, c)) = l;
        }
        fence_proxy_async();
        mbar_arrive(&bars[second ? B_VHA_READY1 : B_VHA_READY]);
        ++nkv;
        ++uses;
    }
    return true;
}

// P group: E_P for every phase-C block.
//
// Full blocks take a fast path: in chunks that lie entirely on the causal
// side of the diagonal, the decay lam^m of consecutive columns is formed by
// repeated multiplication by lam^2 along two chains (pairs of columns, f32x2),
// starting from the exact table values, and always toward larger exponents,
// so underflow only ever reaches values that are zero in fp32 anyway. The
// diagonal chunk and partial blocks read the exact table per element.
template <int REV, int MODE>
__device__ void p_role(const Params& p, const Smem& sm, uint32_t tmem, int warp, int lane)
{
    constexpr bool SO = MODE == 1, ONE = MODE == 2;
    uint64_t* bars = sm.bars;
    const int w = warp & 3;
    const int row = (w << 5) | lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(w << 5) << 16);
    float* pw = sm.pw;
    uint32_t g = 0, n_sync = 0, nkv = 0, n_vh = 0, n_vh1 = 0;
    Item it;
    for (uint32_t k = 0;; ++k) {
        if (!next_item(p, sm, k, it, true, lane)) break;
        const float slope = p.slopes[it.head];
        if (((!ONE && it.p_ord < it.nseg - 1) || SO) &&
            !phase_a_ev<REV, MODE>(p, sm, it, slope, row, 3, 6, nkv, n_vh, n_vh1))
            break;
        if (SO) continue;  // no phase C
        nkv += num_blocks(it.len);   // phase C: E_V is the VO group's alone
        n_vh += num_blocks(it.len);
        if (!group_sync(&bars[B_P_SYNC], n_sync, sm.abort, p.hdr)) break;
        pw[row] = expf(-slope * (float)row);
        if (row == 0) pw[C] = expf(-slope * (float)C);
        if (!group_sync(&bars[B_P_SYNC], n_sync, sm.abort, p.hdr)) break;
        const float lam2 = pw[2];
        const uint64_t L2 = f2(lam2, lam2);
        const int nb = num_blocks(it.len);
        bool ok = true;
        for (int kb = 0; kb < nb && ok; ++kb, ++g) {
            const int L = min(C, it.len - block_t0(it.len, kb, REV));
            const int buf = g & 1;
            ok = wait_warp(&bars[B_SP_FULL0 + buf], (g >> 1) & 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
            const uint32_t base = lane_addr + COL_SP + 128u * buf;
            // Chunk c covers columns 32c..32c+31; warp w holds rows 32w..32w+31,
            // so chunks before (forward) / after (reverse) the diagonal chunk
            // are fully causal and the rest fully masked.
            const bool full = L == C;
            const bool row_live = REV ? true : row < L;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t hi[16], lo[16];
                const bool active = REV ? (c >= w) : (c <= w);
                if (active) {
                    uint32_t r32[32];
                    tmem_ld32(base + 32 * c, r32);
                    uint64_t W[16];  // decay of columns (32c + 2e, 32c + 2e + 1)
                    if (full && c != w) {
                        // Exponent of column 32c + t: E - t (forward) or E + t (reverse).
                        const int E = REV ? 32 * c - row : row - 32 * c;
                        uint64_t wa, wb;  // chains over pairs 15..8 and 7..0 (forward) / 0..7 and 8..15
                        if (REV) {
                            wa = f2(pw[E], pw[E + 1]);
                            wb = f2(pw[E + 16], pw[E + 17]);
                        } else {
                            wa = f2(pw[E - 30], pw[E - 31]);
                            wb = f2(pw[E - 14], pw[E - 15]);
                        }
#pragma unroll
                        for (int step = 0; step < 8; ++step) {
                            W[REV ? step : 15 - step] = wa;
                            W[REV ? 8 + step : 7 - step] = wb;
                            wa = mul2(wa, L2);
                            wb = mul2(wb, L2);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float x2[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int j = 32 * c + 2 * e + u;
                                bool keep;
                                int m;
                                if (REV) {
                                    keep = (c > w || j >= row) && j < L;
                                    m = j - row;
                                } else {
                                    keep = (c < w || j <= row) && row_live;
                                    m = row - j;
                                }
                                x2[u] = keep ? pw[keep ? m : 0] : 0.f;
                            }
                            W[e] = f2(x2[0], x2[1]);
                        }
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        split_pair(mul2(f2u(r32[2 * e], r32[2 * e + 1]), W[e]), hi[e], lo[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
                }
                tmem_st16(base + 32 * c, hi);
                tmem_st16(base + 32 * c + 16, lo);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_P_READY0 + buf]);
        }
        if (!ok) break;
    }
}

// VO group: E_V (decayed values, hi and lo, for every block) and E_O (the
// output rows of every phase-C block).
template <int REV, int OUT_F32, int MODE>
__device__ void vo_role(const Params& p, const Smem& sm, uint32_t tmem, int warp, int lane)
{
    constexpr bool SO = MODE == 1, ONE = MODE == 2;
    uint64_t* bars = sm.bars;
    const int w = warp & 3;
    const int row = (w << 5) | lane;  // E_V: token row of the V tile; E_O: output row
    const uint32_t lane_addr = tmem + ((uint32_t)(w << 5) << 16);
    uint32_t nkv = 0, n_vh = 0, n_vh1 = 0, g = 0;
    Item it;
    // E_V for the block at segment offset t0 with L valid tokens; the value
    // of token j is scaled by lam^m(j) (0 for j >= L).
    auto e_v = [&](float slope, int L, int m) -> bool {
        const int s = nkv & 1;
        if (!wait_warp(&bars[B_VF0 + s], (nkv >> 1) & 1, sm.abort, p.hdr)) return false;
        if (!wait_warp(&bars[B_VH_FREE], (n_vh & 1) ^ 1, sm.abort, p.hdr)) return false;
        const float f = row < L ? expf(-slope * (float)m) : 0.f;
        const uint64_t ff = f2(f, f);
        const uint8_t* src = sm.v(s);
        // Two 16-byte chunks in flight: E_V sits between this block's MMA4 and
        // the next one, and its latency, not its instruction count, is what counts.
#pragma unroll 2
        for (int c = 0; c < 8; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(src + swz(row, c));
            uint4 h, l;
            split_pair(mul2(bf2_to_f2(u.x), ff), h.x, l.x);
            split_pair(mul2(bf2_to_f2(u.y), ff), h.y, l.y);
            split_pair(mul2(bf2_to_f2(u.z), ff), h.z, l.z);
            split_pair(mul2(bf2_to_f2(u.w), ff), h.w, l.w);
            *reinterpret_cast<uint4*>(sm.vh() + swz(row, c)) = h;
            *reinterpret_cast<uint4*>(sm.vl() + swz(row, c)) = l;
        }
        fence_proxy_async();
        mbar_arrive(&bars[B_VH_READY]);
        ++nkv;
        ++n_vh;
        return true;
    };
    for (uint32_t k = 0;; ++k) {
        if (!next_item(p, sm, k, it, true, lane)) break;
        const float slope = p.slopes[it.head];
        const int nb = num_blocks(it.len);
        const bool has_succ = !ONE && it.p_ord < it.nseg - 1;
        bool ok = true;
        if ((has_succ || SO) &&
            !phase_a_ev<REV, MODE>(p, sm, it, slope, row, 0, 3, nkv, n_vh, n_vh1))
            break;
        if (SO) continue;
        auto e_v_c = [&](int kb) -> bool {
            const int L = min(C, it.len - block_t0(it.len, kb, REV));
            return e_v(slope, L, REV ? row : L - 1 - row);
        };
        if (!e_v_c(0)) break;
        for (int kb = 0; kb < nb && ok; ++kb, ++g) {
            if (kb + 1 < nb && !(ok = e_v_c(kb + 1))) break;
            // E_O: O = OI + lam^(i+1) OE (reverse: lam^(L-i)).
            ok = wait_warp(&bars[B_O_FULL], g & 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
            const int t0 = block_t0(it.len, kb, REV);
            const int L = min(C, it.len - t0);
            const float rowc = expf(-slope * (float)(REV ? max(L - row, 0) : row + 1));
            const uint64_t rc2 = f2(rowc, rowc);
            const bool store = row < L;
            const long long orow = it.out_row0 + t0 + row;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t ri[16], rh[16], rl[16];
                tmem_ld16(lane_addr + COL_OI + 16 * c, ri);
                tmem_ld16(lane_addr + COL_OE + 16 * c, rh);
                tmem_ld16(lane_addr + COL_OE + DV + 16 * c, rl);
                tmem_wait_ld();
                if (c == 3) {
                    tc_fence_before();
                    mbar_arrive(&bars[B_OE_FREE]);
                }
                uint64_t ov[8];
#pragma unroll
                for (int x = 0; x < 8; ++x)
                    ov[x] = fma2(rc2, add2(f2u(rh[2 * x], rh[2 * x + 1]), f2u(rl[2 * x], rl[2 * x + 1])),
                                 f2u(ri[2 * x], ri[2 * x + 1]));
                if (store) {
                    const size_t off = (size_t)orow * D + DV * it.half + 16 * c;
                    if (OUT_F32) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + off);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            dst[x] = make_float4(f2x(ov[2 * x]), f2y(ov[2 * x]), f2x(ov[2 * x + 1]),
                                                 f2y(ov[2 * x + 1]));
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + off);
#pragma unroll
                        for (int x = 0; x < 2; ++x)
                            dst[x] = make_uint4(pack_bf16x2(f2x(ov[4 * x + 0]), f2y(ov[4 * x + 0])),
                                                pack_bf16x2(f2x(ov[4 * x + 1]), f2y(ov[4 * x + 1])),
                                                pack_bf16x2(f2x(ov[4 * x + 2]), f2y(ov[4 * x + 2])),
                                                pack_bf16x2(f2x(ov[4 * x + 3]), f2y(ov[4 * x + 3])));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[B_O_EMPTY]);
        }
        if (!ok) break;
    }
}

// S group: E_S (the fp32 state, row a of this item's 128 x 64 state per
// thread, kept as 32 f32x2 pairs), the hi/lo state copies for MMA3, and the
// scan between segments.
template <int REV, int MODE>
__device__ void s_role(const Params& p, const Smem& sm, uint32_t tmem, int warp, int lane)
{
    constexpr bool SO = MODE == 1, ONE = MODE == 2;
    uint64_t* bars = sm.bars;
    const int a = ((warp & 3) << 5) | lane;  // TMEM lane = key dim a
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) << 5) << 16);
    uint32_t n_ds = 0, n_s = 0, n_sync = 0, nkv = 0, n_vh = 0, n_vh1 = 0;
    uint64_t S[DV / 2];
    Item it;
    // DS row a -> S (S = dL * S + DS when accumulate).
    auto read_ds = [&](float dL, bool accumulate) -> bool {
        if (!wait_warp(&bars[B_DS_FULL], n_ds & 1, sm.abort, p.hdr)) return false;
        tc_fence_after();
        const uint64_t d2 = f2(dL, dL);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
            tmem_ld32(lane_addr + COL_DS + 32 * h, r);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const uint64_t ds = f2u(r[2 * x], r[2 * x + 1]);
                S[16 * h + x] = accumulate ? fma2(d2, S[16 * h + x], ds) : ds;
            }
        }
        tc_fence_before();
        mbar_arrive(&bars[B_DS_EMPTY]);
        ++n_ds;
        return true;
    };
    // Phase A's local state: S = DS_hi + DS_lo (score columns 0..63 and 64..127).
    auto read_ds_pair = [&]() -> bool {
        if (!wait_warp(&bars[B_DS_FULL], n_ds & 1, sm.abort, p.hdr)) return false;
        tc_fence_after();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t rh[16], rl[16];
            tmem_ld16(lane_addr + COL_SP + 16 * q4, rh);
            tmem_ld16(lane_addr + COL_SP + DV + 16 * q4, rl);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 8; ++x)
                S[8 * q4 + x] = add2(f2u(rh[2 * x], rh[2 * x + 1]), f2u(rl[2 * x], rl[2 * x + 1]));
        }
        tc_fence_before();
        mbar_arrive(&bars[B_DS_EMPTY]);
        ++n_ds;
        return true;
    };
    // Row a of this half's 64 columns of the final state.
    auto write_state = [&](const Item& itm) {
        if (!p.state_out) return;
        float4* dst = reinterpret_cast<float4*>(p.state_out + ((size_t)itm.chain * D + a) * D +
                                                DV * itm.half);
#pragma unroll
        for (int x = 0; x < DV / 4; ++x)
            dst[x] = make_float4(f2x(S[2 * x]), f2y(S[2 * x]), f2x(S[2 * x + 1]), f2y(S[2 * x + 1]));
    };
    // Hi/lo copies of the state (row a of two swizzled 128 x 64 boxes) for the next MMA3.
    auto publish_copy = [&]() -> bool {
        if (!wait_warp(&bars[B_S_FREE], (n_s & 1) ^ 1, sm.abort, p.hdr)) return false;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 h, l;
            split_pair(S[4 * c + 0], h.x, l.x);
            split_pair(S[4 * c + 1], h.y, l.y);
            split_pair(S[4 * c + 2], h.z, l.z);
            split_pair(S[4 * c + 3], h.w, l.w);
            *reinterpret_cast<uint4*>(sm.sh() + swz(a, c)) = h;
            *reinterpret_cast<uint4*>(sm.sl() + swz(a, c)) = l;
        }
        fence_proxy_async();
        mbar_arrive(&bars[B_S_READY]);
        ++n_s;
        return true;
    };
    for (uint32_t k = 0;; ++k) {
        if (!next_item(p, sm, k, it, true, lane)) break;
        const float slope = p.slopes[it.head];
        const int nb = num_blocks(it.len);
        const bool has_succ = !ONE && it.p_ord < it.nseg - 1;
        const int chain2 = 2 * it.chain + it.half;
        bool ok = true;
        if ((has_succ || SO) &&
            !phase_a_ev<REV, MODE>(p, sm, it, slope, a, 6, 8, nkv, n_vh, n_vh1))
            break;
        if (!SO) {
            nkv += nb;  // phase C: E_V is the VO group's alone
            n_vh += nb;
        }
        if (SO) {
            // The chain's whole local state, plus lam^len times the incoming state.
            if (!read_ds_pair()) break;
            if (p.state_in) {
                const float dl = expf(-slope * (float)it.len);
                const uint64_t dl2 = f2(dl, dl);
                const float* s_in = p.state_in + ((size_t)it.chain * D + a) * D + DV * it.half;
#pragma unroll
                for (int x = 0; x < DV / 4; ++x) {
                    const float4 w = ld_cg_ordered(s_in + 4 * x);
                    S[2 * x] = fma2(dl2, f2(w.x, w.y), S[2 * x]);
                    S[2 * x + 1] = fma2(dl2, f2(w.z, w.w), S[2 * x + 1]);
                }
            }
            write_state(it);
            continue;
        }
        if (has_succ) {
            if (!read_ds_pair()) break;  // S = S_loc
        } else {
#pragma unroll
            for (int x = 0; x < DV / 2; ++x) S[x] = 0ull;
        }
        // Incoming state: the predecessor's inclusive prefix; for the first
        // segment the caller's state before token 0, or zero.
        const float* src = p.incl + (((size_t)chain2 * 2 + ((it.p_ord - 1) & 1)) * D + a) * DV;
        if (!ONE && it.p_ord > 0) {
            if (a == 0) {
                const int* flag = p.chain_flags + chain2;
                const unsigned long long t0 = globaltimer();
                int seen;
                for (uint32_t spin = 0;; ++spin) {
                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(flag) : "memory");
                    if (seen >= it.p_ord) break;
                    if ((spin & 15) == 15) {
                        if (*sm.abort) break;
                        if (globaltimer() - t0 > p.flag_limit_ns) {
                            atomicExch(&p.hdr->status, (int)LA_ERR_TIMEOUT);
                            break;
                        }
                    }
                    __nanosleep(128);
                }
            }
            if (!group_sync(&bars[B_S_SYNC], n_sync, sm.abort, p.hdr)) break;
        }
        {
            // S_prev = the predecessor's prefix; with a successor, publish
            // lam^len S_prev + S_loc. Phase C continues from S_prev.
            const float dl = expf(-slope * (float)it.len);
            const uint64_t dl2 = f2(dl, dl);
            float* dst = p.incl + (((size_t)chain2 * 2 + (it.p_ord & 1)) * D + a) * DV;
            const bool has_prev = !ONE && it.p_ord > 0;
            // The caller's state may be the state_out array itself: it is read here,
            // before this chain's first publish, and written after the last segment.
            const float* s_in = (has_prev || p.state_in == nullptr)
                                    ? nullptr
                                    : p.state_in + ((size_t)it.chain * D + a) * D + DV * it.half;
#pragma unroll
            for (int x = 0; x < DV / 4; ++x) {
                const float4 w = has_prev ? ld_cg_ordered(src + 4 * x)
                                 : s_in   ? ld_cg_ordered(s_in + 4 * x)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                const uint64_t w0 = f2(w.x, w.y), w1 = f2(w.z, w.w);
                if (has_succ) {
                    const uint64_t o0 = fma2(dl2, w0, S[2 * x]), o1 = fma2(dl2, w1, S[2 * x + 1]);
                    st_cg_ordered(dst + 4 * x, make_float4(f2x(o0), f2y(o0), f2x(o1), f2y(o1)));
                }
                S[2 * x] = w0;
                S[2 * x + 1] = w1;
            }
        }
        if (has_succ) {
            __threadfence();
            if (!group_sync(&bars[B_S_SYNC], n_sync, sm.abort, p.hdr)) break;
            if (a == 0 && !p.skip_publish) {
                int* flag = p.chain_flags + chain2;
                asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(it.p_ord + 1) : "memory");
            }
        }
        if (!publish_copy()) break;
        for (int kb = 0; kb < nb && ok; ++kb) {
            const int L = min(C, it.len - block_t0(it.len, kb, REV));
            if (!(ok = read_ds(expf(-slope * (float)L), true))) break;
            if (kb + 1 < nb && !(ok = publish_copy())) break;
        }
        if (!ok) break;
        if (it.p_ord == it.nseg - 1) write_state(it);
    }
}

// Small shared state at the start of the dynamic region; the 1024-aligned
// tile region follows (SMEM_BYTES reserves the worst-case alignment gap).
constexpr uint32_t SM_BARS = 0;                       // NUM_BARS x 8 B
constexpr uint32_t SM_RING = 320;                     // 2 x Item
constexpr uint32_t SM_PW = 448;                       // (C + 1) floats
constexpr uint32_t SM_TMEM = SM_PW + 4 * (C + 4);     // u32
constexpr uint32_t SM_ABORT = SM_TMEM + 4;            // int
constexpr uint32_t SM_SMALL = SM_ABORT + 4;
static_assert(NUM_BARS * 8 <= SM_RING, "barrier area");
static_assert(sizeof(Item) * 2 <= SM_PW - SM_RING, "ring area");
constexpr uint32_t SMEM_BYTES = SM_SMALL + 1023 + SMEM_TILES;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

template <int REV, int OUT_F32, int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_forward_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const Params p)
{
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(dsmem + SM_BARS);
    uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(dsmem + SM_TMEM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(dsmem + SM_ABORT);
    Smem sm;
    sm.tiles = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(dsmem) + SM_SMALL + 1023) & ~uintptr_t(1023));
    sm.bars = bars;
    sm.ring = reinterpret_cast<Item*>(dsmem + SM_RING);
    sm.abort = abort_flag;
    sm.pw = reinterpret_cast<float*>(dsmem + SM_PW);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < NUM_BARS; ++i) {
            uint32_t count = 1;  // TMA expect_tx arrivals, MMA commits, single threads
            if (i == B_P_READY0 || i == B_P_READY1 || i == B_VH_READY || i == B_DS_EMPTY ||
                i == B_S_READY || i == B_O_EMPTY || i == B_OE_FREE || i == B_P_SYNC ||
                i == B_S_SYNC)
                count = 128;
            if (i == B_ITEM_EMPTY0 || i == B_ITEM_EMPTY1) count = 1 + 12;  // MMA lane + 12 group warps
            if (i == B_VHA_READY || i == B_VHA_READY1) count = 3 * 128;  // phase-A E_V: VO, P, S
            mbar_init(&bars[i], count);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tq)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_base_sh)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_sh;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_CTRL));
        if (warp == 0) producer_role<MODE>(p, &tq, &tk, &tv, sm, lane);
        if (warp == 1) mma_role<MODE>(p, sm, tmem, lane);
    } else if (warp < 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_P));
        p_role<REV, MODE>(p, sm, tmem, warp, lane);
    } else if (warp < 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_VO));
        vo_role<REV, OUT_F32, MODE>(p, sm, tmem, warp, lane);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_S));
        s_role<REV, MODE>(p, sm, tmem, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

// Varlen planner: segment-major list of (chain, p_ord, nseg) items; the
// final state of an empty sequence is its incoming state (or zero).
// Sequences with 0 < length < min_len get no items (another kernel serves
// them). One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) plan_varlen_kernel(const int* cu, int num_seqs, int H,
                                                           int seg, int4* items, int max_items,
                                                           WsHeader* hdr, float* state_out,
                                                           const float* state_in, int min_len)
{
    __shared__ int warp_tot[32];
    __shared__ int s_max;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto nseg_of = [&](int s) -> int {
        const long long L = (long long)cu[s + 1] - cu[s];
        return L > 0 && L >= min_len ? (int)((L + seg - 1) / seg) : 0;
    };
    if (tid == 0) s_max = 0;
    __syncthreads();
    int mx = 0;
    for (int s = tid; s < num_seqs; s += blockDim.x) mx = max(mx, nseg_of(s));
    atomicMax(&s_max, mx);
    if (state_out) {
        for (int s = 0; s < num_seqs; ++s) {
            if (cu[s + 1] - cu[s] > 0) continue;
            float4* dst = reinterpret_cast<float4*>(state_out + (size_t)s * H * D * D);
            const float4* src =
                state_in ? reinterpret_cast<const float4*>(state_in + (size_t)s * H * D * D) : nullptr;
            for (int x = tid; x < H * D * D / 4; x += blockDim.x)
                dst[x] = src ? src[x] : make_float4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    const int maxseg = s_max;
    if (maxseg == 1 && num_seqs <= 8192) {
        // One segment per sequence: no item waits on another, so order the
        // sequences longest first (ties by index) to shorten the tail.
        auto len_of = [&](int s) -> long long { return (long long)cu[s + 1] - cu[s]; };
        __shared__ int s_count;
        if (tid == 0) s_count = 0;
        __syncthreads();
        for (int s = tid; s < num_seqs; s += blockDim.x) {
            const long long Ls = len_of(s);
            if (Ls <= 0 || Ls < min_len) continue;
            atomicAdd(&s_count, 1);
            int rank = 0;
            for (int s2 = 0; s2 < num_seqs; ++s2) {
                const long long L2 = len_of(s2);
                rank += (L2 > Ls || (L2 == Ls && s2 < s)) ? 1 : 0;
            }
            for (int h = 0; h < H; ++h) {
                const long long t = (long long)rank * H + h;
                if (t < max_items) items[t] = make_int4(s * H + h, 0, 1, 0);
            }
        }
        __syncthreads();
        if (tid == 0) {
            const long long n = (long long)s_count * H;
            hdr->num_items = (int)min(n, (long long)max_items);
            if (n > max_items) atomicExch(&hdr->status, (int)LA_ERR_INVALID_ARG);
        }
        return;
    }
    long long offset = 0;
    for (int pp = 0; pp < maxseg; ++pp) {
        int running = 0;
        for (int base = 0; base < num_seqs; base += blockDim.x) {
            const int s = base + tid;
            const int ns = s < num_seqs ? nseg_of(s) : 0;
            const int pred = ns > pp ? 1 : 0;
            int incl = pred;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) warp_tot[warp] = incl;
            __syncthreads();
            int wbase = 0, tot = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
                if (w < warp) wbase += warp_tot[w];
                tot += warp_tot[w];
            }
            if (pred) {
                const long long r = running + wbase + incl - 1;
                for (int h = 0; h < H; ++h) {
                    const long long t = offset + r * H + h;
                    if (t < max_items) items[t] = make_int4(s * H + h, pp, ns, 0);
                }
            }
            running += tot;
            __syncthreads();
        }
        offset += (long long)running * H;
    }
    if (tid == 0) {
        hdr->num_items = (int)min(offset, (long long)max_items);
        if (offset > max_items) atomicExch(&hdr->status, (int)LA_ERR_INVALID_ARG);
    }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D map over [dim2][dim1][128] bf16 rows, boxes of 128 rows x 64 columns, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, unsigned long long dim1,
                     unsigned long long dim2)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)dim1, (cuuint64_t)dim2};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)dim1 * D * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms()
{
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// Segment length: the tuning value, or the candidate (powers of two from 1K
// tokens up to one segment per chain) that minimises (rounds of persistent
// CTAs) x (blocks per item + a fixed per-item cost), with phase A counted
// for items that have a successor. Independent of the device, so that the
// workspace size depends only on the arguments.
static int choose_seg(const Problems& P, int seg_tuning, bool varlen)
{
    if (seg_tuning > 0) return seg_tuning;
    if (varlen) {
        // With enough (sequence, head, half) items to keep every SM busy, each
        // sequence is one segment (no scan; the planner orders them longest
        // first); otherwise segments of 8K tokens add the parallelism.
        const long long pairs = 2LL * P.num_seqs * P.H;
        return pairs >= 4LL * 148 ? (1 << 30) : 8192;
    }
    const long long N = P.N, items_per_seg = 2 * P.count();
    const int sms = 148;
    const long long whole = std::max<long long>(128, (N + 127) / 128 * 128);
    double best = 1e300;
    long long best_seg = whole;
    for (long long seg = 1024;; seg *= 2) {
        const long long s = std::min(seg, whole);
        const long long nseg = (N + s - 1) / s;
        const long long items = items_per_seg * nseg;
        const double rounds = (double)((items + sms - 1) / sms);
        const double per_item = (s / 128.0) * (nseg > 1 ? 1.4 : 1.0) + 2.0;
        const double cost = rounds * per_item;
        if (cost < best * 0.999) {
            best = cost;
            best_seg = s;
        }
        if (s == whole) break;
    }
    return (int)std::min<long long>(best_seg, 1 << 30);
}

struct WsLayout {
    size_t flags, items, incl, end;
    long long nchains, max_items;
};

static WsLayout layout(const Problems& P, int seg, bool varlen)
{
    WsLayout w;
    w.nchains = P.count();
    if (varlen)
        w.max_items = (long long)P.H * ((P.total + seg - 1) / seg + P.num_seqs);
    else
        w.max_items = w.nchains * ((P.N + seg - 1) / seg);
    w.flags = sizeof(WsHeader);
    w.items = align_up(w.flags + sizeof(int) * 2 * (size_t)w.nchains, 256);
    w.incl = align_up(w.items + (varlen ? sizeof(int4) * (size_t)w.max_items : 0), 256);
    w.end = align_up(w.incl + sizeof(float) * (size_t)w.nchains * 2 * 2 * D * DV, 256);
    return w;
}

}  // namespace tc

FaultInjection g_fault;

size_t tc_workspace_bytes(const Problems& P, int d, int seg_tuning, bool varlen)
{
    (void)d;
    const int seg = tc::choose_seg(P, seg_tuning, varlen);
    return tc::layout(P, seg, varlen).end - sizeof(WsHeader);
}

cudaError_t launch_tc_forward(const Problems& P, const void* q, const void* k, const void* v,
                              const float* slopes, void* o, float* state_out, int d, int out_t,
                              int seg_tuning, void* workspace, cudaStream_t stream, int reverse,
                              const float* state_in, int state_only)
{
    using namespace tc;
    (void)d;
    const bool varlen = P.cu_seqlens != nullptr;
    // State only: one segment per chain (phase A needs no scan).
    const int seg = state_only ? (1 << 30) : choose_seg(P, seg_tuning, varlen);
    const WsLayout w = layout(P, seg, varlen);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaError_t err;
    if (!varlen && P.N == 0) {
        const size_t bytes = sizeof(float) * (size_t)P.count() * D * D;
        if (state_out && state_in && state_in != state_out)
            return cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, stream);
        if (state_out && !state_in) return cudaMemsetAsync(state_out, 0, bytes, stream);
        return cudaSuccess;
    }
    if (varlen && P.total == 0 && P.num_seqs == 0) return cudaSuccess;
    // Clear the header and the per-chain counters.
    err = cudaMemsetAsync(ws, 0, w.items, stream);
    if (err != cudaSuccess) return err;

    Params prm{};
    prm.H = P.H;
    prm.nchains = (int)w.nchains;
    prm.seg_tokens = seg;
    prm.N = P.N;
    prm.nseg = varlen ? 0 : (int)((P.N + seg - 1) / seg);
    prm.cu_seqlens = P.cu_seqlens;
    prm.total = P.total;
    prm.items = varlen ? reinterpret_cast<const int4*>(ws + w.items) : nullptr;
    prm.num_items_dense = varlen ? 0 : (int)w.max_items;
    prm.slopes = slopes;
    prm.o = o;
    prm.state_out = state_out;
    prm.state_in = reverse ? nullptr : state_in;
    prm.reverse = reverse;
    prm.hdr = reinterpret_cast<WsHeader*>(ws);
    prm.chain_flags = reinterpret_cast<int*>(ws + w.flags);
    prm.incl = reinterpret_cast<float*>(ws + w.incl);
    prm.flag_limit_ns = g_fault.wait_limit_us > 0 ? 1000ull * (unsigned long long)g_fault.wait_limit_us
                                                   : FLAG_LIMIT_NS;
    prm.skip_publish = g_fault.skip_publish;

    CUtensorMap mq, mk, mv;
    const unsigned long long dim1 = varlen ? (unsigned long long)std::max<long long>(P.total, 1)
                                           : (unsigned long long)P.N;
    const unsigned long long dim2 = varlen ? (unsigned long long)P.H : (unsigned long long)P.count();
    if (!make_map(&mq, q, dim1, dim2) || !make_map(&mk, k, dim1, dim2) || !make_map(&mv, v, dim1, dim2))
        return cudaErrorInvalidValue;

    if (varlen) {
        plan_varlen_kernel<<<1, 1024, 0, stream>>>(P.cu_seqlens, P.num_seqs, P.H, seg,
                                                    const_cast<int4*>(prm.items), (int)w.max_items,
                                                    prm.hdr, state_out, prm.state_in, P.min_len);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        if (P.total == 0) return cudaSuccess;
    }
    const long long max_items = 2 * w.max_items;
    const int grid = (int)std::min<long long>(num_sms(), std::max<long long>(1, max_items));
    auto launch = [&](auto kern) -> cudaError_t {
        // The warpgroups' setmaxnreg split assumes the CTA launches with 128
        // registers per thread; with fewer, the S group's increase would wait forever.
        cudaFuncAttributes fa{};
        cudaError_t e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != 65536 / NUM_THREADS) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, mv, prm);
        count_launch();
        return cudaGetLastError();
    };
    const bool f32 = out_t == LA_F32;
    // The state-only pass (forward, no output rows) is its own instantiation,
    // so that its paths add no code to the prefill's.
    if (state_only && !reverse) return launch(tc_forward_kernel<0, 0, 1>);
    if (state_only) return cudaErrorInvalidValue;
    // One segment per chain (dense, long enough segments): no phase A and no
    // scan, an instantiation without their code.
    if (!varlen && prm.nseg == 1) {
        if (reverse)
            return f32 ? launch(tc_forward_kernel<1, 1, 2>) : launch(tc_forward_kernel<1, 0, 2>);
        return f32 ? launch(tc_forward_kernel<0, 1, 2>) : launch(tc_forward_kernel<0, 0, 2>);
    }
    if (reverse)
        return f32 ? launch(tc_forward_kernel<1, 1, 0>) : launch(tc_forward_kernel<1, 0, 0>);
    return f32 ? launch(tc_forward_kernel<0, 1, 0>) : launch(tc_forward_kernel<0, 0, 0>);
}

cudaError_t launch_tc_backward(const Problems& P, const void* dO, const void* q, const void* k,
                               const void* v, const float* slopes, void* dq, void* dk, void* dv,
                               int d, int out_t, int seg_tuning, void* workspace,
                               cudaStream_t stream)
{
    cudaError_t e = launch_tc_forward(P, dO, v, k, slopes, dq, nullptr, d, out_t, seg_tuning,
                                      workspace, stream, 0);
    if (e == cudaSuccess)
        e = launch_tc_forward(P, v, dO, q, slopes, dk, nullptr, d, out_t, seg_tuning, workspace,
                              stream, 1);
    if (e == cudaSuccess)
        e = launch_tc_forward(P, k, q, dO, slopes, dv, nullptr, d, out_t, seg_tuning, workspace,
                              stream, 1);
    return e;
}

}  // namespace la
