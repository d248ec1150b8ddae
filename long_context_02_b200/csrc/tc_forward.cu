// Lightning attention on the sm_100a tensor cores: tcgen05 MMAs with TMEM
// accumulators, TMA-staged tiles, a chunk-parallel scan of the d x d state
// across segments, bf16 inputs, head dim 128.
//
// What is computed (per (sequence, head) "chain", decay lam = exp(-slope)):
//   O_i = sum_{j<=i} lam^(i-j) (q_i . k_j) v_j,   final state sum_j lam^(N-1-j) k_j^T v_j.
// "MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary":
//   section 2.2 - tiles: a masked intra-tile product plus the product with the
//                 accumulated key-value state, which is then updated;
//   section 3.2 - LASP+: each partition summarizes its keys/values locally, the
//                 summaries are combined into global prefixes, so partitions
//                 need not wait for the full serial pass before them;
//   section 3.3 - tiles of 32..256 tokens, batched matmuls (here tcgen05).
//
// Work decomposition. A chain of N tokens is cut into segments of SEG tokens
// (a multiple of the 128-token block). A work item is one (chain, segment).
// Persistent CTAs (one per SM) take items from an atomic ticket in
// segment-major order, so an item's predecessor in its chain always holds a
// smaller ticket and is already running or done. For each item:
//   phase A (if a later segment needs it): the segment's local state
//     S_loc = sum_j lam^(len-1-j) k_j^T v_j, block by block; then wait for the
//     predecessor's inclusive prefix S_prev (bounded spin on a per-chain
//     counter) and publish S_incl = lam^len S_prev + S_loc: the scan combine
//     (a1, S1) o (a2, S2) = (a1 a2, a2 S1 + S2).
//   phase C: run the segment's 128-token blocks from S_in = S_prev:
//     MMA1  SB  = Q K^T                     (fp32 in TMEM)
//     E_P   P   = SB * lam^(i-j) [j<=i]      (fp16, written back into TMEM)
//     MMA2  OI  = P V                       (A operand from TMEM)
//     MMA3  OE  = Q S                       (S: fp32 state kept in registers)
//     E_O   O   = OI + lam^(i+1) OE          -> global (bf16 or fp32)
//     E_K   Kt  = lam^(L-1-j) k_j            (in place in shared memory)
//     MMA4  DS^T = V^T Kt
//     E_S   S   = lam^L S + DS               (fp32, registers; fp16 copy for MMA3)
// Only non-negative decay exponents <= the block length appear, so nothing
// overflows; terms that underflow are below fp32 resolution of the result.
//
// Precision. Every tensor-core operand is fp16 with exact power-of-two
// scaling: the relative rounding of the operands the kernel forms itself (P,
// the state copy, the decayed keys) is 2^-11 (bf16 would be 2^-8, too coarse
// for a max error of 1e-2 of rms), and fp16's narrow exponent range never
// bites. As tiles land, converter warps rewrite Q (one scale per row), K and
// V (one scale per tile) as fp16 in [1, 2) magnitude; the bf16 -> fp16 step
// is exact. Then Q K^T is bounded by 512, so P needs no rescaling, and the
// decayed keys are bounded by the K tile. Each column of the state copy has
// its own scale (the state is held transposed, one value column per thread,
// so that is a thread-local choice). All scales are undone in fp32 in the
// epilogues.
//
// Warp roles (16 warps, 4 warpgroups): warp 0 TMA producer, warp 1 MMA
// issuer (also owns TMEM), warps 2-3 Q converters; 4-7 K/V converters (fp16
// tiles as they land); 8-11 "PE" (E_P and E_K after Q K^T); 12-15 "OS" (E_O,
// E_S and the scan). TMEM: 512 columns = SB/P | OI | OE | DS^T, 128 lanes.
// Shared memory: 2 stages x (Q, K, V) 128x128 16-bit tiles + the fp16 state
// copy, all in the 128-byte-swizzled layout TMA writes.
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
constexpr int C = 128;                           // tokens per block
constexpr int NUM_THREADS = 512;                 // 4 warpgroups
// Register split (setmaxnreg, which ptxas also uses to allocate each role):
// launched at 65536 / 512 = 128 per thread, i.e. 65536 per CTA. The control
// warpgroup drops to 64, the converters to 104, the PE group to 112, the OS
// group rises to 232: 128 * (64 + 104 + 112 + 232) = 65536, and per SM
// sub-partition (one warp of each group) 32 * 512 = 16384.
constexpr int REGS_CTRL = 64, REGS_CV = 104, REGS_PE = 112, REGS_OS = 232;
constexpr uint32_t BOX_BYTES = 128 * 64 * 2;     // one TMA box: 128 rows x 64 bf16
constexpr uint32_t TILE_BYTES = 2 * BOX_BYTES;   // 128 x 128 bf16
constexpr uint32_t STAGE_BYTES = 3 * TILE_BYTES; // Q, K, V
constexpr uint32_t SMEM_TILES = 2 * STAGE_BYTES + TILE_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_SB = 0, COL_OI = 128, COL_OE = 256, COL_DS = 384;
constexpr unsigned long long WAIT_LIMIT_NS = 4000000000ull;
constexpr unsigned long long FLAG_LIMIT_NS = 2000000000ull;
constexpr unsigned long long DRAIN_LIMIT_NS = 200000000ull;

enum {
    B_FULL0, B_FULL1, B_EMPTY0, B_EMPTY1, B_CONV0, B_CONV1, B_KT0, B_KT1, B_SBLK_FULL,
    B_SB_FREE, B_P_READY, B_O_FULL, B_O_EMPTY, B_DS_FULL, B_DS_EMPTY, B_S_READY, B_SC_FULL0,
    B_SC_FULL1, B_SC_FULL2, B_SC_FULL3, B_SC_EMPTY0, B_SC_EMPTY1, B_SC_EMPTY2, B_SC_EMPTY3,
    B_ITEM_FULL0, B_ITEM_FULL1, B_ITEM_EMPTY0, B_ITEM_EMPTY1, B_FIN, B_CV_SYNC, B_PE_SYNC,
    B_OS_SYNC, B_QFULL0, B_QFULL1, NUM_BARS
};
// A barrier's waiter must not skip phases: a parity wait on a barrier two
// phases behind returns at once. So the Q tile, which only phase-C blocks
// load, completes its own B_QFULL barrier rather than B_FULL, which every
// block completes and the Q converters would otherwise skip in phase A.

// tcgen05 instruction descriptors (kind::f16): D fp32, M = N = 128.
// bits: [4,6) D format (1 = f32), [7,10) A format and [10,13) B format
// (0 = f16, 1 = bf16; A and B always share one type), 15 A major, 16 B major
// (0 = K-major, 1 = MN-major), [17,23) N >> 3, [24,29) M >> 4.
constexpr uint32_t idesc(uint32_t fmt, uint32_t a_mn_major, uint32_t b_mn_major)
{
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
           ((128u >> 3) << 17) | ((128u >> 4) << 24);
}
constexpr uint32_t F16 = 0, BF16 = 1;
constexpr uint32_t IDESC_QK = idesc(F16, 0, 0);   // Q K^T: both K-major
constexpr uint32_t IDESC_PV = idesc(F16, 0, 1);   // P (TMEM) V: V MN-major
constexpr uint32_t IDESC_QS = idesc(F16, 0, 0);   // Q S: S stored as rows of S^T (K-major)
constexpr uint32_t IDESC_VK = idesc(F16, 1, 1);   // V^T Kt: both MN-major

struct Params {
    int H;
    int nchains;        // dense: B*H
    int nseg;           // dense: segments per chain
    int seg_tokens;
    long long N;        // dense: tokens per chain
    const int* cu_seqlens;  // varlen when not null
    long long total;
    const int4* items;  // varlen: planned items {chain, p_ord, nseg, 0}
    int num_items_dense;
    const float* slopes;
    void* o;
    float* state_out;
    int reverse;
    WsHeader* hdr;
    int* chain_flags;   // per chain: segments published so far
    float* incl;        // [chains][2][D][D] inclusive prefixes (ring of two)
    unsigned long long flag_limit_ns;  // bound of the inter-CTA wait
    int skip_publish;   // fault injection (tests): never raise the chain counters
};

struct Item {
    int valid;
    int chain;
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
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort,
                                       WsHeader* hdr,
                                       unsigned long long limit = WAIT_LIMIT_NS)
{
    if (mbar_try_wait(b, parity)) return true;
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

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Warp-uniform bounded wait for the 4-warp epilogue groups: every lane polls,
// and the warp proceeds only if all lanes saw the phase complete.
__device__ __forceinline__ bool wait_warp(uint64_t* b, uint32_t parity, volatile int* abort,
                                          WsHeader* hdr)
{
    const bool ok = mbar_wait(b, parity, abort, hdr);
    return __all_sync(0xffffffffu, ok);
}

// Bounded barrier over one 128-thread epilogue group (an mbarrier of count 128).
__device__ __forceinline__ bool group_sync(uint64_t* b, uint32_t& n, volatile int* abort,
                                           WsHeader* hdr)
{
    mbar_arrive(b);
    return wait_warp(b, n++ & 1, abort, hdr);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
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

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
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

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 version bit.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// K-major 128x128 tile (two 64-column boxes): k-step ks covers K elements [16ks, 16ks+16).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int ks)
{
    return sdesc(tile + (uint32_t)(ks >> 2) * BOX_BYTES + (uint32_t)(ks & 3) * 32u, 16u, 1024u);
}

// MN-major 128x128 tile (rows = K dim, two 64-element boxes along MN):
// k-step ks covers rows [16ks, 16ks+16).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int ks)
{
    return sdesc(tile + (uint32_t)ks * 2048u, BOX_BYTES, 1024u);
}

__device__ __forceinline__ int num_blocks(int len) { return (len + C - 1) / C; }

// Segment offset of the k-th block in processing order.
__device__ __forceinline__ int block_t0(int len, int k, int rev)
{
    const int nb = num_blocks(len);
    return (rev ? nb - 1 - k : k) * C;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Ordered L2 loads/stores (volatile asm keeps their program order, which
// bounds how many values are in flight and stops loads being hoisted).
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

// Exact power-of-two scales for a max magnitude m: down * m lies in [1, 2),
// up = 1 / down. Zero, subnormal or non-finite m keep scale 1.
// `ue` is the biased fp32 exponent of `up` (how the scale is kept in shared memory).
struct Pow2 {
    float down, up;
    uint8_t ue;
};
__device__ __forceinline__ Pow2 pow2_for(float m)
{
    const uint32_t e = (__float_as_uint(m) >> 23) & 0xffu;
    if (e == 0u || e == 255u) return {1.f, 1.f, (uint8_t)127};
    return {__uint_as_float((254u - e) << 23), __uint_as_float(e << 23), (uint8_t)e};
}
__device__ __forceinline__ float up_of(uint8_t ue) { return __uint_as_float((uint32_t)ue << 23); }

// Offset of 16-byte chunk c (0..15) of row r in a 128x128 16-bit tile stored as
// two 128-byte-swizzled 64-column boxes (the layout TMA writes).
__device__ __forceinline__ uint32_t chunk_off(int r, int c)
{
    return (uint32_t)(c >> 3) * BOX_BYTES + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Load row r of a bf16 tile as 128 floats.
__device__ __forceinline__ void load_row_bf16(const uint8_t* tile, int r, float (&x)[128])
{
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(tile + chunk_off(r, c));
        x[8 * c + 0] = bf16_lo(w.x); x[8 * c + 1] = bf16_hi(w.x);
        x[8 * c + 2] = bf16_lo(w.y); x[8 * c + 3] = bf16_hi(w.y);
        x[8 * c + 4] = bf16_lo(w.z); x[8 * c + 5] = bf16_hi(w.z);
        x[8 * c + 6] = bf16_lo(w.w); x[8 * c + 7] = bf16_hi(w.w);
    }
}

// Store 128 floats times f as fp16 into row r of a tile.
__device__ __forceinline__ void store_row_f16(uint8_t* tile, int r, const float (&x)[128], float f)
{
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        uint4 w;
        w.x = pack_f16x2(x[8 * c + 0] * f, x[8 * c + 1] * f);
        w.y = pack_f16x2(x[8 * c + 2] * f, x[8 * c + 3] * f);
        w.z = pack_f16x2(x[8 * c + 4] * f, x[8 * c + 5] * f);
        w.w = pack_f16x2(x[8 * c + 6] * f, x[8 * c + 7] * f);
        *reinterpret_cast<uint4*>(tile + chunk_off(r, c)) = w;
    }
}

__device__ __forceinline__ float row_absmax(const float (&x)[128])
{
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 128; ++i) m = fmaxf(m, fabsf(x[i]));
    return m;
}

// Convert row r of a bf16 tile in place to fp16 scaled to [1, 2); rows at or
// beyond `valid` become zero. Returns the scale (`up` undoes it).
__device__ __forceinline__ Pow2 convert_row(uint8_t* tile, int r, int valid)
{
    float x[128];
    load_row_bf16(tile, r, x);
    const Pow2 s = pow2_for(row_absmax(x));
    store_row_f16(tile, r, x, r < valid ? s.down : 0.f);
    return s;
}

// ------------------------------------------------------------------ work items

__device__ Item make_item(const Params& p, int t, int num_items)
{
    Item it{};
    it.valid = 0;
    if (t >= num_items) return it;
    int chain, p_ord, nseg;
    long long seq_start, seq_len, rowbase;
    if (p.cu_seqlens == nullptr) {
        p_ord = t / p.nchains;
        chain = t % p.nchains;
        nseg = p.nseg;
        it.head = chain % p.H;
        it.z = chain;
        seq_start = 0;
        seq_len = p.N;
        rowbase = (long long)chain * p.N;
    } else {
        const int4 w = p.items[t];
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

// Scales of one loaded block, handed from the converter group to the OS group
// through a ring of four slots (B_SC_FULL / B_SC_EMPTY). Each byte is the
// biased fp32 exponent of the factor that undoes a power-of-two scaling.
struct ScaleRec {
    uint8_t qe[C];  // Q rows (phase-C blocks)
    uint8_t kc;     // K tile (phase C: K as fed to Q K^T; phase A: decayed keys)
    uint8_t vc;     // V tile
    uint8_t pad[14];
};

struct Smem {
    uint8_t* tiles;  // 1024-aligned: stage0 {Q,K,V}, stage1 {Q,K,V}, S16
    uint64_t* bars;
    Item* ring;
    volatile int* abort;
    float* pw_pe;    // [C+1] lam^m of the PE group's current item
    ScaleRec* sc;    // [4]
    float* red;      // [2][8] partial tile maxima of the converter group
    uint8_t* hs;     // [2][4] state-copy scales, one per 32 columns (OS group)
    __device__ uint8_t* q(int s) const { return tiles + s * STAGE_BYTES; }
    __device__ uint8_t* k(int s) const { return tiles + s * STAGE_BYTES + TILE_BYTES; }
    __device__ uint8_t* v(int s) const { return tiles + s * STAGE_BYTES + 2 * TILE_BYTES; }
    __device__ uint8_t* s16() const { return tiles + 2 * STAGE_BYTES; }
};

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

__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int x, int y, int z, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}

__device__ void producer_role(const Params& p, const CUtensorMap* tq, const CUtensorMap* tk,
                              const CUtensorMap* tv, const Smem& sm)
{
    uint64_t* bars = sm.bars;
    const int num_items =
        p.cu_seqlens ? *reinterpret_cast<volatile int*>(&p.hdr->num_items) : p.num_items_dense;
    // K and V read in phase A are read again in phase C: keep them in L2;
    // everything read for the last time goes first.
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    uint32_t n_load = 0;
    uint32_t uses[2] = {0, 0}, quses[2] = {0, 0};
    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!mbar_wait(&bars[B_ITEM_EMPTY0 + slot], ((k >> 1) & 1) ^ 1, sm.abort, p.hdr)) break;
        const int t = atomicAdd(&p.hdr->ticket, 1);
        const Item it = make_item(p, t, num_items);
        sm.ring[slot] = it;
        mbar_arrive(&bars[B_ITEM_FULL0 + slot]);
        if (!it.valid) break;
        const int nb = num_blocks(it.len);
        const bool has_succ = it.p_ord < it.nseg - 1;
        bool ok = true;
        for (int pass = has_succ ? 0 : 1; pass < 2 && ok; ++pass) {
            for (int kb = 0; kb < nb; ++kb) {
                const int s = n_load & 1;
                ok = mbar_wait(&bars[B_EMPTY0 + s], ((n_load >> 1) & 1) ^ 1, sm.abort, p.hdr);
                if (!ok) break;
                uint64_t* full = &bars[B_FULL0 + s];
                const int y = it.y0 + block_t0(it.len, kb, p.reverse);
                const uint64_t kv_pol = pass == 0 ? keep : drop;
                mbar_expect_tx(full, 2 * TILE_BYTES);
                if (pass == 1) {
                    uint64_t* qfull = &bars[B_QFULL0 + s];
                    mbar_expect_tx(qfull, TILE_BYTES);
                    tma_load_3d_hint(sm.q(s), tq, qfull, 0, y, it.z, drop);
                    tma_load_3d_hint(sm.q(s) + BOX_BYTES, tq, qfull, 64, y, it.z, drop);
                    ++quses[s];
                }
                tma_load_3d_hint(sm.k(s), tk, full, 0, y, it.z, kv_pol);
                tma_load_3d_hint(sm.k(s) + BOX_BYTES, tk, full, 64, y, it.z, kv_pol);
                tma_load_3d_hint(sm.v(s), tv, full, 0, y, it.z, kv_pol);
                tma_load_3d_hint(sm.v(s) + BOX_BYTES, tv, full, 64, y, it.z, kv_pol);
                ++uses[s];
                ++n_load;
            }
        }
        if (!ok) break;
    }
    if (*sm.abort) {
        // Wind down: let this CTA's copies in flight land before it exits.
        for (int s = 0; s < 2; ++s)
            if (uses[s] > 0) {
                volatile int never = 0;
                mbar_wait(&bars[B_FULL0 + s], (uses[s] - 1) & 1, &never, p.hdr, DRAIN_LIMIT_NS);
                if (quses[s] > 0)
                    mbar_wait(&bars[B_QFULL0 + s], (quses[s] - 1) & 1, &never, p.hdr,
                              DRAIN_LIMIT_NS);
            }
    }
}

__device__ void mma_role(const Params& p, const Smem& sm, uint32_t tmem)
{
    uint64_t* bars = sm.bars;
    const uint32_t s16 = smem_u32(sm.s16());
    uint32_t n_load = 0, n_conv[2] = {0, 0}, n_kt[2] = {0, 0}, n_p = 0, n_c1 = 0, n_o = 0;
    uint32_t n_s = 0, n_ds = 0;
    // DS^T = V^T Kt for the block in stage s (fresh accumulator), then release the stage.
    auto issue_vk = [&](int s) -> bool {
        if (!mbar_wait(&bars[B_KT0 + s], n_kt[s]++ & 1, sm.abort, p.hdr)) return false;
        if (!mbar_wait(&bars[B_DS_EMPTY], (n_ds++ & 1) ^ 1, sm.abort, p.hdr)) return false;
        tc_fence_after();
        const uint32_t kk = smem_u32(sm.k(s)), vv = smem_u32(sm.v(s));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + COL_DS, desc_mnmajor(vv, ks), desc_mnmajor(kk, ks), IDESC_VK,
                   ks > 0 ? 1u : 0u);
        mma_commit(&bars[B_DS_FULL]);
        mma_commit(&bars[B_EMPTY0 + s]);
        return true;
    };
    // SB = Q K^T for the block in stage (nl & 1), once the converters are done with it.
    auto issue_qk = [&](uint32_t nl) -> bool {
        const int s = nl & 1;
        if (!mbar_wait(&bars[B_CONV0 + s], n_conv[s]++ & 1, sm.abort, p.hdr)) return false;
        if (!mbar_wait(&bars[B_SB_FREE], (n_c1++ & 1) ^ 1, sm.abort, p.hdr)) return false;
        tc_fence_after();
        const uint32_t qq = smem_u32(sm.q(s)), kk = smem_u32(sm.k(s));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + COL_SB, desc_kmajor(qq, ks), desc_kmajor(kk, ks), IDESC_QK,
                   ks > 0 ? 1u : 0u);
        mma_commit(&bars[B_SBLK_FULL]);
        return true;
    };
    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!mbar_wait(&bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)) break;
        const Item it = sm.ring[slot];
        mbar_arrive(&bars[B_ITEM_EMPTY0 + slot]);
        if (!it.valid) break;
        const int nb = num_blocks(it.len);
        const bool has_succ = it.p_ord < it.nseg - 1;
        bool ok = true;
        if (has_succ) {
            // Phase A: the segment's local state, block by block (accumulated by OS).
            for (int b = 0; b < nb && ok; ++b) {
                ok = issue_vk(n_load & 1);
                ++n_load;
            }
            if (!ok) break;
        }
        // Phase C.
        if (!issue_qk(n_load)) break;
        for (int kb = 0; kb < nb && ok; ++kb) {
            const int s = n_load & 1;
            const uint32_t qq = smem_u32(sm.q(s)), vv = smem_u32(sm.v(s));
            ok = mbar_wait(&bars[B_P_READY], n_p++ & 1, sm.abort, p.hdr) &&
                 mbar_wait(&bars[B_O_EMPTY], (n_o++ & 1) ^ 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ts(tmem + COL_OI, tmem + COL_SB + ks * 8, desc_mnmajor(vv, ks), IDESC_PV,
                       ks > 0 ? 1u : 0u);
            mma_commit(&bars[B_SB_FREE]);
            ok = mbar_wait(&bars[B_S_READY], n_s++ & 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(tmem + COL_OE, desc_kmajor(qq, ks), desc_kmajor(s16, ks), IDESC_QS,
                       ks > 0 ? 1u : 0u);
            mma_commit(&bars[B_O_FULL]);
            // MMA4 of this block, then MMA1 of the next (its tiles are converted
            // while this block's epilogues run).
            if (!(ok = issue_vk(s))) break;
            if (kb + 1 < nb && !(ok = issue_qk(n_load + 1))) break;
            ++n_load;
        }
        if (!ok) break;
    }
    // Make sure no MMA is in flight before TMEM is released.
    mma_commit(&bars[B_FIN]);
    volatile int never = 0;
    mbar_wait(&bars[B_FIN], 0, &never, p.hdr, DRAIN_LIMIT_NS);
}

// Row r of a 16-bit tile as 64 packed words (two elements each).
__device__ __forceinline__ void load_row_packed(const uint8_t* tile, int r, uint32_t (&w)[64])
{
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint4 x = *reinterpret_cast<const uint4*>(tile + chunk_off(r, c));
        w[4 * c + 0] = x.x;
        w[4 * c + 1] = x.y;
        w[4 * c + 2] = x.z;
        w[4 * c + 3] = x.w;
    }
}

__device__ __forceinline__ float absmax_bf16_packed(const uint32_t (&w)[64])
{
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    return m;
}

// Store packed bf16 words times f as fp16 into row r.
__device__ __forceinline__ void store_bf16_packed_as_f16(uint8_t* tile, int r,
                                                         const uint32_t (&w)[64], float f)
{
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        uint4 x;
        x.x = pack_f16x2(bf16_lo(w[4 * c + 0]) * f, bf16_hi(w[4 * c + 0]) * f);
        x.y = pack_f16x2(bf16_lo(w[4 * c + 1]) * f, bf16_hi(w[4 * c + 1]) * f);
        x.z = pack_f16x2(bf16_lo(w[4 * c + 2]) * f, bf16_hi(w[4 * c + 2]) * f);
        x.w = pack_f16x2(bf16_lo(w[4 * c + 3]) * f, bf16_hi(w[4 * c + 3]) * f);
        *reinterpret_cast<uint4*>(tile + chunk_off(r, c)) = x;
    }
}

// Max |x| of row r of a bf16 tile (streaming, few registers). With the sign
// bit cleared, bf16 bit patterns order like their magnitudes, so the maximum
// is a packed unsigned 16-bit maximum.
__device__ __forceinline__ float row_absmax_bf16(const uint8_t* tile, int r)
{
    uint32_t m = 0u;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        const uint4 x = *reinterpret_cast<const uint4*>(tile + chunk_off(r, c));
        m = __vmaxu2(m, __vmaxu2(__vmaxu2(x.x & 0x7fff7fffu, x.y & 0x7fff7fffu),
                                 __vmaxu2(x.z & 0x7fff7fffu, x.w & 0x7fff7fffu)));
    }
    return fmaxf(bf16_lo(m), bf16_hi(m));
}

// Rewrite row r of a bf16 tile in place as fp16 times f (streaming).
__device__ __forceinline__ void row_bf16_to_f16(uint8_t* tile, int r, float f)
{
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        uint4* ptr = reinterpret_cast<uint4*>(tile + chunk_off(r, c));
        const uint4 x = *ptr;
        *ptr = make_uint4(pack_f16x2(bf16_lo(x.x) * f, bf16_hi(x.x) * f),
                          pack_f16x2(bf16_lo(x.y) * f, bf16_hi(x.y) * f),
                          pack_f16x2(bf16_lo(x.z) * f, bf16_hi(x.z) * f),
                          pack_f16x2(bf16_lo(x.w) * f, bf16_hi(x.w) * f));
    }
}

// Q converters (the two spare warps of the control warpgroup): fp16 Q with
// one power-of-two scale per row, for phase-C blocks, in parallel with the K
// and V converters. Thread t owns rows t and t + 64.
__device__ void qcv_role(const Params& p, const Smem& sm, int warp, int lane)
{
    uint64_t* bars = sm.bars;
    const int t = ((warp & 1) << 5) | lane;
    uint32_t n_load = 0, n_q[2] = {0, 0};
    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!wait_warp(&bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)) break;
        const Item it = sm.ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_ITEM_EMPTY0 + slot]);
        if (!it.valid) break;
        const int nb = num_blocks(it.len);
        bool ok = true;
        for (int pass = it.p_ord < it.nseg - 1 ? 0 : 1; pass < 2 && ok; ++pass) {
            for (int kb = 0; kb < nb && ok; ++kb) {
                const int s = n_load & 1;
                const int sl = n_load & 3;
                ok = wait_warp(&bars[B_SC_EMPTY0 + sl], ((n_load >> 2) & 1) ^ 1, sm.abort, p.hdr);
                if (!ok) break;
                if (pass == 1) {
                    ok = wait_warp(&bars[B_QFULL0 + s], n_q[s]++ & 1, sm.abort, p.hdr);
                    if (!ok) break;
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        const int r = t + 64 * h;
                        const Pow2 qs = pow2_for(row_absmax_bf16(sm.q(s), r));
                        row_bf16_to_f16(sm.q(s), r, qs.down);
                        sm.sc[sl].qe[r] = qs.ue;
                    }
                    fence_proxy_async();
                    mbar_arrive(&bars[B_CONV0 + s]);
                }
                mbar_arrive(&bars[B_SC_FULL0 + sl]);
                ++n_load;
            }
        }
        if (!ok) break;
    }
}

// Converter group: fp16 operands for the tensor cores as soon as a block's
// tiles land. Thread r owns row r of each tile. Q rows get their own
// power-of-two scale; K and V get one scale per tile (a maximum over the
// group). Phase-A blocks only need the decayed keys and V. The scales go to
// the OS group through the ScaleRec ring.
__device__ void cv_role(const Params& p, const Smem& sm, int warp, int lane)
{
    uint64_t* bars = sm.bars;
    const int r = ((warp & 3) << 5) | lane;
    const int w = warp & 3;
    const int rev = p.reverse;
    uint32_t n_load = 0, n_sync = 0;

    // Tile maxima of (a, b) over the 128 rows.
    auto tile_max2 = [&](float& a, float& b) -> bool {
        a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
        b = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(b)));
        float* red = sm.red + (n_load & 1) * 8;
        if (lane == 0) {
            red[w] = a;
            red[4 + w] = b;
        }
        if (!group_sync(&bars[B_CV_SYNC], n_sync, sm.abort, p.hdr)) return false;
        a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        b = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
        return true;
    };

    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!wait_warp(&bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)) break;
        const Item it = sm.ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_ITEM_EMPTY0 + slot]);
        if (!it.valid) break;
        const float slope = p.slopes[it.head];
        const int nb = num_blocks(it.len);
        const bool has_succ = it.p_ord < it.nseg - 1;
        bool ok = true;
        for (int pass = has_succ ? 0 : 1; pass < 2 && ok; ++pass) {
            for (int kb = 0; kb < nb && ok; ++kb) {
                const int s = n_load & 1;
                const int L = min(C, it.len - block_t0(it.len, kb, rev));
                const int sl = n_load & 3;
                ScaleRec* rec = sm.sc + sl;
                ok = wait_warp(&bars[B_FULL0 + s], (n_load >> 1) & 1, sm.abort, p.hdr) &&
                     wait_warp(&bars[B_SC_EMPTY0 + sl], ((n_load >> 2) & 1) ^ 1, sm.abort, p.hdr);
                if (!ok) break;
                const bool live = r < L;
                // K (phase A: already decayed) and V: one scale per tile.
                const float kf = pass == 0
                                     ? (live ? expf(-slope * (float)(rev ? r : L - 1 - r)) : 0.f)
                                     : (live ? 1.f : 0.f);
                float km = row_absmax_bf16(sm.k(s), r) * kf;
                float vm = live ? row_absmax_bf16(sm.v(s), r) : 0.f;
                if (!(ok = tile_max2(km, vm))) break;
                const Pow2 ks = pow2_for(km), vs = pow2_for(vm);
                row_bf16_to_f16(sm.v(s), r, live ? vs.down : 0.f);
                row_bf16_to_f16(sm.k(s), r, kf * ks.down);
                if (r == 0) {
                    rec->kc = ks.ue;
                    rec->vc = vs.ue;
                }
                fence_proxy_async();
                mbar_arrive(&bars[pass == 0 ? B_KT0 + s : B_CONV0 + s]);
                mbar_arrive(&bars[B_SC_FULL0 + sl]);
                ++n_load;
            }
        }
        if (!ok) break;
    }
}

// PE group: after Q K^T, the decayed causal mask (fp16 P into TMEM, in place
// over the scores) and the decayed keys for the state update (in place over
// K). Thread i owns TMEM lane / tile row i.
template <int REV>
__device__ void pe_role(const Params& p, const Smem& sm, uint32_t tmem, int warp, int lane)
{
    uint64_t* bars = sm.bars;
    const int w = warp & 3;
    const int row = (w << 5) | lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(w << 5) << 16);
    float* pw = sm.pw_pe;
    uint32_t n_load = 0, n_sblk = 0, n_sync = 0;
    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!wait_warp(&bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)) break;
        const Item it = sm.ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_ITEM_EMPTY0 + slot]);
        if (!it.valid) break;
        const float slope = p.slopes[it.head];
        if (!group_sync(&bars[B_PE_SYNC], n_sync, sm.abort, p.hdr)) break;
        pw[row] = expf(-slope * (float)row);
        if (row == 0) pw[C] = expf(-slope * (float)C);
        if (!group_sync(&bars[B_PE_SYNC], n_sync, sm.abort, p.hdr)) break;
        const int nb = num_blocks(it.len);
        if (it.p_ord < it.nseg - 1) n_load += nb;  // phase A blocks need no PE work
        bool ok = true;
        for (int kb = 0; kb < nb && ok; ++kb) {
            const int s = n_load & 1;
            const int L = min(C, it.len - block_t0(it.len, kb, REV));
            ok = wait_warp(&bars[B_SBLK_FULL], n_sblk++ & 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
            // E_P. Chunk c covers columns 32c..32c+31; warp w holds rows
            // 32w..32w+31, so chunks before (forward) / after (reverse) the
            // diagonal chunk are fully causal and the rest fully masked.
            const bool row_live = REV ? true : row < L;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
                const bool active = REV ? (c >= w) : (c <= w);
                if (active) {
                    uint32_t r32[32];
                    tmem_ld32(lane_addr + COL_SB + 32 * c, r32);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float x2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int j = 32 * c + e + u;
                            bool keep;
                            int m;
                            if (REV) {
                                keep = (c > w || j >= row) && j < L;
                                m = j - row;
                            } else {
                                keep = (c < w || j <= row) && row_live;
                                m = row - j;
                            }
                            x2[u] = keep ? __uint_as_float(r32[e + u]) * pw[keep ? m : 0] : 0.f;
                        }
                        pk[e >> 1] = pack_f16x2(x2[0], x2[1]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                }
                tmem_st16(lane_addr + COL_SB + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_P_READY]);
            // E_K: decayed keys lam^(L-1-j) k_j (reverse: lam^j), in place (fp16).
            {
                const float f = row < L ? pw[REV ? row : L - 1 - row] : 0.f;
                uint8_t* kt = sm.k(s);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint4* ptr = reinterpret_cast<uint4*>(kt + chunk_off(row, c));
                    uint4 x = *ptr;
                    uint32_t* e4 = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&e4[u]));
                        e4[u] = pack_f16x2(h.x * f, h.y * f);
                    }
                    *ptr = x;
                }
            }
            fence_proxy_async();
            mbar_arrive(&bars[B_KT0 + s]);
            ++n_load;
        }
        if (!ok) break;
    }
}

// OS group: S = lam^L S + up * DS for the next DS use (phase A or C).
__device__ __forceinline__ bool os_accumulate_ds(const Params& p, const Smem& sm,
                                                 uint32_t lane_addr, float (&S)[D], int L,
                                                 float slope, float up, uint32_t& n_ds)
{
    if (!wait_warp(&sm.bars[B_DS_FULL], n_ds & 1, sm.abort, p.hdr)) return false;
    tc_fence_after();
    const float dL = expf(-slope * (float)L);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_addr + COL_DS + 32 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x)
            S[32 * c + x] = fmaf(dL, S[32 * c + x], up * __uint_as_float(r[x]));
    }
    tc_fence_before();
    mbar_arrive(&sm.bars[B_DS_EMPTY]);
    mbar_arrive(&sm.bars[B_SC_EMPTY0 + (n_ds & 3)]);
    ++n_ds;
    return true;
}

// OS group: fp16 copy of the state for MMA3 (row a of S^T). One power-of-two
// scale per 32 state columns (one warp), from a warp-wide maximum.
__device__ __forceinline__ void os_publish_s16(const Smem& sm, int a, const float (&S)[D], int par)
{
    const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(row_absmax(S))));
    const Pow2 sc = pow2_for(m);
    store_row_f16(sm.s16(), a, S, sc.down);
    if ((a & 31) == 0) sm.hs[par * 4 + (a >> 5)] = sc.ue;
    fence_proxy_async();
    mbar_arrive(&sm.bars[B_S_READY]);
}

template <int REV, int OUT_F32>
__device__ void os_role(const Params& p, const Smem& sm, uint32_t tmem, int warp, int lane)
{
    uint64_t* bars = sm.bars;
    const int a = ((warp & 3) << 5) | lane;  // TMEM lane: output row i / state column a
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) << 5) << 16);
    float slope = 0.f;
    // n_blk counts phase-C blocks (one o_full and s_ready phase each);
    // n_ds counts DS uses (= blocks loaded = scale records).
    uint32_t n_sync = 0, n_blk = 0, n_ds = 0;
    float S[D];  // column a of the fp32 state: S[x] = state[x][a]

    for (uint32_t k = 0;; ++k) {
        const int slot = k & 1;
        if (!wait_warp(&bars[B_ITEM_FULL0 + slot], (k >> 1) & 1, sm.abort, p.hdr)) break;
        const Item it = sm.ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_ITEM_EMPTY0 + slot]);
        if (!it.valid) break;
        slope = p.slopes[it.head];
        const int nb = num_blocks(it.len);
        const bool has_succ = it.p_ord < it.nseg - 1;
        bool ok = true;

#pragma unroll
        for (int x = 0; x < D; ++x) S[x] = 0.f;
        if (has_succ) {
            // Phase A: local state of the segment.
            for (int kb = 0; kb < nb && ok; ++kb) {
                const int L = min(C, it.len - block_t0(it.len, kb, REV));
                const ScaleRec* rec = sm.sc + (n_ds & 3);
                ok = wait_warp(&bars[B_SC_FULL0 + (n_ds & 3)], (n_ds >> 2) & 1, sm.abort, p.hdr);
                if (!ok) break;
                const float up = up_of(rec->kc) * up_of(rec->vc);
                ok = os_accumulate_ds(p, sm, lane_addr, S, L, slope, up, n_ds);
            }
            if (!ok) break;
        }
        // Incoming state: the predecessor's inclusive prefix (zero for the first segment).
        const float* src = p.incl + ((size_t)it.chain * 2 + ((it.p_ord - 1) & 1)) * D * D +
                           (size_t)a * D;
        if (it.p_ord > 0) {
            if (a == 0) {
                const int* flag = p.chain_flags + it.chain;
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
            if (!group_sync(&bars[B_OS_SYNC], n_sync, sm.abort, p.hdr)) break;
        }
        {
            // S_prev = the predecessor's inclusive prefix (0 for the first
            // segment). With a successor, publish lam^len S_prev + S_loc.
            // Phase C continues from S_prev.
            const float dl = expf(-slope * (float)it.len);
            float* dst = p.incl + ((size_t)it.chain * 2 + (it.p_ord & 1)) * D * D + (size_t)a * D;
            const bool has_prev = it.p_ord > 0;
#pragma unroll
            for (int x = 0; x < D / 4; ++x) {
                const float4 w = has_prev ? ld_cg_ordered(src + 4 * x) : make_float4(0.f, 0.f, 0.f, 0.f);
                if (has_succ)
                    st_cg_ordered(dst + 4 * x,
                                  make_float4(fmaf(dl, w.x, S[4 * x + 0]), fmaf(dl, w.y, S[4 * x + 1]),
                                              fmaf(dl, w.z, S[4 * x + 2]), fmaf(dl, w.w, S[4 * x + 3])));
                S[4 * x + 0] = w.x;
                S[4 * x + 1] = w.y;
                S[4 * x + 2] = w.z;
                S[4 * x + 3] = w.w;
            }
        }
        if (has_succ) {
            __threadfence();
            if (!group_sync(&bars[B_OS_SYNC], n_sync, sm.abort, p.hdr)) break;
            if (a == 0 && !p.skip_publish) {
                int* flag = p.chain_flags + it.chain;
                asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(it.p_ord + 1) : "memory");
            }
        }
        os_publish_s16(sm, a, S, n_blk & 1);

        for (int kb = 0; kb < nb && ok; ++kb) {
            const int par = n_blk & 1;
            const int t0 = block_t0(it.len, kb, REV);
            const int L = min(C, it.len - t0);
            const ScaleRec* rec = sm.sc + (n_ds & 3);
            // E_O: O = up_Q up_K up_V * OI + lam^(i+1) * up_Q * up_S[col] * OE
            // (reverse: lam^(L-i)).
            ok = wait_warp(&bars[B_O_FULL], n_blk & 1, sm.abort, p.hdr) &&
                 wait_warp(&bars[B_S_READY], n_blk & 1, sm.abort, p.hdr) &&
                 wait_warp(&bars[B_SC_FULL0 + (n_ds & 3)], (n_ds >> 2) & 1, sm.abort, p.hdr);
            if (!ok) break;
            tc_fence_after();
            const float up_kv = up_of(rec->kc) * up_of(rec->vc);
            const float up_q = up_of(rec->qe[a]);
            const float gi = up_q * up_kv;
            const float rowc = expf(-slope * (float)(REV ? max(L - a, 0) : a + 1)) * up_q;
            const uint8_t* hsp = sm.hs + par * 4;
            const bool store = a < L;
            const long long orow = it.out_row0 + t0 + a;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t ri[16], re[16];
                tmem_ld16(lane_addr + COL_OI + 16 * c, ri);
                tmem_ld16(lane_addr + COL_OE + 16 * c, re);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float ov[8];
                    const float ec = rowc * up_of(hsp[c >> 1]);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        ov[x] = fmaf(ec, __uint_as_float(re[8 * h + x]), gi * __uint_as_float(ri[8 * h + x]));
                    if (store) {
                        if (OUT_F32) {
                            float4* dst = reinterpret_cast<float4*>(
                                static_cast<float*>(p.o) + orow * D + 16 * c + 8 * h);
                            dst[0] = make_float4(ov[0], ov[1], ov[2], ov[3]);
                            dst[1] = make_float4(ov[4], ov[5], ov[6], ov[7]);
                        } else {
                            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow * D +
                                                      16 * c + 8 * h) =
                                make_uint4(pack_bf16x2(ov[0], ov[1]), pack_bf16x2(ov[2], ov[3]),
                                           pack_bf16x2(ov[4], ov[5]), pack_bf16x2(ov[6], ov[7]));
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[B_O_EMPTY]);
            // E_S.
            if (!(ok = os_accumulate_ds(p, sm, lane_addr, S, L, slope, up_kv, n_ds))) break;
            if (kb + 1 < nb) os_publish_s16(sm, a, S, (n_blk + 1) & 1);
            ++n_blk;
        }
        if (!ok) break;
        if (it.p_ord == it.nseg - 1 && p.state_out) {
            float* dst = p.state_out + (size_t)it.chain * D * D + a;
#pragma unroll
            for (int x = 0; x < D; ++x) dst[(size_t)x * D] = S[x];
        }
    }
}

// Small shared state at the start of the dynamic region; the 1024-aligned
// tile region follows (SMEM_BYTES reserves the worst-case alignment gap).
constexpr uint32_t SM_BARS = 0;                       // 36 x 8 B
constexpr uint32_t SM_RING = 288;                     // 2 x Item
constexpr uint32_t SM_PW = 384;                       // (C+1) floats
constexpr uint32_t SM_SC = 912;                       // 4 x ScaleRec (144 B)
constexpr uint32_t SM_RED = SM_SC + 4 * 144;          // 16 floats
constexpr uint32_t SM_HS = SM_RED + 64;               // [2][128] bytes
constexpr uint32_t SM_TMEM = SM_HS + 256;             // u32
constexpr uint32_t SM_ABORT = SM_TMEM + 4;            // int
constexpr uint32_t SM_SMALL = SM_ABORT + 4;
static_assert(NUM_BARS <= 36, "barrier area");
static_assert(sizeof(Item) * 2 <= SM_PW - SM_RING, "ring area");
static_assert(SM_PW + (C + 1) * 4 <= SM_SC, "pw area");
static_assert(sizeof(ScaleRec) == 144, "scale record");
constexpr uint32_t SMEM_BYTES = SM_SMALL + 1023 + SMEM_TILES;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

template <int REV, int OUT_F32>
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
    sm.pw_pe = reinterpret_cast<float*>(dsmem + SM_PW);
    sm.sc = reinterpret_cast<ScaleRec*>(dsmem + SM_SC);
    sm.red = reinterpret_cast<float*>(dsmem + SM_RED);
    sm.hs = dsmem + SM_HS;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        uint32_t counts[NUM_BARS];
        for (int i = 0; i < NUM_BARS; ++i) counts[i] = 128;
        counts[B_FULL0] = counts[B_FULL1] = counts[B_EMPTY0] = counts[B_EMPTY1] = 1;
        counts[B_SBLK_FULL] = counts[B_SB_FREE] = counts[B_O_FULL] = counts[B_DS_FULL] = 1;
        counts[B_ITEM_FULL0] = counts[B_ITEM_FULL1] = counts[B_FIN] = 1;
        counts[B_QFULL0] = counts[B_QFULL1] = 1;
        counts[B_ITEM_EMPTY0] = counts[B_ITEM_EMPTY1] = 15;  // MMA lane + 14 group warps
        // Q converters (64 threads) join the K/V converters (128).
        counts[B_CONV0] = counts[B_CONV1] = 192;
        counts[B_SC_FULL0] = counts[B_SC_FULL1] = counts[B_SC_FULL2] = counts[B_SC_FULL3] = 192;
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], counts[i]);
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
        if (warp == 0 && lane == 0) producer_role(p, &tq, &tk, &tv, sm);
        if (warp == 1 && lane == 0) mma_role(p, sm, tmem);
        if (warp >= 2) qcv_role(p, sm, warp, lane);
    } else if (warp < 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_CV));
        cv_role(p, sm, warp, lane);
    } else if (warp < 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PE));
        pe_role<REV>(p, sm, tmem, warp, lane);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_OS));
        os_role<REV, OUT_F32>(p, sm, tmem, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

// Varlen planner: segment-major list of (chain, p_ord, nseg) items; zero
// states for empty sequences. One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) plan_varlen_kernel(const int* cu, int num_seqs, int H,
                                                           int seg, int4* items, int max_items,
                                                           WsHeader* hdr, float* state_out)
{
    __shared__ int warp_tot[32];
    __shared__ int s_max;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto nseg_of = [&](int s) -> int {
        const long long L = (long long)cu[s + 1] - cu[s];
        return L > 0 ? (int)((L + seg - 1) / seg) : 0;
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
            for (int x = tid; x < H * D * D / 4; x += blockDim.x) dst[x] = make_float4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    const int maxseg = s_max;
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

// Segment length: the tuning value, or the candidate among 1K..8K tokens
// that minimises (rounds of persistent CTAs) x (blocks per item + fixed
// per-item cost), with phase A counted for items that have a successor.
static int choose_seg(const Problems& P, int seg_tuning, bool varlen)
{
    if (seg_tuning > 0) return seg_tuning;
    if (varlen) return 2048;
    const long long N = P.N, chains = P.count();
    const int sms = 148;
    if (N <= 1024) return (int)std::max<long long>(128, (N + 127) / 128 * 128);
    double best = 1e300;
    int best_seg = 2048;
    for (int seg = 1024; seg <= 8192; seg *= 2) {
        const long long nseg = (N + seg - 1) / seg;
        const long long items = chains * nseg;
        const double rounds = (double)((items + sms - 1) / sms);
        const double blocks = seg / 128.0;
        const double per_item = blocks * (nseg > 1 ? 1.25 : 1.0) + 3.0;
        const double cost = rounds * per_item;
        if (cost < best * 0.999) {
            best = cost;
            best_seg = seg;
        }
    }
    return best_seg;
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
    w.items = align_up(w.flags + sizeof(int) * (size_t)w.nchains, 256);
    w.incl = align_up(w.items + (varlen ? sizeof(int4) * (size_t)w.max_items : 0), 256);
    w.end = align_up(w.incl + sizeof(float) * (size_t)w.nchains * 2 * D * D, 256);
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
                              int seg_tuning, void* workspace, cudaStream_t stream, int reverse)
{
    using namespace tc;
    (void)d;
    const bool varlen = P.cu_seqlens != nullptr;
    const int seg = choose_seg(P, seg_tuning, varlen);
    const WsLayout w = layout(P, seg, varlen);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaError_t err;
    if (!varlen && P.N == 0) {
        if (state_out)
            return cudaMemsetAsync(state_out, 0, sizeof(float) * (size_t)P.count() * D * D, stream);
        return cudaSuccess;
    }
    if (varlen && P.total == 0 && P.num_seqs == 0) return cudaSuccess;
    // Clear the header and per-chain counters.
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
                                                    prm.hdr, state_out);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        if (P.total == 0) return cudaSuccess;
    }
    const long long max_items = w.max_items;
    const int grid = (int)std::min<long long>(num_sms(), std::max<long long>(1, max_items));
    auto launch = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, mv, prm);
        count_launch();
        return cudaGetLastError();
    };
    const bool f32 = out_t == LA_F32;
    if (reverse)
        return f32 ? launch(tc_forward_kernel<1, 1>) : launch(tc_forward_kernel<1, 0>);
    return f32 ? launch(tc_forward_kernel<0, 1>) : launch(tc_forward_kernel<0, 0>);
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
