// attn_fwd_sm100.cuh -- warp-specialised bf16 attention forward for sm_100a.
//
// One CTA owns two 128-row query tiles of one (batch, head) and streams the
// key/value sequence through shared memory in 128-key tiles:
//
//   S_t = Q_t K_j^T               tcgen05.mma, both operands in smem, fp32 acc in TMEM
//   P_t = exp2(S_t*scale*log2e - m_t)   softmax warps, registers, P back to TMEM as bf16
//   O_t += P_t V_j                tcgen05.mma, P from TMEM, V from smem
//
// This is the streaming ("online") softmax that avoids materialising the
// S x S score matrix -- the FlashAttention bullet of "Realtime video
// generation: FLOPS calculation and optimizations" (sudonull.com) -- with
// the running row maximum and row sum kept per query row ("VC-Attention"
// (aikraft.ru), section 02, Restore step: the online softmax already holds
// the row sum).  The exp + cast between the two products is the long pole on
// B200 (same page, section 01), so:
//   * the softmax runs in two warpgroups that alternate with the tensor core:
//     while warpgroup 0 exponentiates tile 0, the tensor core computes P_1 V
//     and S_1 for tile 1, and vice versa;
//   * P is handed over in two 64-key halves, so O_t += P_t V starts on keys
//     0-63 while keys 64-127 are still being exponentiated;
//   * the scale-and-subtract and the row sum run as packed fp32x2 ops, so the
//     issue slots left over around MUFU ex2 stay free for the other warps;
//   * after the first key tile the reference max moves only when a score
//     exceeds it by more than 2^8 (lazy rescaling), and that is checked
//     without a full 128-key max: keys 0-63 are exponentiated against the
//     current reference first, and one of them exceeds it by more than the
//     threshold only if their exponentials sum to more than 2^8; keys 64-127
//     are checked by their max.  The exact tile max is taken only when a
//     check fires;
//   * O leaves through shared memory: after its last P V each tile stages
//     its rows in a ring slot that no product or load uses any more, and one
//     lane per warp stores them with TMA.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3   softmax + correction + epilogue of query tile 0
//   warps 4-7   softmax + correction + epilogue of query tile 1
//   warp  8     TMA producer (Q once, then K_j, V_j into a 4-slot ring)
//   warp  9     TMEM allocator and single-thread tcgen05.mma issuer
//   warp  10    block-sparse only: builds the two tiles' key lists, then idles
//   warp  11    idle
// The kernel is launched at 168 registers a thread (384 x 168 = 64,512); the
// softmax warpgroups then raise theirs to 208 and the third lowers its to 88
// (2 x 128 x 208 + 128 x 88 = 64,512, the same total).
//
// TMEM (512 columns x 128 lanes, fp32): S_0 [0,128), S_1 [128,256),
// O_0 [256,384), O_1 [384,512).  P_t (bf16, two per column) overwrites the
// first 64 columns of S_t; query row r of a tile lives in TMEM lane r.
//
// Every wait on a pipeline barrier is bounded: when it runs out the CTA
// raises a shared abort flag, ORs a code into the device status word, and
// every role leaves its loop so the CTA still reaches teardown.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace vdit {

constexpr int kBlockM = 128;   // query rows per tile
constexpr int kBlockN = 128;   // keys per K/V tile
constexpr int kHeadDim = 128;  // D
constexpr int kQTiles = 2;     // query tiles per CTA
constexpr int kStages = 4;     // K/V ring slots (each holds one K or one V tile)
constexpr int kTileBytes = kBlockM * kHeadDim * 2;  // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;          // 128 rows x 64 bf16, 128B-swizzled
constexpr int kNumThreads = 384;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kLaunchRegs = 168;    // ptxas allocation at launch (checked by the build)
constexpr int kSoftmaxRegs = 208;   // after setmaxnreg.inc in warpgroups 0 and 1
constexpr int kControlRegs = 88;    // after setmaxnreg.dec in warpgroup 2
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kNumThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr int kStageRows = 32;                             // dense epilogue: one warp's rows, staged in a ring slot
constexpr int kStageCols = 64;                             // head dims per TMA store box (128 bytes, 128B-swizzled)
constexpr int kStageWarpBytes = kStageRows * kHeadDim * 2;  // 8 KB per softmax warp: two boxes
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

constexpr int kMaskFull = 0;
constexpr int kMaskBlockCausal = 1;
constexpr int kMaskCross = 2;
constexpr int kMaskBlockSparse = 3;
constexpr int kSparseBlock = 128;        // block-mask granularity = the 128-row/128-key tiles
constexpr int kMaxSparseKvBlocks = 2048; // key blocks a block-sparse call may have (Skv <= 262,144)
constexpr int kMaxSparseEntries = 2 * kMaxSparseKvBlocks;  // both query tiles' key lists, interleaved
constexpr int kListWarp = 10;

// Device status word codes (OR-ed together).
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kSiteProducer = 1u << 8;
constexpr uint32_t kSiteMma = 1u << 9;
constexpr uint32_t kSiteSoftmax = 1u << 10;

struct __align__(8) Barriers {
    uint64_t q_full[kQTiles];
    uint64_t kv_full[kStages];
    uint64_t kv_empty[kStages];
    uint64_t s_full[kQTiles];
    uint64_t p_full[kQTiles][2];  // P keys 0-63 / 64-127 of tile t in TMEM
    uint64_t o_full[kQTiles];
    uint64_t drain;  // MMA issuer's own completion barrier on the abort path
    uint32_t tmem_base;
    int abort;
};

constexpr int kSmemQ = 0;
constexpr int kSmemKV = kQTiles * kTileBytes;
constexpr int kSmemBar = kSmemKV + kStages * kTileBytes;
constexpr int kSmemList = kSmemBar + ((int(sizeof(Barriers)) + 15) / 16) * 16;  // block-sparse tile list
constexpr int kSmemBytes = kSmemList + kMaxSparseKvBlocks * 2 + 16 + 1024;     // + alignment slack
// the block-sparse instantiation holds both tiles' key lists (twice the room)
constexpr int kSmemBytesSparse = kSmemList + kMaxSparseEntries * 2 + 16 + 1024;

struct FwdParams {
    int B, H, Sq, Skv;
    int mask_kind;
    int chunk;
    float scale_log2;  // scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
    unsigned long long timeout_ns;
    int debug_flags;  // test-only fault injection (kDebug*); 0 in every product call
    const uint8_t* block_mask;  // block-sparse: [B][H][n_qb][n_kvb], nonzero = attend
    int n_qb, n_kvb;            // ceil(Sq / 128), ceil(Skv / 128)
};

// Test-only: the producer withholds every K/V tile, so the MMA issuer's
// bounded wait on the first K tile runs out and the timeout path runs.
constexpr int kDebugWithholdKV = 1;

// Written by kernels when a bounded wait runs out; read and cleared by the host.
__device__ uint32_t g_status_word = 0;

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 format:
// start address >> 4 in bits [0,14), leading byte offset >> 4 in [16,30),
// stride byte offset >> 4 in [32,46), version 1 in [46,48), layout 2
// (SWIZZLE_128B) in [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits [4,6) = 1),
// A = B = bf16 ([7,10) = [10,13) = 1), A K-major, B K-major or MN-major
// (bit 16), N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t make_idesc_bf16(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (uint32_t(kBlockN >> 3) << 17) | (uint32_t(kBlockM >> 4) << 24);
}

// ---------------------------------------------------------------- waits

__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                             unsigned long long timeout_ns, uint32_t site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort = 1;
                atomicOr(&g_status_word, kStatusTimeout | site);
                return false;
            }
        }
    }
}

// All 32 lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          unsigned long long timeout_ns, uint32_t site) {
    const bool ok = bounded_wait(bar, parity, abort, timeout_ns, site);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- MMA helpers

// The MMA issuer keeps one descriptor per operand base and advances it by
// adding (byte offset >> 4) to the start-address field: every operand offset
// used below stays inside the 14-bit field, so the add never carries into the
// leading-byte-offset bits.
//
// S[128 x 128] = Q_tile[128 x 128] * K_tile[128 x 128]^T, both K-major with
// 128B swizzle, each stored as two 16 KB halves (head dims 0-63 and 64-127).
// K = 16 per instruction: 4 steps of 32 bytes inside a half, then the next half.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
    constexpr uint32_t idesc = make_idesc_bf16(false);
    static_assert(kHalfBytes == 16384, "descriptor offsets below assume 16 KB halves");
    // The eight K = 16 steps in one asm block: the descriptors advance by
    // 32 bytes (2 in the >> 4 address field) within a 64-dim half and by
    // 16 KB (1024) to the second half; the first step overwrites the
    // accumulator, the others add.  One thread issues these faster as one
    // block than as eight separate statements.
    asm volatile(
        "{\n\t.reg .pred pf, pt;\n\t.reg .b64 a, b;\n\t"
        "setp.ne.b32 pf, %3, %3;\n\t"
        "setp.eq.b32 pt, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pf;\n\t"
        "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 1024;\n\tadd.s64 b, %2, 1024;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 1026;\n\tadd.s64 b, %2, 1026;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 1028;\n\tadd.s64 b, %2, 1028;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
        "add.s64 a, %1, 1030;\n\tadd.s64 b, %2, 1030;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t}" ::"r"(d_tmem),
        "l"(q_desc), "l"(k_desc), "r"(idesc)
        : "memory");
}

// O[128 x 128] (+)= P[128 x keys] * V_tile[keys x 128] for the 64 keys of
// `half`.  P comes from TMEM (two bf16 per column, 8 columns per K = 16
// step).  V is the B operand in MN-major form: head dim is contiguous; 64-dim
// halves are 16 KB apart (leading byte offset), 8-key row groups 1 KB apart
// (stride byte offset), and each 16-key step advances 16 rows = 2 KB.  The
// four steps are one asm block; the first accumulates unless it starts O.
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, int half,
                                              bool accumulate) {
    constexpr uint32_t idesc = make_idesc_bf16(true);
    const uint32_t a0 = p_tmem + uint32_t(half) * 32u;
    const uint64_t b0 = v_desc + uint64_t(half) * 512u;
    asm volatile(
        "{\n\t.reg .pred p0, pt;\n\t.reg .b32 a;\n\t.reg .b64 b;\n\t"
        "setp.ne.b32 p0, %4, 0;\n\t"
        "setp.eq.b32 pt, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
        "add.u32 a, %1, 8;\n\tadd.s64 b, %2, 128;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, pt;\n\t"
        "add.u32 a, %1, 16;\n\tadd.s64 b, %2, 256;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, pt;\n\t"
        "add.u32 a, %1, 24;\n\tadd.s64 b, %2, 384;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, pt;\n\t}" ::"r"(d_tmem),
        "r"(a0), "l"(b0), "r"(idesc), "r"((accumulate || half > 0) ? 1u : 0u)
        : "memory");
}

// ---------------------------------------------------------------- softmax pieces

// Exponentiate 32 logits (one TMEM chunk of the row): x = s*scale*log2e - m as
// packed fp32x2 FMAs, 2^x on MUFU (ex2.approx), the fp32 row sum as packed
// adds into four accumulators, and bf16x2 packing of the pairs into pk[0..15].
// (Taking part of the exponentials on the FMA pipe with a polynomial was
// measured slower than MUFU alone at this occupancy, so every pair uses MUFU.)
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], uint64_t scale2, uint64_t negm2,
                                          uint32_t (&pk)[16], uint64_t (&lsum)[4]) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float x0, x1;
        ffma2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1]), scale2, negm2, x0, x1);
        const float p0 = ex2_approx(x0);
        const float p1 = ex2_approx(x1);
        fadd2_acc(lsum[k & 3], p0, p1);
        pk[k] = pack_bf16x2(p0, p1);
    }
}

// ---------------------------------------------------------------- kernel

// kSparse: the block-sparse instantiation.  Each query tile walks only the
// key blocks its own mask row allows; the two tiles' lists (n0 and n1
// entries) are interleaved into one stream, which the producer loads in
// order: entry k of tile t's list is stream entry 2k + t while k < both =
// min(n0, n1), then the longer list's rest follows (its entry k at 2 both +
// k - both).  So the tiles take turns with the tensor core and MUFU as in the
// dense schedule.  A key block both tiles need appears once for each.
// The dense, block-causal and cross instantiation keeps the plain issue
// order, in which both tiles take part in every key tile.
// tm_o: O as the same 4-D tensor as Q, with 64-dim x 32-row boxes, 128-byte
// swizzled: the dense epilogue's TMA store unit.
template <bool kSparse, bool kLongFirst = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                          const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    Barriers* bars = reinterpret_cast<Barriers*>(smem + kSmemBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = int(threadIdx.x >> 5);
    const int lane = int(threadIdx.x & 31);
    const int h = int(blockIdx.y);
    const int b = int(blockIdx.z);
    // kLongFirst (block-causal): the CTAs of later chunks walk more key tiles;
    // dispatching them first (blocks start in blockIdx order) leaves short
    // CTAs, not long ones, to fill the end of the grid.
    const int q_pair = kLongFirst ? int(gridDim.x - 1u - blockIdx.x) : int(blockIdx.x);
    const int q0 = q_pair * (kQTiles * kBlockM);

    if (threadIdx.x == 0) {
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(smem_addr(&bars->q_full[t]), 1);
            mbar_init(smem_addr(&bars->s_full[t]), 1);
            mbar_init(smem_addr(&bars->p_full[t][0]), 4);  // one elected arrive per softmax warp
            mbar_init(smem_addr(&bars->p_full[t][1]), 4);
            mbar_init(smem_addr(&bars->o_full[t]), 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&bars->kv_full[s]), 1);
            mbar_init(smem_addr(&bars->kv_empty[s]), 1);
        }
        mbar_init(smem_addr(&bars->drain), 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    uint16_t* kv_list = reinterpret_cast<uint16_t*>(smem + kSmemList);
    int* kv_list_len = reinterpret_cast<int*>(smem + kSmemList + kMaxSparseEntries * 2);  // total, n0, n1 (sparse)
    if (kSparse && warp == kListWarp) {
        // Each query tile's allowed key blocks in ascending order, in one
        // pass: tile 0's list at kv_list[0 ..), tile 1's at
        // kv_list[kMaxSparseKvBlocks ..).  The stream the producer loads
        // interleaves them; it is never stored.
        const int qb0 = q0 / kSparseBlock;
        const uint8_t* row0 = p.block_mask + ((static_cast<size_t>(b) * p.H + h) * p.n_qb + qb0) * p.n_kvb;
        const bool has_row1 = qb0 + 1 < p.n_qb;
        const uint32_t below = (1u << lane) - 1u;
        int c0 = 0, c1 = 0;
#pragma unroll 4
        for (int base = 0; base < p.n_kvb; base += 32) {
            const int kv = base + lane;
            const bool a0 = kv < p.n_kvb && row0[kv] != 0;
            const bool a1 = has_row1 && kv < p.n_kvb && row0[p.n_kvb + kv] != 0;
            const uint32_t b0 = __ballot_sync(0xffffffffu, a0);
            const uint32_t b1 = __ballot_sync(0xffffffffu, a1);
            if (a0) kv_list[c0 + __popc(b0 & below)] = uint16_t(kv);
            if (a1) kv_list[kMaxSparseKvBlocks + c1 + __popc(b1 & below)] = uint16_t(kv);
            c0 += __popc(b0);
            c1 += __popc(b1);
        }
        if (lane == 0) {
            kv_list_len[0] = c0 + c1;
            kv_list_len[1] = c0;
            kv_list_len[2] = c1;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    constexpr bool sparse = kSparse;

    // Keys this CTA needs: all of them, or for block-causal everything up to
    // the end of the chunk that holds the CTA's last valid query row.
    int kv_end = p.Skv;
    if (p.mask_kind == kMaskBlockCausal) {
        const int last_row = min(q0 + kQTiles * kBlockM - 1, p.Sq - 1);
        const long long lim = (static_cast<long long>(last_row / p.chunk) + 1) * p.chunk;
        kv_end = static_cast<int>(min(static_cast<long long>(p.Skv), lim));
    }
    const int n_kv = sparse ? *kv_list_len : (kv_end + kBlockN - 1) / kBlockN;

    const uint32_t sQ = smem_addr(smem + kSmemQ);
    const uint32_t sKV = smem_addr(smem + kSmemKV);

    if (warp >= 8) {
        setmaxnreg_dec<kControlRegs>();
        if (warp == kLoadWarp && lane == 0) {
            // ------------------------------------------------ TMA producer
            griddep_wait();  // Q/K written by a preceding kernel (fused Q/K norm) are complete
            for (int t = 0; n_kv > 0 && t < kQTiles; ++t) {
                const uint32_t bar = smem_addr(&bars->q_full[t]);
                mbar_arrive_expect_tx(bar, kTileBytes);
                tma_load_4d(sQ + t * kTileBytes, &tm_q, bar, 0, h, q0 + t * kBlockM, b);
                tma_load_4d(sQ + t * kTileBytes + kHalfBytes, &tm_q, bar, 64, h, q0 + t * kBlockM, b);
            }
            const int n_loads = (p.debug_flags & kDebugWithholdKV) ? 0 : 2 * n_kv;
            for (int u = 0; u < n_loads; ++u) {
                const int slot = u % kStages;
                const uint32_t phase = uint32_t(u / kStages) & 1u;
                if (!bounded_wait(smem_addr(&bars->kv_empty[slot]), phase ^ 1u, abort_flag, p.timeout_ns,
                                  kSiteProducer))
                    break;
                const uint32_t full = smem_addr(&bars->kv_full[slot]);
                const CUtensorMap* map = (u & 1) ? &tm_v : &tm_k;
                int blk = u >> 1;
                if constexpr (kSparse) {  // stream entry u >> 1 -> (tile, list entry)
                    const int e = u >> 1, n0 = kv_list_len[1], n1 = kv_list_len[2];
                    const int both2 = 2 * min(n0, n1);
                    blk = e < both2 ? int(kv_list[(e & 1) * kMaxSparseKvBlocks + (e >> 1)])
                                    : int(kv_list[(n0 >= n1 ? 0 : kMaxSparseKvBlocks) + (e - both2 / 2)]);
                }
                const int row = blk * kBlockN;
                mbar_arrive_expect_tx(full, kTileBytes);
                tma_load_4d(sKV + slot * kTileBytes, map, full, 0, h, row, b);
                tma_load_4d(sKV + slot * kTileBytes + kHalfBytes, map, full, 64, h, row, b);
            }
        } else if (warp == kMmaWarp && lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t tS[2] = {tmem, tmem + 128};
            const uint32_t tO[2] = {tmem + 256, tmem + 384};
            // descriptor bases: Q tiles (K-major), ring slots as K (K-major) and as V (MN-major)
            const uint64_t q_desc[2] = {smem_desc_sw128(sQ, 16, 1024), smem_desc_sw128(sQ + kTileBytes, 16, 1024)};
            const uint64_t k_desc0 = smem_desc_sw128(sKV, 16, 1024);
            const uint64_t v_desc0 = smem_desc_sw128(sKV, kHalfBytes, 1024);
            constexpr uint64_t kSlotStep = kTileBytes >> 4;
            bool ok = n_kv > 0 &&
                      bounded_wait(smem_addr(&bars->q_full[0]), 0, abort_flag, p.timeout_ns, kSiteMma) &&
                      bounded_wait(smem_addr(&bars->q_full[1]), 0, abort_flag, p.timeout_ns, kSiteMma);
            if constexpr (!kSparse) {
            // prologue: S_0 and S_1 against K_0
            if (ok) ok = bounded_wait(smem_addr(&bars->kv_full[0]), 0, abort_flag, p.timeout_ns, kSiteMma);
            if (ok) {
                tc_fence_after_sync();
                issue_qk(tS[0], q_desc[0], k_desc0);
                umma_commit(smem_addr(&bars->s_full[0]));
                issue_qk(tS[1], q_desc[1], k_desc0);
                umma_commit(smem_addr(&bars->s_full[1]));
                umma_commit(smem_addr(&bars->kv_empty[0]));
            }
            // steady state, per key tile j:
            //   PV0(j) [two halves]  S0(j+1)  PV1(j) [two halves]  S1(j+1)
            for (int j = 0; ok && j < n_kv; ++j) {
                const int uv = 2 * j + 1;
                const int v_slot = uv % kStages;
                const int uk = 2 * (j + 1);
                const int k_slot = uk % kStages;
                const uint32_t ph = uint32_t(j) & 1u;
                const bool more = (j + 1) < n_kv;
                ok = bounded_wait(smem_addr(&bars->kv_full[v_slot]), uint32_t(uv / kStages) & 1u, abort_flag,
                                  p.timeout_ns, kSiteMma);
                for (int t = 0; ok && t < kQTiles; ++t) {
                    for (int hf = 0; ok && hf < 2; ++hf) {
                        ok = bounded_wait(smem_addr(&bars->p_full[t][hf]), ph, abort_flag, p.timeout_ns, kSiteMma);
                        if (ok) {
                            tc_fence_after_sync();
                            issue_pv_half(tO[t], tS[t], v_desc0 + uint64_t(v_slot) * kSlotStep, hf, j > 0);
                        }
                    }
                    if (!ok) break;
                    if (t == 1) umma_commit(smem_addr(&bars->kv_empty[v_slot]));
                    if (more) {
                        if (t == 0) {
                            ok = bounded_wait(smem_addr(&bars->kv_full[k_slot]), uint32_t(uk / kStages) & 1u,
                                              abort_flag, p.timeout_ns, kSiteMma);
                            if (!ok) break;
                            tc_fence_after_sync();
                        }
                        issue_qk(tS[t], q_desc[t], k_desc0 + uint64_t(k_slot) * kSlotStep);
                        umma_commit(smem_addr(&bars->s_full[t]));
                        if (t == 1) umma_commit(smem_addr(&bars->kv_empty[k_slot]));
                    } else {
                        umma_commit(smem_addr(&bars->o_full[t]));
                    }
                }
            }
            } else {
            // Block-sparse: stream entry e belongs to one query tile.  After
            // that tile's P V on e comes its S on its next entry (two entries
            // on while both lists last, then the next one), so the two tiles
            // keep taking turns.  Barrier phases count each tile's own entries.
            // The stream's shape follows from the two list lengths alone:
            // entries [0, both2) alternate between the tiles,
            // the rest belong to the tile with the longer list.  Owner and
            // next entry are register arithmetic, no shared-memory reads.
            const int n0 = kv_list_len[1], n1 = kv_list_len[2];
            const int both2 = 2 * min(n0, n1);
            const int lt = n0 >= n1 ? 0 : 1;
            auto owner = [&](int e) -> int { return e < both2 ? (e & 1) : lt; };
            auto next_own = [&](int e) -> int {  // the owner's next entry after e, or -1
                if (e + 2 < both2) return e + 2;
                if (e < both2) return ((e & 1) == lt && both2 < n_kv) ? both2 : -1;
                return e + 1 < n_kv ? e + 1 : -1;
            };
            int done0 = 0, done1 = 0;  // P V products issued per tile (scalars: no local-memory array)
            // prologue: the scores of each tile's first entry (entries 0 and 1
            // while both tiles have entries)
            for (int e = 0; ok && e < 2 && e < n_kv; ++e) {
                if (e == 1 && both2 == 0) break;
                ok = bounded_wait(smem_addr(&bars->kv_full[(2 * e) % kStages]), 0, abort_flag, p.timeout_ns, kSiteMma);
                if (!ok) break;
                tc_fence_after_sync();
                const int t = owner(e);
                issue_qk(t ? tS[1] : tS[0], t ? q_desc[1] : q_desc[0], k_desc0 + uint64_t((2 * e) % kStages) * kSlotStep);
                umma_commit(smem_addr(&bars->s_full[t]));
                umma_commit(smem_addr(&bars->kv_empty[(2 * e) % kStages]));
            }
            for (int e = 0; ok && e < n_kv; ++e) {
                const int t = owner(e);
                const int uv = 2 * e + 1;
                const int v_slot = uv % kStages;
                ok = bounded_wait(smem_addr(&bars->kv_full[v_slot]), uint32_t(uv / kStages) & 1u, abort_flag,
                                  p.timeout_ns, kSiteMma);
                const int done_t = t ? done1 : done0;
                const uint32_t ph = uint32_t(done_t) & 1u;
                for (int hf = 0; ok && hf < 2; ++hf) {
                    ok = bounded_wait(smem_addr(&bars->p_full[t][hf]), ph, abort_flag, p.timeout_ns, kSiteMma);
                    if (ok) {
                        tc_fence_after_sync();
                        issue_pv_half(t ? tO[1] : tO[0], t ? tS[1] : tS[0], v_desc0 + uint64_t(v_slot) * kSlotStep, hf,
                                      done_t > 0);
                    }
                }
                if (!ok) break;
                umma_commit(smem_addr(&bars->kv_empty[v_slot]));
                if (t) ++done1; else ++done0;
                const int f = next_own(e);
                if (f < 0) {
                    umma_commit(smem_addr(&bars->o_full[t]));
                } else if (f > 1 || both2 == 0) {  // entries 0 and 1 of two tiles had theirs in the prologue
                    const int uk = 2 * f;
                    const int k_slot = uk % kStages;
                    ok = bounded_wait(smem_addr(&bars->kv_full[k_slot]), uint32_t(uk / kStages) & 1u, abort_flag,
                                      p.timeout_ns, kSiteMma);
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_qk(t ? tS[1] : tS[0], t ? q_desc[1] : q_desc[0], k_desc0 + uint64_t(k_slot) * kSlotStep);
                    umma_commit(smem_addr(&bars->s_full[t]));
                    umma_commit(smem_addr(&bars->kv_empty[k_slot]));
                }
            }
            }
            if (!ok) {
                // Let every MMA already issued finish before TMEM is released;
                // this wait ignores the abort flag but keeps its time limit.
                umma_commit(smem_addr(&bars->drain));
                const uint32_t drain = smem_addr(&bars->drain);
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax warpgroups
        setmaxnreg_inc<kSoftmaxRegs>();
        const int t = warp >> 2;        // query tile
        const int quarter = warp & 3;   // TMEM lane quarter this warp may access
        const int row_in_tile = quarter * 32 + lane;
        const int row = q0 + t * kBlockM + row_in_tile;
        const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_bits + uint32_t(t) * 128u;
        const uint32_t tO = tmem + lane_bits + 256u + uint32_t(t) * 128u;
        const uint32_t s_full = smem_addr(&bars->s_full[t]);

        int kv_lim = p.Skv;  // keys [0, kv_lim) are allowed for this row
        if (p.mask_kind == kMaskBlockCausal) {
            const long long lim = (static_cast<long long>(row / p.chunk) + 1) * p.chunk;
            kv_lim = static_cast<int>(min(static_cast<long long>(p.Skv), lim));
        }
        const float scale_log2 = p.scale_log2;
        const uint64_t scale2 = pack_f32x2(scale_log2, scale_log2);
        float m = -INFINITY;  // reference max (log2 units) the exponentials are taken against
        float l = 0.0f;       // running row sum at that reference
        bool ok = true;

        // key tiles this query tile takes part in: all n_kv, or its own block-sparse entries
        const int n_mine = kSparse ? kv_list_len[1 + t] : n_kv;
        for (int j = 0; j < n_mine; ++j) {
            const int idx = j;
            ok = warp_wait(s_full, uint32_t(idx) & 1u, abort_flag, p.timeout_ns, kSiteSoftmax);
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t s[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + uint32_t(c) * 32u, s[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(s[c]);

            // keys of this tile allowed for the row: [0, lim) of the tile
            int lim;
            if (sparse) {
                lim = p.Skv - int(kv_list[t * kMaxSparseKvBlocks + j]) * kBlockN;
            } else {
                lim = kv_lim - j * kBlockN;
            }
            if (lim < kBlockN) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i >= lim) s[c][i] = __float_as_uint(-INFINITY);
            }
            // Row max over the tile: eight independent 3-input max chains.
            auto tile_max = [&]() {
                float mxc[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint32_t* v = &s[g >> 1][(g & 1) * 16];
                    float a = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
                    for (int i = 2; i < 16; i += 2) a = fmax3(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                    mxc[g] = a;
                }
                return fmax3(fmax3(mxc[0], mxc[1], mxc[2]), fmax3(mxc[3], mxc[4], mxc[5]), fmaxf(mxc[6], mxc[7]));
            };
            uint64_t lsum[4] = {0, 0, 0, 0};
            uint32_t pa[2][16];  // packed P of keys 0-63, held until the reference max is settled
            if (idx == 0) {
                // first key tile: the reference max is the tile max
                m = tile_max() * scale_log2;
                const float m_use = (m == -INFINITY) ? 0.0f : m;
                const uint64_t negm2 = pack_f32x2(-m_use, -m_use);
                exp_chunk(s[0], scale2, negm2, pa[0], lsum);
                exp_chunk(s[1], scale2, negm2, pa[1], lsum);
            } else {
                // Exponentiate keys 0-63 against the current reference and
                // store them to TMEM at once (released only after the check);
                // the check needs no full tile max: a key of 0-63 exceeds the
                // reference by more than the threshold exactly when its
                // exponential exceeds 2^threshold, so their sum bounds it, and
                // keys 64-127 take a max over 64 values.
                const float m_use0 = (m == -INFINITY) ? 0.0f : m;
                const uint64_t negm2 = pack_f32x2(-m_use0, -m_use0);
                exp_chunk(s[0], scale2, negm2, pa[0], lsum);
                tmem_st16(tS, pa[0]);
                exp_chunk(s[1], scale2, negm2, pa[1], lsum);
                tmem_st16(tS + 16u, pa[1]);
                float sum0 = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    sum0 += __uint_as_float(uint32_t(lsum[q])) + __uint_as_float(uint32_t(lsum[q] >> 32));
                float mx[4];
#pragma unroll
                for (int g = 4; g < 8; ++g) {
                    const uint32_t* v = &s[g >> 1][(g & 1) * 16];
                    float a = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
                    for (int i = 2; i < 16; i += 2) a = fmax3(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                    mx[g - 4] = a;
                }
                const float m_hi = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
                const bool check = sum0 > 256.0f || m_hi > m + kRescaleThreshold;  // 256 = 2^threshold
                if (__any_sync(0xffffffffu, check)) {
                    const float m_tile = tile_max() * scale_log2;
                    const bool rescale = m_tile > m + kRescaleThreshold;
                    float alpha = 1.0f;
                    if (rescale) {
                        alpha = ex2_approx(m - m_tile);
                        m = m_tile;
                        l *= alpha;
                        // redo keys 0-63 against the new reference
                        const float m_use1 = m;
                        const uint64_t negm2b = pack_f32x2(-m_use1, -m_use1);
#pragma unroll
                        for (int q = 0; q < 4; ++q) lsum[q] = 0;
                        exp_chunk(s[0], scale2, negm2b, pa[0], lsum);
                        exp_chunk(s[1], scale2, negm2b, pa[1], lsum);
                    }
                    // the (possibly redone) keys 0-63 over the speculative store
                    tmem_st_wait();
                    tmem_st16(tS, pa[0]);
                    tmem_st16(tS + 16u, pa[1]);
                    // O_t holds sum_k P_k V_k at the old reference: bring it to
                    // the new one before any of this tile's P is released.
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + uint32_t(c) * 32u, o);
                        tmem_ld_wait(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tO + uint32_t(c) * 32u, o);
                    }
                }
            }
            // release keys 0-63 (stored above, or here for the first tile),
            // then exponentiate and release keys 64-127
            if (idx == 0) {
                tmem_st16(tS, pa[0]);
                tmem_st16(tS + 16u, pa[1]);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[t][0]));
            {
                const float m_use = (m == -INFINITY) ? 0.0f : m;
                const uint64_t negm2 = pack_f32x2(-m_use, -m_use);
#pragma unroll
                for (int c = 2; c < 4; ++c) {
                    uint32_t pk[16];
                    exp_chunk(s[c], scale2, negm2, pk, lsum);
                    tmem_st16(tS + uint32_t(c) * 16u, pk);
                }
            }
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[t][1]));
            {
                float part = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    part += __uint_as_float(uint32_t(lsum[q])) + __uint_as_float(uint32_t(lsum[q] >> 32));
                l += part;
            }
        }

        // With no key tile for this query tile (nothing it attends to in a
        // block-sparse mask) O stays 0 and LSE = -inf; nothing was issued for
        // it, so there is nothing to wait for.
        if (ok && n_mine > 0) ok = warp_wait(smem_addr(&bars->o_full[t]), 0, abort_flag, p.timeout_ns, kSiteSoftmax);
        if (ok) {
            tc_fence_after_sync();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            if constexpr (!kSparse) {
                // O leaves through shared memory.  Every product that read
                // ring slot (2 n_kv - 2) mod 4 (the last K tile) completed
                // before tile 0's last P V, and slot (2 n_kv - 3) mod 4 (the
                // V tile before the last) before tile 1's, and no load is in
                // flight any more: tile 0 stages its 128 rows in the first,
                // tile 1 in the second.  Each thread writes its row (256
                // bytes) into its warp's 8 KB as two 128B-swizzled 32-row x
                // 64-dim boxes, and one lane stores both with TMA instead of
                // 32 rows of 16-byte pieces per store instruction.
                const int slot = (t == 0 ? 2 * n_kv - 2 : 2 * n_kv - 3) & (kStages - 1);
                uint8_t* stage = smem + kSmemKV + slot * kTileBytes + quarter * kStageWarpBytes;
                const uint32_t stage_addr = smem_addr(stage);
                uint8_t* my_row = stage + lane * 128;
                const uint32_t swz = uint32_t(lane & 7) << 4;  // 128-byte swizzle: 16-byte chunk ^= row % 8
#pragma unroll 1
                for (int c = 0; c < kHeadDim / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + uint32_t(c) * 32u, o);
                    tmem_ld_wait(o);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                    // dims 32c .. 32c+31: box c / 2, 16-byte chunks 4 (c % 2) + i of the row
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(my_row + (c >> 1) * (kStageWarpBytes / 2) +
                                                  ((uint32_t((4 * (c & 1) + i) << 4)) ^ swz)) =
                            make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                const int warp_row0 = q0 + t * kBlockM + quarter * kStageRows;
                if (lane == 0 && warp_row0 < p.Sq) {
                    tma_store_4d(&tm_o, stage_addr, 0, h, warp_row0, b);
                    tma_store_4d(&tm_o, stage_addr + kStageWarpBytes / 2, kStageCols, h, warp_row0, b);
                    bulk_commit_group();
                }
            } else {
            __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Sq + row) * p.H + h) * kHeadDim;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                if (n_mine > 0) {
                    tmem_ld32(tO + uint32_t(c) * 32u, o);
                    tmem_ld_wait(o);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                if (row < p.Sq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            }
            if (p.lse != nullptr && row < p.Sq) {
                const float m_use = (m == -INFINITY) ? 0.0f : m;
                p.lse[(static_cast<size_t>(b) * p.H + h) * p.Sq + row] =
                    (m_use + __log2f(l)) * 0.69314718055994531f;
            }
        }
    }

    // ------------------------------------------------ teardown
    if (!kSparse && warp < 8 && lane == 0) bulk_wait_all();  // the epilogue's stores are complete
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace vdit
