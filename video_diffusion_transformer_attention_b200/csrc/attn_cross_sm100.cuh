// attn_cross_sm100.cuh -- bf16 attention forward for a short key sequence:
// the cross-attention of the video tokens to a few hundred text tokens.
//
// The arithmetic is that of attn_fwd_sm100.cuh (S = Q K^T in TMEM, online
// softmax with exp2 in registers, O += P V with P from TMEM); only the
// schedule differs.  The full kernel gives a CTA two query tiles that take
// turns with the tensor core, and holds all 512 TMEM columns and 198 KB of
// shared memory, so one CTA fits on an SM.  With 512 text keys a query tile
// meets only four key tiles, and such a CTA spends most of its life in its
// prologue (barrier and TMEM setup, the Q load from HBM, the first product
// before any softmax can start) and epilogue, with nothing to overlap them.
// Here a work item is one 128-row query tile, and the kernel is persistent:
// two CTAs per SM (256 TMEM columns for S and O, 97 KB of shared memory for Q
// and a two-slot K/V ring, each), each taking items c, c + gridDim.x, ...
// The next item's Q loads as soon as the current item's last S has read Q,
// so a CTA's item switch costs no HBM round trip, and the other CTA on the SM
// fills the tensor core and MUFU while this one is in its epilogue.  The
// epilogue stages O in the V slot (free once the item's last P V is done) and
// writes it with TMA stores of 32-row boxes, not with per-thread row stores
// that touch 32 rows per instruction; the producer loads the next item's first
// V only after those stores have read the slot.
//
// Roles (192 threads):
//   warps 0-3   softmax, correction and epilogue of the query tile
//   warp  4     TMA producer: an item's Q, then K_j into slot 0 and V_j into slot 1
//   warp  5     TMEM allocator and single-thread tcgen05.mma issuer
// Two CTAs of 192 threads leave at most 168 registers a thread, which the
// softmax warps use without spilling.  Registers are not re-split with
// setmaxnreg: it acts on whole warpgroups, and warps 4-5 are only half of one.
//
// TMEM (256 columns x 128 lanes): S [0,128), O [128,256); P (bf16, two per
// column) overwrites the first 64 columns of S.  Issue order per key tile j:
// P V_j [two 64-key halves], then S_(j+1) = Q K_(j+1)^T; the tensor core runs a
// thread's MMAs in order, so S_(j+1) overwrites P only after P V_j read it.
//
// Every pipeline wait is bounded, as in the full kernel: on a timeout the
// CTA raises its abort flag, ORs a code into the device status word, and
// every role leaves its loop so the CTA still reaches teardown.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace vdit {

constexpr int kCrossThreads = 192;
constexpr int kCrossLoadWarp = 4;
constexpr int kCrossMmaWarp = 5;
constexpr uint32_t kCrossTmemCols = 256;

struct __align__(8) CrossBarriers {
    uint64_t q_full;
    uint64_t q_empty;      // the item's last S has read Q
    uint64_t kv_full[2];   // slot 0: K_j, slot 1: V_j
    uint64_t kv_empty[2];
    uint64_t s_full;
    uint64_t p_full[2];    // P keys 0-63 / 64-127 in TMEM
    uint64_t o_full;
    uint64_t stage_free;   // the epilogue's TMA stores have read the V slot it staged O in
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kCrossStageRows = 32;  // epilogue: one warp's rows, staged in the V slot
constexpr int kCrossStageCols = 64;  // head dims per TMA store box (128 bytes of a bf16 row, 128B-swizzled)
constexpr int kCrossStageBytes = kCrossStageRows * kHeadDim * 2;  // 8 KB per softmax warp: two boxes

constexpr int kCrossSmemQ = 0;
constexpr int kCrossSmemKV = kTileBytes;
constexpr int kCrossSmemBar = kCrossSmemKV + 2 * kTileBytes;
constexpr int kCrossSmemBytes = kCrossSmemBar + ((int(sizeof(CrossBarriers)) + 15) / 16) * 16 + 1024;  // + alignment

// Item i is query tile i % n_qb of (batch, head) i / n_qb: the CTAs running at
// one time share one head's text K/V in L2.
__device__ __forceinline__ void cross_item(const FwdParams& p, long long item, int& b, int& h, int& q0) {
    const long long bh = item / p.n_qb;
    q0 = static_cast<int>(item - bh * p.n_qb) * kBlockM;
    h = static_cast<int>(bh % p.H);
    b = static_cast<int>(bh / p.H);
}

// Test-only residency record: when `spans` is non-null, CTA c < max_ctas
// writes spans[3c] = its SM id, spans[3c+1] / spans[3c+2] = the global timer
// (ns) when its producer starts and finishes.  Null in every product call.
struct CrossSpans {
    unsigned long long* spans;
    int max_ctas;
};

// tm_o: O as the same 4-D tensor as Q, with 64-dim x 32-row boxes, 128-byte
// swizzled: the epilogue's TMA store unit.
__global__ void __launch_bounds__(kCrossThreads, 2)
    attn_cross_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                            const FwdParams p, const CrossSpans rec) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    CrossBarriers* bars = reinterpret_cast<CrossBarriers*>(smem + kCrossSmemBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = int(threadIdx.x >> 5);
    const int lane = int(threadIdx.x & 31);
    const long long n_items = static_cast<long long>(p.n_qb) * p.H * p.B;
    const int n_kv = (p.Skv + kBlockN - 1) / kBlockN;

    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bars->q_full), 1);
        mbar_init(smem_addr(&bars->q_empty), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&bars->kv_full[s]), 1);
            mbar_init(smem_addr(&bars->kv_empty[s]), 1);
            mbar_init(smem_addr(&bars->p_full[s]), 4);  // one elected arrive per softmax warp
        }
        mbar_init(smem_addr(&bars->s_full), 1);
        mbar_init(smem_addr(&bars->o_full), 1);
        mbar_init(smem_addr(&bars->stage_free), 4);  // one elected arrive per softmax warp
        mbar_init(smem_addr(&bars->drain), 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == kCrossLoadWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    if (warp == kCrossMmaWarp) {
        tmem_alloc(smem_addr(&bars->tmem_base), kCrossTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t sQ = smem_addr(smem + kCrossSmemQ);
    const uint32_t sKV = smem_addr(smem + kCrossSmemKV);

    if (warp >= 4) {
        if (warp == kCrossLoadWarp && lane == 0) {
            // ------------------------------------------------ TMA producer
            griddep_wait();  // Q/K written by a preceding kernel (fused Q/K norm) are complete
            // test-only: the SM this CTA runs on and its producer's lifetime
            unsigned long long* span = (rec.spans != nullptr && int(blockIdx.x) < rec.max_ctas)
                                           ? rec.spans + 3 * size_t(blockIdx.x)
                                           : nullptr;
            if (span != nullptr) {
                uint32_t smid;
                asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
                span[0] = smid;
                span[1] = global_timer_ns();
            }
            uint32_t kt = 0;  // key tiles loaded by earlier items: each used slot 0 (K) and slot 1 (V) once
            uint32_t qi = 0;  // earlier items (only the parities of these counters matter)
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
                int b, h, q0;
                cross_item(p, item, b, h, q0);
                if (item != blockIdx.x && !bounded_wait(smem_addr(&bars->q_empty), (qi - 1u) & 1u, abort_flag,
                                            p.timeout_ns, kSiteProducer)) {
                    ok = false;
                    break;
                }
                const uint32_t qbar = smem_addr(&bars->q_full);
                mbar_arrive_expect_tx(qbar, kTileBytes);
                tma_load_4d(sQ, &tm_q, qbar, 0, h, q0, b);
                tma_load_4d(sQ + kHalfBytes, &tm_q, qbar, 64, h, q0, b);
                if (p.debug_flags & kDebugWithholdKV) break;  // test-only: the issuer's wait on K_0 runs out
                for (int j = 0; ok && j < n_kv; ++j) {
                    for (int slot = 0; slot < 2; ++slot) {  // K_j, then V_j
                        if (!bounded_wait(smem_addr(&bars->kv_empty[slot]), ((kt + uint32_t(j)) & 1u) ^ 1u,
                                          abort_flag, p.timeout_ns, kSiteProducer)) {
                            ok = false;
                            break;
                        }
                        // the previous item's epilogue staged O in the V slot
                        if (slot == 1 && j == 0 && qi > 0 &&
                            !bounded_wait(smem_addr(&bars->stage_free), (qi - 1u) & 1u, abort_flag, p.timeout_ns,
                                          kSiteProducer)) {
                            ok = false;
                            break;
                        }
                        const uint32_t full = smem_addr(&bars->kv_full[slot]);
                        const CUtensorMap* map = slot ? &tm_v : &tm_k;
                        mbar_arrive_expect_tx(full, kTileBytes);
                        tma_load_4d(sKV + slot * kTileBytes, map, full, 0, h, j * kBlockN, b);
                        tma_load_4d(sKV + slot * kTileBytes + kHalfBytes, map, full, 64, h, j * kBlockN, b);
                    }
                }
                kt += uint32_t(n_kv);
            }
            if (span != nullptr) span[2] = global_timer_ns();
        } else if (warp == kCrossMmaWarp && lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t tS = tmem;
            const uint32_t tO = tmem + 128;
            const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t k_desc = smem_desc_sw128(sKV, 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(sKV + kTileBytes, kHalfBytes, 1024);
            uint32_t kt = 0;  // key tiles of earlier items (K/V, S and P barrier phases)
            uint32_t qi = 0;  // earlier items (Q and O barrier phases)
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
                ok = bounded_wait(smem_addr(&bars->q_full), qi & 1u, abort_flag, p.timeout_ns, kSiteMma) &&
                     bounded_wait(smem_addr(&bars->kv_full[0]), kt & 1u, abort_flag, p.timeout_ns,
                                  kSiteMma);
                if (!ok) break;
                tc_fence_after_sync();
                issue_qk(tS, q_desc, k_desc);
                umma_commit(smem_addr(&bars->s_full));
                if (n_kv == 1) umma_commit(smem_addr(&bars->q_empty));
                umma_commit(smem_addr(&bars->kv_empty[0]));
                for (int j = 0; ok && j < n_kv; ++j) {
                    const uint32_t ph = (kt + uint32_t(j)) & 1u;
                    ok = bounded_wait(smem_addr(&bars->kv_full[1]), ph, abort_flag, p.timeout_ns, kSiteMma);
                    for (int hf = 0; ok && hf < 2; ++hf) {
                        ok = bounded_wait(smem_addr(&bars->p_full[hf]), ph, abort_flag, p.timeout_ns, kSiteMma);
                        if (ok) {
                            tc_fence_after_sync();
                            issue_pv_half(tO, tS, v_desc, hf, j > 0);
                        }
                    }
                    if (!ok) break;
                    umma_commit(smem_addr(&bars->kv_empty[1]));
                    if (j + 1 < n_kv) {
                        ok = bounded_wait(smem_addr(&bars->kv_full[0]), ph ^ 1u, abort_flag, p.timeout_ns,
                                          kSiteMma);
                        if (!ok) break;
                        tc_fence_after_sync();
                        issue_qk(tS, q_desc, k_desc);
                        umma_commit(smem_addr(&bars->s_full));
                        if (j + 2 == n_kv) umma_commit(smem_addr(&bars->q_empty));  // the item's last read of Q
                        umma_commit(smem_addr(&bars->kv_empty[0]));
                    } else {
                        umma_commit(smem_addr(&bars->o_full));
                    }
                }
                kt += uint32_t(n_kv);
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
        // ------------------------------------------------ softmax warpgroup
        const int row_in_tile = warp * 32 + lane;  // warp w may access TMEM lanes [32w, 32w + 32)
        const uint32_t lane_bits = uint32_t(warp * 32) << 16;
        const uint32_t tS = tmem + lane_bits;
        const uint32_t tO = tmem + lane_bits + 128u;
        const uint32_t s_full = smem_addr(&bars->s_full);
        const float scale_log2 = p.scale_log2;
        const uint64_t scale2 = pack_f32x2(scale_log2, scale_log2);
        bool ok = true;
        uint32_t kt = 0;  // key tiles of earlier items (S phases)
        uint32_t qi = 0;  // earlier items (O phases)

        for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
            float m = -INFINITY;  // reference max (log2 units) the exponentials are taken against
            float l = 0.0f;       // running row sum at that reference
            for (int j = 0; j < n_kv; ++j) {
                ok = warp_wait(s_full, (kt + uint32_t(j)) & 1u, abort_flag, p.timeout_ns, kSiteSoftmax);
                if (!ok) break;
                tc_fence_after_sync();
                uint32_t s[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + uint32_t(c) * 32u, s[c]);
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_wait(s[c]);

                const int lim = p.Skv - j * kBlockN;  // keys [0, lim) of this tile exist
                if (lim < kBlockN) {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c * 32 + i >= lim) s[c][i] = __float_as_uint(-INFINITY);
                }
                // row max over the tile: eight independent 3-input max chains
                float mxc[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint32_t* v = &s[g >> 1][(g & 1) * 16];
                    float a = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
                    for (int i = 2; i < 16; i += 2) a = fmax3(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                    mxc[g] = a;
                }
                const float m_tile =
                    fmax3(fmax3(mxc[0], mxc[1], mxc[2]), fmax3(mxc[3], mxc[4], mxc[5]), fmaxf(mxc[6], mxc[7])) *
                    scale_log2;
                bool rescale_o = false;  // warp-uniform: some row of this warp moves its reference
                float alpha = 1.0f;
                if (j == 0) {
                    m = m_tile;  // every row has at least one key in the first tile
                } else {
                    // Lazy rescaling: the reference moves only when the max grew past
                    // the threshold; O (the earlier P V at the old reference) is then
                    // scaled below, before any of this tile's P is released.
                    const bool rescale = m_tile > m + kRescaleThreshold;
                    rescale_o = __any_sync(0xffffffffu, rescale);
                    if (rescale) {
                        alpha = ex2_approx(m - m_tile);
                        m = m_tile;
                        l *= alpha;
                    }
                }
                const uint64_t negm2 = pack_f32x2(-m, -m);
                uint64_t lsum[4] = {0, 0, 0, 0};
                // keys 0-63, released first so P V can start on them
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
                    exp_chunk(s[c], scale2, negm2, pk, lsum);
                    tmem_st16(tS + uint32_t(c) * 16u, pk);
                }
                if (rescale_o) {
                    // after keys 0-63, whose scores are no longer held in registers
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
                tmem_st_wait();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[0]));
                // keys 64-127
#pragma unroll
                for (int c = 2; c < 4; ++c) {
                    uint32_t pk[16];
                    exp_chunk(s[c], scale2, negm2, pk, lsum);
                    tmem_st16(tS + uint32_t(c) * 16u, pk);
                }
                tmem_st_wait();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[1]));
                float part = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    part += __uint_as_float(uint32_t(lsum[q])) + __uint_as_float(uint32_t(lsum[q] >> 32));
                l += part;
            }

            if (ok) ok = warp_wait(smem_addr(&bars->o_full), qi & 1u, abort_flag, p.timeout_ns, kSiteSoftmax);
            if (ok) {
                tc_fence_after_sync();
                int b, h, q0;
                cross_item(p, item, b, h, q0);
                const int row = q0 + row_in_tile;
                const int warp_row0 = q0 + warp * kCrossStageRows;  // first row of this warp's TMA boxes
                const float inv_l = 1.0f / l;  // l >= 1: the row's maximum key contributes 2^0
                // O leaves through shared memory: each thread writes its row
                // (256 bytes) into the warp's 8 KB of the V slot -- free once
                // the item's last P V has completed -- as two 128B-swizzled
                // 32-row x 64-dim boxes, and one lane stores both with TMA
                // instead of 32 rows of 16-byte pieces per store instruction.
                uint8_t* stage = smem + kCrossSmemKV + kTileBytes + warp * kCrossStageBytes;
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
                        *reinterpret_cast<uint4*>(my_row + (c >> 1) * (kCrossStageBytes / 2) +
                                                  ((uint32_t((4 * (c & 1) + i) << 4)) ^ swz)) =
                            make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (warp_row0 < p.Sq) {
                        tma_store_4d(&tm_o, stage_addr, 0, h, warp_row0, b);
                        tma_store_4d(&tm_o, stage_addr + kCrossStageBytes / 2, kCrossStageCols, h, warp_row0, b);
                        bulk_commit_group();
                        bulk_wait_read_all();  // the boxes have left shared memory
                    }
                    mbar_arrive(smem_addr(&bars->stage_free));
                }
                if (p.lse != nullptr && row < p.Sq)
                    p.lse[(static_cast<size_t>(b) * p.H + h) * p.Sq + row] = (m + __log2f(l)) * 0.69314718055994531f;
            }
            kt += uint32_t(n_kv);
        }
    }

    // ------------------------------------------------ teardown
    if (warp < 4 && lane == 0) bulk_wait_all();  // the epilogue's stores are complete
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kCrossMmaWarp) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, kCrossTmemCols);
    }
}

}  // namespace vdit
