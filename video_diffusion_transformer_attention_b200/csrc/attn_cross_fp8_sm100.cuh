// attn_cross_fp8_sm100.cuh -- the 8-bit attention forward (E4M3 Q and K,
// V-Smooth residuals, ExpCast-FP8 probabilities; attn_fwd_fp8_sm100.cuh) for
// a short key sequence: the cross-attention of the video tokens to a few
// hundred text tokens.
//
// The arithmetic per key tile is that of the 8-bit kernel: S = Q8 K8^T in
// TMEM, each probability's E4M3 byte from one FMA against the row's lazily
// raised reference, the row sum as packed fp16 adds, O += P8 Vt8 with P from
// TMEM, and the V-Smooth restore as one kind::f16 product into the same
// accumulator.  Only the schedule differs, as the bf16 cross kernel differs
// from the bf16 full kernel (attn_cross_sm100.cuh): with 512 text keys a
// query tile meets four key tiles, and a CTA that owns two query tiles and
// all 512 TMEM columns spends most of its life in its prologue and epilogue.
// Here a work item is one 128-row query tile and the kernel is persistent,
// two CTAs per SM (256 TMEM columns and 86 KB of shared memory each), each
// taking items c, c + gridDim.x, ...; the next item's Q codes load as soon as
// the current item's last S has read Q, and the other CTA on the SM keeps
// the tensor core busy while this one is in its epilogue.  The epilogue
// writes O through a 32 KB staging buffer with TMA stores of 32-row boxes.
//
// Roles (192 threads): warps 0-3 softmax and epilogue of the query tile,
// warp 4 TMA producer (an item's Q codes, then K_j codes into slot 0 and
// Vt_j codes plus its restore tile into slot 1), warp 5 TMEM allocator and
// single-thread tcgen05.mma issuer.
//
// TMEM (256 columns): S [0, 128), O [128, 256); the bytes of P take columns
// [0, 32) of S and the restore operand columns [32, 40).  Issue order per key
// tile j: P V_j [two 64-key halves], the restore product, then S_(j+1).
//
// Every pipeline wait is bounded, as in the other kernels.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "attn_cross_sm100.cuh"
#include "attn_fwd_fp8_sm100.cuh"

namespace vdit {

struct __align__(8) F8CrossBarriers {
    uint64_t q_full;
    uint64_t q_empty;     // the item's last S has read Q
    uint64_t kv_full[2];  // slot 0: K_j codes, slot 1: Vt_j codes + restore tile
    uint64_t kv_empty[2];
    uint64_t s_full;
    uint64_t p_full[2];   // P keys 0-63 / 64-127 (and the restore operand with the second) in TMEM
    uint64_t o_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kF8CrossSmemQ = 0;
constexpr int kF8CrossSmemKV = kF8TileBytes;                           // slot 0 K, slot 1 Vt (16 KB each)
constexpr int kF8CrossSmemMu = kF8CrossSmemKV + 2 * kF8TileBytes;      // the Vt slot's 4 KB restore tile
constexpr int kF8CrossSmemStage = kF8CrossSmemMu + kF8MuBytes;         // O staging: 8 KB per softmax warp
constexpr int kF8CrossSmemBar = kF8CrossSmemStage + 4 * kCrossStageBytes;
constexpr int kF8CrossSmemBytes =
    kF8CrossSmemBar + ((int(sizeof(F8CrossBarriers)) + 15) / 16) * 16 + 1024;  // + alignment slack
static_assert(kF8CrossSmemMu % 1024 == 0 && kF8CrossSmemStage % 1024 == 0, "swizzled tiles need 1 KB alignment");

// Item i is query tile i % nqb of (batch, head) i / nqb.
__device__ __forceinline__ void f8_cross_item(const Fp8FwdParams& p, long long item, int& b, int& h, int& q0) {
    const long long bh = item / p.nqb;
    q0 = static_cast<int>(item - bh * p.nqb) * kBlockM;
    h = static_cast<int>(bh % p.H);
    b = static_cast<int>(bh / p.H);
}

// One work item's softmax for the warp's 32 rows over the item's key tiles,
// then its epilogue.  kt: key tiles of the CTA's earlier items (S and P
// barrier phases); qi: earlier items (O phase).  Returns false on a timeout.
template <bool kNarrow>
__device__ __forceinline__ bool f8_cross_rows(const Fp8FwdParams& p, F8CrossBarriers* bars, volatile int* abort_flag,
                                              int warp, int lane, int b, int h, int q0, uint32_t tS, uint32_t tO,
                                              int n_kv, float cq, uint32_t kt, uint32_t qi, uint8_t* stage,
                                              const CUtensorMap* tm_o) {
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const int row = q0 + warp * 32 + lane;
    const uint32_t s_full = smem_addr(&bars->s_full);
    float ref_n = 0.0f;  // reference = ref_n + 0.65 (code units); set by the first tile
    float l = 0.0f;      // running row sum in byte-value units at that reference
    bool ok = true;
    float sk_next = p.k_scale[bh * p.nkb];
    for (int j = 0; j < n_kv; ++j) {
        const float sk = sk_next;
        if (j + 1 < n_kv) sk_next = p.k_scale[bh * p.nkb + j + 1];
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
        const float a = cq * sk;
        const uint64_t a2 = pack_f32x2(a, a);
        auto zmax_of = [&](float smax) { return smax == -INFINITY ? -INFINITY : smax * a; };
        uint32_t acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        uint32_t pw[32];  // 128 bytes of P
        if (j == 0) {
            const float zmax = zmax_of(tile_max());
            ref_n = zmax == -INFINITY ? 0.0f : ceilf(zmax - kF8RefFrac);
            const float bc = kMagic + float(kF8CodeOffset) - ref_n;
            const uint64_t b2 = pack_f32x2(bc, bc);
            code_chunk<kNarrow>(s[0], a2, b2, pw, acc);
            code_chunk<kNarrow>(s[1], a2, b2, pw + 8, acc);
        } else {
            {
                const float bc = kMagic + float(kF8CodeOffset) - ref_n;
                const uint64_t b2 = pack_f32x2(bc, bc);
                code_chunk<kNarrow>(s[0], a2, b2, pw, acc);
                code_chunk<kNarrow>(s[1], a2, b2, pw + 8, acc);
            }
            const float zmax = zmax_of(tile_max());
            const bool rescale = zmax > ref_n + kF8RefFrac + kF8RescaleCodes;
            if (__any_sync(0xffffffffu, rescale)) {
                float alpha = 1.0f;
                if (rescale) {
                    const float new_n = ceilf(zmax - kF8RefFrac);
                    alpha = ex2_approx((ref_n - new_n) * 0.125f);
                    ref_n = new_n;
                    l *= alpha;
                    const float bc = kMagic + float(kF8CodeOffset) - ref_n;
                    const uint64_t b2 = pack_f32x2(bc, bc);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[q] = 0;
                    code_chunk<kNarrow>(s[0], a2, b2, pw, acc);
                    code_chunk<kNarrow>(s[1], a2, b2, pw + 8, acc);
                }
                // O holds the earlier tiles' products at the old reference (the
                // item's previous P V and restore completed before this S)
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
        // release keys 0-63
        tmem_st16(tS, pw);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[0]));
        {
            const float bc = kMagic + float(kF8CodeOffset) - ref_n;
            const uint64_t b2 = pack_f32x2(bc, bc);
            code_chunk<kNarrow>(s[2], a2, b2, pw + 16, acc);
            code_chunk<kNarrow>(s[3], a2, b2, pw + 24, acc);
        }
        // l_j in byte-value units, and the restore operand [l_hi, l_lo, l_hi, 0 ...] (bf16)
        float lj = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float2 f = f16x2_to_float2(acc[q]);
            lj += f.x + f.y;
        }
        lj *= 256.0f;
        l += lj;
        const __nv_bfloat16 l_hi = __float2bfloat16_rn(lj);
        const __nv_bfloat16 l_lo = __float2bfloat16_rn(lj - __bfloat162float(l_hi));
        const uint32_t hi_bits = uint32_t(__bfloat16_as_ushort(l_hi));
        uint32_t rop[8] = {hi_bits | (uint32_t(__bfloat16_as_ushort(l_lo)) << 16), hi_bits, 0, 0, 0, 0, 0, 0};
        tmem_st16(tS + 16u, pw + 16);
        tmem_st8(tS + 32u, rop);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[1]));
    }

    if (ok) ok = warp_wait(smem_addr(&bars->o_full), qi & 1u, abort_flag, p.timeout_ns, kSiteSoftmax);
    if (!ok) return false;
    tc_fence_after_sync();
    // O = v_scale[d] O / l leaves through the warp's 8 KB of staging as two
    // 128B-swizzled 32-row x 64-dim boxes, stored by one lane with TMA.  The
    // warp's boxes of the previous item must have left the buffer first.
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
    const float* vs = p.v_scale + bh * kHeadDim;
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
        for (int i = 0; i < 16; ++i) {
            const float2 sc = *reinterpret_cast<const float2*>(vs + c * 32 + 2 * i);
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * (sc.x * inv_l), __uint_as_float(o[2 * i + 1]) * (sc.y * inv_l));
        }
        // dims 32c .. 32c+31: box c / 2, 16-byte chunks 4 (c % 2) + i of the row
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(my_row + (c >> 1) * (kCrossStageBytes / 2) +
                                      ((uint32_t((4 * (c & 1) + i) << 4)) ^ swz)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    const int warp_row0 = q0 + warp * kCrossStageRows;
    if (lane == 0 && warp_row0 < p.Sq) {
        tma_store_4d(tm_o, stage_addr, 0, h, warp_row0, b);
        tma_store_4d(tm_o, stage_addr + kCrossStageBytes / 2, kCrossStageCols, h, warp_row0, b);
        bulk_commit_group();
    }
    if (p.lse != nullptr && row < p.Sq)
        p.lse[bh * p.Sq + row] = ((ref_n + kF8RefFrac) * 0.125f - kF8PShift + __log2f(l)) * 0.69314718055994531f;
    return true;
}

// tm_o: O (bf16) as a 4-D tensor with 64-dim x 32-row boxes, 128-byte
// swizzled, as in the bf16 cross kernel.
__global__ void __launch_bounds__(kCrossThreads, 2)
    attn_cross_fp8_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_o,
                                const Fp8FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    F8CrossBarriers* bars = reinterpret_cast<F8CrossBarriers*>(smem + kF8CrossSmemBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = int(threadIdx.x >> 5);
    const int lane = int(threadIdx.x & 31);
    const long long n_items = static_cast<long long>(p.nqb) * p.H * p.B;
    const int n_kv = p.nkb;

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
        mbar_init(smem_addr(&bars->drain), 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == kCrossLoadWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_vt);
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
    const uint32_t sQ = smem_addr(smem + kF8CrossSmemQ);
    const uint32_t sK = smem_addr(smem + kF8CrossSmemKV);
    const uint32_t sVt = sK + kF8TileBytes;
    const uint32_t sMu = smem_addr(smem + kF8CrossSmemMu);

    if (warp >= 4) {
        if (warp == kCrossLoadWarp && lane == 0) {
            // ------------------------------------------------ TMA producer
            griddep_wait();  // the codes come from the preprocessing kernels queued just before
            uint32_t kt = 0;  // key tiles loaded by earlier items
            uint32_t qi = 0;  // earlier items
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
                int b, h, q0;
                f8_cross_item(p, item, b, h, q0);
                const long long bh = static_cast<long long>(b) * p.H + h;
                if (item != blockIdx.x && !bounded_wait(smem_addr(&bars->q_empty), (qi - 1u) & 1u, abort_flag,
                                                        p.timeout_ns, kSiteProducer))
                    break;
                const uint32_t qbar = smem_addr(&bars->q_full);
                mbar_arrive_expect_tx(qbar, kF8TileBytes);
                tma_load_4d(sQ, &tm_q, qbar, 0, h, q0, b);
                for (int j = 0; ok && j < n_kv; ++j) {
                    const uint32_t ph = ((kt + uint32_t(j)) & 1u) ^ 1u;
                    if (!bounded_wait(smem_addr(&bars->kv_empty[0]), ph, abort_flag, p.timeout_ns, kSiteProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full0 = smem_addr(&bars->kv_full[0]);
                    mbar_arrive_expect_tx(full0, kF8TileBytes);
                    tma_load_4d(sK, &tm_k, full0, 0, h, j * kBlockN, b);
                    if (!bounded_wait(smem_addr(&bars->kv_empty[1]), ph, abort_flag, p.timeout_ns, kSiteProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full1 = smem_addr(&bars->kv_full[1]);
                    mbar_arrive_expect_tx(full1, kF8TileBytes + kF8MuBytes);
                    tma_load_3d(sVt, &tm_vt, full1, 0, 0, int(bh * p.nkb + j));
                    bulk_load(sMu, p.mu_img + (bh * p.nkb + j) * kF8MuBytes, kF8MuBytes, full1);
                }
                kt += uint32_t(n_kv);
            }
        } else if (warp == kCrossMmaWarp && lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t tS = tmem;
            const uint32_t tO = tmem + 128;
            const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t k_desc = smem_desc_sw128(sK, 16, 1024);
            const uint64_t vt_desc = smem_desc_sw128(sVt, 16, 1024);  // Vt codes, K-major
            const uint64_t mu_desc = smem_desc_sw128(sMu, 2048, 1024);  // restore tile, MN-major bf16
            constexpr uint32_t idesc_restore = make_idesc_bf16(true);
            uint32_t kt = 0;
            uint32_t qi = 0;
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
                ok = bounded_wait(smem_addr(&bars->q_full), qi & 1u, abort_flag, p.timeout_ns, kSiteMma) &&
                     bounded_wait(smem_addr(&bars->kv_full[0]), kt & 1u, abort_flag, p.timeout_ns, kSiteMma);
                if (!ok) break;
                tc_fence_after_sync();
                issue_qk_f8(tS, q_desc, k_desc);
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
                            issue_pv_f8_half(tO, tS, vt_desc, hf, j > 0);
                        }
                    }
                    if (!ok) break;
                    umma_ts(tO, tS + 32u, mu_desc, idesc_restore, 1u);  // O += l_j mu'_j (V-Smooth restore)
                    umma_commit(smem_addr(&bars->kv_empty[1]));
                    if (j + 1 < n_kv) {
                        ok = bounded_wait(smem_addr(&bars->kv_full[0]), ph ^ 1u, abort_flag, p.timeout_ns,
                                          kSiteMma);
                        if (!ok) break;
                        tc_fence_after_sync();
                        issue_qk_f8(tS, q_desc, k_desc);
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
        const uint32_t lane_bits = uint32_t(warp * 32) << 16;  // warp w may access TMEM lanes [32w, 32w + 32)
        const uint32_t tS = tmem + lane_bits;
        const uint32_t tO = tmem + lane_bits + 128u;
        uint8_t* stage = smem + kF8CrossSmemStage + warp * kCrossStageBytes;
        uint32_t kt = 0;
        uint32_t qi = 0;
        bool ok = true;
        for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++qi) {
            int b, h, q0;
            f8_cross_item(p, item, b, h, q0);
            const size_t bh = static_cast<size_t>(b) * p.H + h;
            const float cq = p.c0 * p.q_scale[bh * p.nqb + q0 / kBlockM];
            // the 16-bit clamp's bound, as in the 8-bit kernel: from the item's
            // Q scale and the head's largest K scale
            float sk_max = 0.0f;
            for (int i = lane; i < p.nkb; i += 32) sk_max = fmaxf(sk_max, p.k_scale[bh * p.nkb + i]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sk_max = fmaxf(sk_max, __shfl_xor_sync(0xffffffffu, sk_max, off));
            const bool narrow = 2.0f * cq * sk_max * kF8MaxScoreCodes + 2.0f < 32000.0f;
            ok = narrow ? f8_cross_rows<true>(p, bars, abort_flag, warp, lane, b, h, q0, tS, tO, n_kv, cq, kt, qi,
                                              stage, &tm_o)
                        : f8_cross_rows<false>(p, bars, abort_flag, warp, lane, b, h, q0, tS, tO, n_kv, cq, kt, qi,
                                               stage, &tm_o);
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
