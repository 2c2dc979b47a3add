// attn_fwd_fp8_sm100.cuh -- the 8-bit attention forward for sm_100a:
// E4M3 Q, K and V-Smooth residuals on the tensor cores, ExpCast-FP8
// probabilities written straight from the log-domain scores.
//
// "VC-Attention: revolution in video generation speed without retraining"
// (aikraft.ru): section 01 -- on B200 the fp32 exp + cast between the two
// matrix products is the longest stage; section 02 -- V-Smooth (block mean
// removed before quantisation, restored through the softmax row sum);
// section 03 -- ExpCast-FP8: an E4M3 byte read as an integer is about
// 8 log2(v) + 56, so one FMA from the log-domain score writes the byte
// (beta = -0.35 centres the error), with no exponential at all.
//
// Per CTA: two 128-row query tiles of one (b, h), key tiles j of 128:
//   S_t  = Q8_t K8_j^T                    tcgen05 kind::f8f6f4, fp32 in TMEM
//   z    = S * A_j,  A_j = 8 log2(e) scale sq_t sk_j       (code units)
//   byte = rint(z - ref + 95.65), clamped at 0: one packed FMA into a float
//          whose low bits are the integer (the "magic number" 1.5 * 2^23 plus
//          an integer addend, since ref is kept on the grid N + 0.65), a max,
//          and byte permutes.  The bytes are p * 2^5 in E4M3.
//   l_j  = sum of the bytes' values: a byte y shifted left by 7 is exactly
//          the fp16 encoding of value(y) * 2^-8, so the row sum is packed
//          fp16 adds, no decoding table and no exponential.
//   O_t += P8_t Vt8_j                     kind::f8f6f4, P from TMEM
//   O_t += [l_hi l_lo l_hi] [mu'_hi; mu'_hi; mu'_lo]   kind::f16, one K = 16
//          step: the V-Smooth restore, l_j times the block mean (in units of
//          the channel scale), accumulated in the same TMEM tile
//   O    = v_scale[d] * O_t / l,  LSE = ln2 (ref/8 - 5 + log2 l)
//
// The reference max ref (code units) is set from the first tile and raised
// only when a tile's max exceeds it by more than 24 codes (3 in log2), so
// the largest byte is rint(24 + 95.65) = 120 < 126 (448 is byte 126).
//
// Roles, barriers, bounded waits and the TMEM plan follow the bf16 kernel
// (attn_fwd_sm100.cuh): warps 0-7 softmax (tile = warp / 4), warp 8 TMA
// producer, warp 9 MMA issuer.  Shared memory: Q (2 x 16 KB), an 8-slot ring
// of 16 KB tiles (K_j in even slots, Vt_j in odd), and one 4 KB restore tile
// per odd slot.  TMEM: S_0, S_1, O_0, O_1 as in the bf16 kernel; the bytes of
// P_t take columns [0, 32) of S_t and the restore operand columns [32, 40).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd_sm100.cuh"
#include "sm100_fp8_ptx.cuh"

namespace vdit {

constexpr int kF8Stages = 8;
constexpr int kF8TileBytes = kBlockM * kHeadDim;  // 16 KB of E4M3
constexpr int kF8MuBytes = 4096;
constexpr int kF8SmemQ = 0;
constexpr int kF8SmemKV = kQTiles * kF8TileBytes;
constexpr int kF8SmemMu = kF8SmemKV + kF8Stages * kF8TileBytes;
constexpr int kF8SmemBar = kF8SmemMu + (kF8Stages / 2) * kF8MuBytes;
constexpr float kF8RescaleCodes = 24.0f;   // 3 in log2 units
constexpr float kF8RefFrac = 0.65f;        // the reference sits on N + 0.65
constexpr int kF8CodeOffset = 95;          // 8*5 + 56 - 0.35 = 95.65 = 95 + 0.65
constexpr float kF8PShift = 5.0f;          // bytes are p * 2^5
constexpr float kMagic = 12582912.0f;      // 1.5 * 2^23: integers in the low mantissa bits

struct __align__(8) Fp8Barriers {
    uint64_t q_full[kQTiles];
    uint64_t kv_full[kF8Stages];
    uint64_t kv_empty[kF8Stages];
    uint64_t s_full[kQTiles];
    uint64_t p_full[kQTiles][2];
    uint64_t o_full[kQTiles];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
constexpr int kF8SmemBytes = kF8SmemBar + ((int(sizeof(Fp8Barriers)) + 15) / 16) * 16 + 1024;

struct Fp8FwdParams {
    int B, H, Sq, Skv;
    int mask_kind;
    int chunk;
    float c0;                 // 8 * log2(e) * scale
    const float* q_scale;     // [B][H][nqb]
    const float* k_scale;     // [B][H][nkb]
    const float* v_scale;     // [B][H][128]
    const uint8_t* mu_img;    // [B][H][nkb][4096]
    int nqb, nkb;
    __nv_bfloat16* o;
    float* lse;
    unsigned long long timeout_ns;
};

// kind::f8f6f4, E4M3 x E4M3 -> fp32, both operands K-major, M = N = 128.
__host__ __device__ constexpr uint32_t make_idesc_e4m3() {
    return (1u << 4) | (uint32_t(kBlockN >> 3) << 17) | (uint32_t(kBlockM >> 4) << 24);
}

// S = Q8 K8^T: K = 128 head dims = 4 steps of 32 codes (32 bytes) inside the
// one 128-byte swizzled row.
__device__ __forceinline__ void issue_qk_f8(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
    constexpr uint32_t idesc = make_idesc_e4m3();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) umma_ss_f8(d_tmem, q_desc + uint64_t(kk * 2), k_desc + uint64_t(kk * 2), idesc, kk > 0);
}

// O (+)= P8 Vt8 over the 64 keys of `half`: P from TMEM (8 columns per 32
// keys), Vt K-major (channel rows, 128 token bytes each).
__device__ __forceinline__ void issue_pv_f8_half(uint32_t d_tmem, uint32_t p_tmem, uint64_t vt_desc, int half,
                                                 bool accumulate) {
    constexpr uint32_t idesc = make_idesc_e4m3();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int kk = half * 2 + i;
        umma_ts_f8(d_tmem, p_tmem + uint32_t(kk) * 8u, vt_desc + uint64_t(kk * 2), idesc,
                   (accumulate || kk > 0) ? 1u : 0u);
    }
}

// 32 scores -> 8 words of 4 ExpCast bytes, and the row-sum contribution in
// 8 packed-fp16 accumulators (value * 2^-8 per byte).
//
// The FMA leaves t = 1.5 * 2^23 + y, so the low 16 bits of t are y whenever
// -2^15 <= y < 2^15 (and 0 for t = -inf, a masked key).  kNarrow clamps y at 0
// on those 16-bit lanes, two per instruction; that is exact when every score
// of the row lies within 2^15 - 95 codes below the reference, which the caller
// checks from the scales.  Otherwise t itself is clamped at 1.5 * 2^23 first.
template <bool kNarrow>
__device__ __forceinline__ void code_chunk(const uint32_t (&s)[32], uint64_t a2, uint64_t b2, uint32_t* pw,
                                           uint32_t (&acc)[8]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float t0, t1, t2, t3;
        ffma2(__uint_as_float(s[4 * q]), __uint_as_float(s[4 * q + 1]), a2, b2, t0, t1);
        ffma2(__uint_as_float(s[4 * q + 2]), __uint_as_float(s[4 * q + 3]), a2, b2, t2, t3);
        uint32_t h01, h23;
        if (kNarrow) {
            h01 = max_s16x2(prmt(__float_as_uint(t0), __float_as_uint(t1), 0x5410u), 0u);
            h23 = max_s16x2(prmt(__float_as_uint(t2), __float_as_uint(t3), 0x5410u), 0u);
        } else {
            h01 = prmt(__float_as_uint(fmaxf(t0, kMagic)), __float_as_uint(fmaxf(t1, kMagic)), 0x5410u);
            h23 = prmt(__float_as_uint(fmaxf(t2, kMagic)), __float_as_uint(fmaxf(t3, kMagic)), 0x5410u);
        }
        pw[q] = prmt(h01, h23, 0x6420u);  // y0 y1 y2 y3  (h01 = y0 | y1 << 16)
        hadd2_acc(acc[q], h01 << 7);
        hadd2_acc(acc[q], h23 << 7);
    }
}

// Largest |code product sum| of one score: 128 head dims x 448 x 448.
constexpr float kF8MaxScoreCodes = 128.0f * 448.0f * 448.0f;

// One query tile's softmax loop (the warp's 32 rows) over all key tiles, then
// its epilogue.  Shared state lives in the kernel; see the kernel for roles.
template <bool kNarrow>
__device__ __forceinline__ void fp8_softmax_rows(const Fp8FwdParams& p, Fp8Barriers* bars, volatile int* abort_flag,
                                                 int t, int lane, int row, size_t bh, uint32_t tS, uint32_t tO,
                                                 int n_kv, int kv_lim, float cq) {
    const uint32_t s_full = smem_addr(&bars->s_full[t]);
    float ref_n = 0.0f;   // reference = ref_n + 0.65 (code units); set by the first tile
    float l = 0.0f;       // running row sum in byte-value units at that reference
    bool ok = true;
    float sk_next = n_kv > 0 ? p.k_scale[bh * p.nkb] : 0.0f;
    for (int j = 0; j < n_kv; ++j) {
        const float sk = sk_next;
        if (j + 1 < n_kv) sk_next = p.k_scale[bh * p.nkb + j + 1];  // hidden behind this tile
        ok = warp_wait(s_full, uint32_t(j) & 1u, abort_flag, p.timeout_ns, kSiteSoftmax);
        if (!ok) break;
        tc_fence_after_sync();
        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + uint32_t(c) * 32u, s[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(s[c]);
        const int lim = kv_lim - j * kBlockN;
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
        if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[t][0]));
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
        if (lane == 0) mbar_arrive(smem_addr(&bars->p_full[t][1]));
    }

    if (ok && n_kv > 0) ok = warp_wait(smem_addr(&bars->o_full[t]), 0, abort_flag, p.timeout_ns, kSiteSoftmax);
    if (ok) {
        tc_fence_after_sync();
        const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
        const float* vs = p.v_scale + bh * kHeadDim;
        const int b = int(bh / p.H), h = int(bh % p.H);
        __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Sq + row) * p.H + h) * kHeadDim;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + uint32_t(c) * 32u, o);
            tmem_ld_wait(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 sc = *reinterpret_cast<const float2*>(vs + c * 32 + 2 * i);
                pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * (sc.x * inv_l),
                                    __uint_as_float(o[2 * i + 1]) * (sc.y * inv_l));
            }
            if (row < p.Sq) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
        if (p.lse != nullptr && row < p.Sq)
            p.lse[bh * p.Sq + row] = ((ref_n + kF8RefFrac) * 0.125f - kF8PShift + __log2f(l)) * 0.69314718055994531f;
    }
}

// kLongFirst (block-causal): block x takes query-tile pair gridDim.x - 1 - x,
// so each head's CTAs with the most key tiles start first, as in the bf16
// kernel.
template <bool kLongFirst = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    attn_fwd_fp8_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_vt, const Fp8FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    Fp8Barriers* bars = reinterpret_cast<Fp8Barriers*>(smem + kF8SmemBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = int(threadIdx.x >> 5);
    const int lane = int(threadIdx.x & 31);
    const int h = int(blockIdx.y);
    const int b = int(blockIdx.z);
    const int q0 = (kLongFirst ? int(gridDim.x - 1u - blockIdx.x) : int(blockIdx.x)) * (kQTiles * kBlockM);
    const size_t bh = static_cast<size_t>(b) * p.H + h;

    if (threadIdx.x == 0) {
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(smem_addr(&bars->q_full[t]), 1);
            mbar_init(smem_addr(&bars->s_full[t]), 1);
            mbar_init(smem_addr(&bars->p_full[t][0]), 4);
            mbar_init(smem_addr(&bars->p_full[t][1]), 4);
            mbar_init(smem_addr(&bars->o_full[t]), 1);
        }
        for (int s = 0; s < kF8Stages; ++s) {
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
        tma_prefetch_desc(&tm_vt);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_addr(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    int kv_end = p.Skv;
    if (p.mask_kind == kMaskBlockCausal) {
        const int last_row = min(q0 + kQTiles * kBlockM - 1, p.Sq - 1);
        const long long lim = (static_cast<long long>(last_row / p.chunk) + 1) * p.chunk;
        kv_end = static_cast<int>(min(static_cast<long long>(p.Skv), lim));
    }
    const int n_kv = (kv_end + kBlockN - 1) / kBlockN;

    const uint32_t sQ = smem_addr(smem + kF8SmemQ);
    const uint32_t sKV = smem_addr(smem + kF8SmemKV);
    const uint32_t sMu = smem_addr(smem + kF8SmemMu);

    if (warp >= 8) {
        setmaxnreg_dec<kControlRegs>();
        if (warp == kLoadWarp && lane == 0) {
            // ------------------------------------------------ TMA producer
            griddep_wait();  // the codes come from the preprocessing kernels queued just before
            for (int t = 0; n_kv > 0 && t < kQTiles; ++t) {
                const uint32_t bar = smem_addr(&bars->q_full[t]);
                mbar_arrive_expect_tx(bar, kF8TileBytes);
                tma_load_4d(sQ + t * kF8TileBytes, &tm_q, bar, 0, h, q0 + t * kBlockM, b);
            }
            for (int u = 0; u < 2 * n_kv; ++u) {
                const int slot = u % kF8Stages;
                const uint32_t phase = uint32_t(u / kF8Stages) & 1u;
                if (!bounded_wait(smem_addr(&bars->kv_empty[slot]), phase ^ 1u, abort_flag, p.timeout_ns,
                                  kSiteProducer))
                    break;
                const uint32_t full = smem_addr(&bars->kv_full[slot]);
                const int j = u >> 1;
                if ((u & 1) == 0) {
                    mbar_arrive_expect_tx(full, kF8TileBytes);
                    tma_load_4d(sKV + slot * kF8TileBytes, &tm_k, full, 0, h, j * kBlockN, b);
                } else {
                    mbar_arrive_expect_tx(full, kF8TileBytes + kF8MuBytes);
                    tma_load_3d(sKV + slot * kF8TileBytes, &tm_vt, full, 0, 0, int(bh * p.nkb + j));
                    bulk_load(sMu + (slot >> 1) * kF8MuBytes, p.mu_img + (bh * p.nkb + j) * kF8MuBytes, kF8MuBytes,
                              full);
                }
            }
        } else if (warp == kMmaWarp && lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t tS[2] = {tmem, tmem + 128};
            const uint32_t tO[2] = {tmem + 256, tmem + 384};
            const uint64_t q_desc[2] = {smem_desc_sw128(sQ, 16, 1024), smem_desc_sw128(sQ + kF8TileBytes, 16, 1024)};
            const uint64_t kv_desc0 = smem_desc_sw128(sKV, 16, 1024);     // K tiles and Vt tiles, K-major
            const uint64_t mu_desc0 = smem_desc_sw128(sMu, 2048, 1024);   // restore tile, MN-major bf16
            constexpr uint64_t kSlotStep = kF8TileBytes >> 4;
            constexpr uint64_t kMuStep = kF8MuBytes >> 4;
            constexpr uint32_t idesc_restore = make_idesc_bf16(true);
            bool ok = n_kv > 0 &&
                      bounded_wait(smem_addr(&bars->q_full[0]), 0, abort_flag, p.timeout_ns, kSiteMma) &&
                      bounded_wait(smem_addr(&bars->q_full[1]), 0, abort_flag, p.timeout_ns, kSiteMma);
            if (ok) ok = bounded_wait(smem_addr(&bars->kv_full[0]), 0, abort_flag, p.timeout_ns, kSiteMma);
            if (ok) {
                tc_fence_after_sync();
                issue_qk_f8(tS[0], q_desc[0], kv_desc0);
                umma_commit(smem_addr(&bars->s_full[0]));
                issue_qk_f8(tS[1], q_desc[1], kv_desc0);
                umma_commit(smem_addr(&bars->s_full[1]));
                umma_commit(smem_addr(&bars->kv_empty[0]));
            }
            // per key tile j:  PV0(j) [two halves] R0(j) S0(j+1)  PV1(j) [two halves] R1(j) S1(j+1)
            for (int j = 0; ok && j < n_kv; ++j) {
                const int uv = 2 * j + 1;
                const int v_slot = uv % kF8Stages;
                const int uk = 2 * (j + 1);
                const int k_slot = uk % kF8Stages;
                const uint32_t ph = uint32_t(j) & 1u;
                const bool more = (j + 1) < n_kv;
                ok = bounded_wait(smem_addr(&bars->kv_full[v_slot]), uint32_t(uv / kF8Stages) & 1u, abort_flag,
                                  p.timeout_ns, kSiteMma);
                for (int t = 0; ok && t < kQTiles; ++t) {
                    for (int hf = 0; ok && hf < 2; ++hf) {
                        ok = bounded_wait(smem_addr(&bars->p_full[t][hf]), ph, abort_flag, p.timeout_ns, kSiteMma);
                        if (ok) {
                            tc_fence_after_sync();
                            issue_pv_f8_half(tO[t], tS[t], kv_desc0 + uint64_t(v_slot) * kSlotStep, hf, j > 0);
                        }
                    }
                    if (!ok) break;
                    umma_ts(tO[t], tS[t] + 32u, mu_desc0 + uint64_t(v_slot >> 1) * kMuStep, idesc_restore, 1u);
                    if (t == 1) umma_commit(smem_addr(&bars->kv_empty[v_slot]));
                    if (more) {
                        if (t == 0) {
                            ok = bounded_wait(smem_addr(&bars->kv_full[k_slot]), uint32_t(uk / kF8Stages) & 1u,
                                              abort_flag, p.timeout_ns, kSiteMma);
                            if (!ok) break;
                            tc_fence_after_sync();
                        }
                        issue_qk_f8(tS[t], q_desc[t], kv_desc0 + uint64_t(k_slot) * kSlotStep);
                        umma_commit(smem_addr(&bars->s_full[t]));
                        if (t == 1) umma_commit(smem_addr(&bars->kv_empty[k_slot]));
                    } else {
                        umma_commit(smem_addr(&bars->o_full[t]));
                    }
                }
            }
            if (!ok) {
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
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        const int row = q0 + t * kBlockM + row_in_tile;
        const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_bits + uint32_t(t) * 128u;
        const uint32_t tO = tmem + lane_bits + 256u + uint32_t(t) * 128u;

        int kv_lim = p.Skv;
        if (p.mask_kind == kMaskBlockCausal) {
            const long long lim = (static_cast<long long>(row / p.chunk) + 1) * p.chunk;
            kv_lim = static_cast<int>(min(static_cast<long long>(p.Skv), lim));
        }
        const int qblk = min(q0 / kBlockM + t, p.nqb - 1);
        const float cq = p.c0 * p.q_scale[bh * p.nqb + qblk];
        // The 16-bit clamp is exact when no score of a row lies more than
        // 2^15 - 95 codes below its reference; |score| <= cq * sk * 128 * 448^2,
        // so a span bound of twice the largest such value (plus one code of
        // reference rounding) below 32000 suffices.
        float sk_max = 0.0f;
        for (int i = lane; i < p.nkb; i += 32) sk_max = fmaxf(sk_max, p.k_scale[bh * p.nkb + i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sk_max = fmaxf(sk_max, __shfl_xor_sync(0xffffffffu, sk_max, off));
        const bool narrow = 2.0f * cq * sk_max * kF8MaxScoreCodes + 2.0f < 32000.0f;
        if (narrow)
            fp8_softmax_rows<true>(p, bars, abort_flag, t, lane, row, bh, tS, tO, n_kv, kv_lim, cq);
        else
            fp8_softmax_rows<false>(p, bars, abort_flag, t, lane, row, bh, tS, tO, n_kv, kv_lim, cq);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace vdit
