// fp8_quant.cuh -- preprocessing of the 8-bit attention path: E4M3 codes of
// Q and K per 128-token block, and V-Smooth for V.
//
// "VC-Attention: revolution in video generation speed without retraining"
// (aikraft.ru), section 02 "V-Smooth": per hardware block of 128 tokens the
// mean of V is subtracted ("Demean") and only the residual is quantised per
// channel to E4M3; the mean goes back in through the softmax row sum
// ("Restore").  Section 04: the preprocessing is fused into few kernels.
//
// Workspace contents written here (byte offsets from Fp8Layout):
//   q8, k8    E4M3 codes, [B][S][H][128], the layout of Q and K
//   vt8       E4M3 residual codes of V, per block transposed:
//             [B][H][nkb][128 channels][128 tokens] (the K-major B operand of P.V)
//   mu_img    per block, the 4 KB shared-memory image of the restore operand:
//             a 16 x 128 bf16 tile, MN-major, 128B-swizzled, two 64-channel
//             halves of 16 rows x 128 B; rows 0, 1, 2 hold mu'_hi, mu'_hi,
//             mu'_lo (mu' = block mean in units of the channel scale), the
//             other rows are zero
//   q_scale, k_scale   fp32 [B][H][nb]: amax / 448 per block
//   v_scale   fp32 [B][H][128]: per channel of a head, amax / 448
//   v_amax_r, v_amax_mu  uint32 [B][H][128]: running maxima (fp32 bits) of
//             |residual| and |block mean| over the head's blocks; zeroed by
//             the host before v_stats_kernel
//   mu        fp32 [B][H][nkb][128]: block means
//
// Every quantity that decides a stored code is computed with the same fp32
// operations in the same order as the test oracle: amax exactly, the
// quotients 448 / amax and amax / 448 with IEEE division, products rounded
// to fp32, the block mean as a sequential fp32 sum divided by the token
// count, and the E4M3 conversion rounding to nearest even with saturation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace vdit {

constexpr int kQuantBlock = 128;          // tokens per block
constexpr float kE4M3Max = 448.0f;
constexpr float kMuFloor = 1.0f / 256.0f;  // channel amax >= 2^-8 x max |block mean|
constexpr int kMuImgBytes = 4096;

struct Fp8Tensors {
    uint8_t* q8;
    uint8_t* k8;
    uint8_t* vt8;
    uint8_t* mu_img;
    float* q_scale;
    float* k_scale;
    float* v_scale;
    uint32_t* v_amax_r;
    uint32_t* v_amax_mu;
    float* mu;
};

// Two fp32 values -> two E4M3 codes (low byte = a), nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    return uint32_t(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

constexpr int kQuantThreads = 256;

// One CTA (256 threads) per (tensor, b, h, block).  Warp w holds tokens
// 16w .. 16w+15 of the block; lane l holds channels 4l .. 4l+3 of each, so
// every load and store instruction of a warp covers one whole token row.
__global__ void __launch_bounds__(kQuantThreads, 3)
    qk_quant_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, Fp8Tensors t,
                    int B, int H, int Sq, int Skv) {
    constexpr int kWarps = kQuantThreads / 32;
    constexpr int kTokPerWarp = kQuantBlock / kWarps;
    __shared__ float warp_max[kWarps];
    const int nqb = (Sq + kQuantBlock - 1) / kQuantBlock;
    const int nkb = (Skv + kQuantBlock - 1) / kQuantBlock;
    long long id = blockIdx.x;
    const long long n_q = static_cast<long long>(B) * H * nqb;
    const bool is_k = id >= n_q;
    if (is_k) id -= n_q;
    const int nb = is_k ? nkb : nqb;
    const int S = is_k ? Skv : Sq;
    const int blk = static_cast<int>(id % nb);
    const int h = static_cast<int>((id / nb) % H);
    const int b = static_cast<int>(id / (static_cast<long long>(nb) * H));
    const __nv_bfloat16* src = is_k ? k : q;
    uint8_t* dst = is_k ? t.k8 : t.q8;
    float* scale_out = is_k ? t.k_scale : t.q_scale;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tok0 = blk * kQuantBlock + warp * kTokPerWarp;
    const size_t row_stride = static_cast<size_t>(H) * 128;  // elements between tokens
    const size_t first = ((static_cast<size_t>(b) * S + tok0) * H + h) * 128 + lane * 4;
    const int n_here = min(kTokPerWarp, S - tok0);
    uint2 x[kTokPerWarp];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
        x[i] = make_uint2(0u, 0u);
        if (i < n_here) x[i] = __ldcs(reinterpret_cast<const uint2*>(src + first + i * row_stride));
    }
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
        const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&x[i]);
        const float2 f0 = __bfloat1622float2(v[0]), f1 = __bfloat1622float2(v[1]);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) warp_max[warp] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, warp_max[w]);
    const float inv = amax > 0.0f ? kE4M3Max / amax : 0.0f;
    if (threadIdx.x == 0) scale_out[(static_cast<size_t>(b) * H + h) * nb + blk] = amax / kE4M3Max;
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
        if (i >= n_here) break;
        const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&x[i]);
        const float2 f0 = __bfloat1622float2(v[0]), f1 = __bfloat1622float2(v[1]);
        const uint32_t c = e4m3x2(f0.x * inv, f0.y * inv) | (e4m3x2(f1.x * inv, f1.y * inv) << 16);
        *reinterpret_cast<uint32_t*>(dst + first + i * row_stride) = c;
    }
}

// Stage one (b, h) block of V ([128 tokens][128 channels] bf16, 32 KB) in
// shared memory with whole-row loads (warp w loads tokens w, w+8, ...; lane l
// loads channels 4l .. 4l+3); rows past Skv are zero.
__device__ __forceinline__ void stage_v_block(const __nv_bfloat16* __restrict__ v, __nv_bfloat16* tile, int b, int h,
                                              int H, int Skv, int t0, int n) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kRows = kQuantBlock / (kQuantThreads / 32);  // rows per warp, all loads in flight at once
    uint2 x[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = warp + r * (kQuantThreads / 32);
        x[r] = make_uint2(0u, 0u);
        if (i < n) x[r] = __ldcs(reinterpret_cast<const uint2*>(v + ((static_cast<size_t>(b) * Skv + t0 + i) * H + h) * 128) + lane);
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) reinterpret_cast<uint2*>(tile + (warp + r * (kQuantThreads / 32)) * 128)[lane] = x[r];
}

// One CTA (256 threads) per (b, h, block); after staging, thread d < 128
// takes the block mean of channel d (a sequential fp32 sum over the block's
// tokens, then / n: one dependent chain per channel, in token order), and
// both halves of the CTA then take the largest |v - mean| of channel d over
// tokens 0-63 and 64-127 (a max, exact in any order), combined through shared
// memory.  Thread d < 128 then updates the running per-channel maxima over
// the head's blocks (atomicMax on the bits of non-negative floats, which
// order like the floats).
__global__ void __launch_bounds__(kQuantThreads)
    v_stats_kernel(const __nv_bfloat16* __restrict__ v, Fp8Tensors t, int B, int H, int Skv) {
    __shared__ __align__(16) __nv_bfloat16 tile[kQuantBlock * 128];
    __shared__ float mu_s[128], rmax_s[128];
    const int nkb = (Skv + kQuantBlock - 1) / kQuantBlock;
    const int blk = blockIdx.x % nkb;
    const int h = (blockIdx.x / nkb) % H;
    const int b = blockIdx.x / (nkb * H);
    const int t0 = blk * kQuantBlock;
    const int n = min(kQuantBlock, Skv - t0);
    stage_v_block(v, tile, b, h, H, Skv, t0, n);
    __syncthreads();
    const int d = threadIdx.x & 127;
    const int half = threadIdx.x >> 7;
    if (half == 0) {
        float sum = 0.0f;
        if (n == kQuantBlock) {
#pragma unroll 16
            for (int i = 0; i < kQuantBlock; ++i) sum += __bfloat162float(tile[i * 128 + d]);
        } else {
            for (int i = 0; i < n; ++i) sum += __bfloat162float(tile[i * 128 + d]);
        }
        mu_s[d] = sum / static_cast<float>(n);
    }
    __syncthreads();
    const float mu = mu_s[d];
    const int i1 = min(n, (half + 1) * (kQuantBlock / 2));
    float rmax = 0.0f;
#pragma unroll 8
    for (int i = half * (kQuantBlock / 2); i < i1; ++i)
        rmax = fmaxf(rmax, fabsf(__bfloat162float(tile[i * 128 + d]) - mu));
    if (half == 1) rmax_s[d] = rmax;
    __syncthreads();
    if (half == 0) {
        rmax = fmaxf(rmax, rmax_s[d]);
        const size_t bh = static_cast<size_t>(b) * H + h;
        t.mu[(bh * nkb + blk) * 128 + d] = mu;
        atomicMax(t.v_amax_r + bh * 128 + d, __float_as_uint(rmax));
        atomicMax(t.v_amax_mu + bh * 128 + d, __float_as_uint(fabsf(mu)));
    }
}

// One CTA (256 threads) per (b, h, block).  After staging, threads d and
// d + 128 compute the residual codes E4M3((v - mean) * 448 / amax_d) of
// channel d, four 16-token groups each, into a transposed shared-memory tile
// ([channel][token] bytes), which the whole CTA then writes out as
// contiguous 16-byte rows; the block's restore tile (rows 3-15 zero as
// 16-byte stores, rows 0-2 one bf16 per thread) is written in between.
__global__ void __launch_bounds__(kQuantThreads)
    v_quant_kernel(const __nv_bfloat16* __restrict__ v, Fp8Tensors t, int B, int H, int Skv) {
    __shared__ __align__(16) __nv_bfloat16 tile[kQuantBlock * 128];
    __shared__ __align__(16) uint8_t codes[128 * kQuantBlock];
    const int nkb = (Skv + kQuantBlock - 1) / kQuantBlock;
    const int blk = blockIdx.x % nkb;
    const int h = (blockIdx.x / nkb) % H;
    const int b = blockIdx.x / (nkb * H);
    const int t0 = blk * kQuantBlock;
    const int n = min(kQuantBlock, Skv - t0);
    const size_t bh = static_cast<size_t>(b) * H + h;
    stage_v_block(v, tile, b, h, H, Skv, t0, n);
    __syncthreads();
    uint8_t* img = t.mu_img + (bh * nkb + blk) * kMuImgBytes;
    const int d = threadIdx.x & 127;
    const float amax = fmaxf(__uint_as_float(t.v_amax_r[bh * 128 + d]),
                             __uint_as_float(t.v_amax_mu[bh * 128 + d]) * kMuFloor);
    const float inv = amax > 0.0f ? kE4M3Max / amax : 0.0f;
    const float mu = t.mu[(bh * nkb + blk) * 128 + d];
    const int hsel = threadIdx.x >> 7;
    if (hsel == 0 && blk == 0) t.v_scale[bh * 128 + d] = amax / kE4M3Max;
    {
        // 16 tokens per 16-byte word; half hsel takes the words of parity
        // hsel, rotated by the channel so that a warp's 16-byte stores spread
        // over the banks
#pragma unroll 1
        for (int gi = 0; gi < 4; ++gi) {
            const int g = (2 * (gi + (d >> 2)) + hsel) & 7;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float r[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = g * 16 + e * 4 + u;
                    r[u] = i < n ? (__bfloat162float(tile[i * 128 + d]) - mu) * inv : 0.0f;
                }
                w[e] = e4m3x2(r[0], r[1]) | (e4m3x2(r[2], r[3]) << 16);
            }
            reinterpret_cast<uint4*>(codes + d * kQuantBlock)[g] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    // zero rows 3-15 of both halves: 2 x 13 rows x 8 chunks of 16 bytes
    for (int i = threadIdx.x; i < 2 * 13 * 8; i += kQuantThreads) {
        const int half = i / (13 * 8), r = 3 + (i / 8) % 13, ch = i % 8;
        *reinterpret_cast<uint4*>(img + half * 2048 + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
    }
    if (hsel == 1) {
        // Restore tile: element (row k, channel d) of half d / 64 at
        // k * 128 + ((c / 8) ^ (k & 7)) * 16 + (c % 8) * 2, c = d % 64.
        const float mu_p = mu * inv;
        const __nv_bfloat16 hi = __float2bfloat16_rn(mu_p);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mu_p - __bfloat162float(hi));
        const int half = d >> 6, c = d & 63;
        const __nv_bfloat16 rows[3] = {hi, hi, lo};
#pragma unroll
        for (int kr = 0; kr < 3; ++kr)
            *reinterpret_cast<__nv_bfloat16*>(img + half * 2048 + kr * 128 + (((c >> 3) ^ kr) << 4) + (c & 7) * 2) =
                rows[kr];
    }
    __syncthreads();
    uint4* out = reinterpret_cast<uint4*>(t.vt8 + (bh * nkb + blk) * 128 * kQuantBlock);
    for (int i = threadIdx.x; i < 128 * kQuantBlock / 16; i += kQuantThreads) out[i] = reinterpret_cast<const uint4*>(codes)[i];
}

}  // namespace vdit
