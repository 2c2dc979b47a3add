// qk_norm.cuh -- per-head RMS norm of the query and key tensors, one launch
// for both.
//
// For every (b, s, h) row x of D = 128 bf16 values of Q (weight w = w_q) and
// of K (w = w_k):
//   y[d] = x[d] * rsqrt(mean_d(x^2) + eps) * w[h][d]      (fp32, rounded to bf16)
// This is the query/key normalisation of the Wan2.x blocks (the model the
// gonka DiT-support discussion #1155 proposes to serve); its "Pricing policy"
// section counts normalisation among the parts of a forward pass whose cost
// grows linearly with the number of latent patches.
//
// HBM-bound: 256 B read and 256 B written per row.  Running it inside the
// attention kernel instead would repeat the K rows' norm once per 256-query
// block (every CTA streams every K tile), so it runs once here, ahead of the
// attention, which is launched as its programmatic dependent: the norm grid
// lets it start early and the attention's TMA producer waits for the norm
// grid to finish before its first load.
//
// 16 lanes own one row (16 bytes = 8 values each), so a warp covers two rows
// per pass with 512 contiguous bytes; the sum of squares is reduced by
// shuffles inside each 16-lane half.  Each half-warp keeps 4 rows in flight.
// Output rows may be the input rows (in place): every 16-byte chunk is read
// and written by the same thread.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace vdit {

constexpr int kNormThreads = 256;
constexpr int kNormMinBlocks = 4;     // 1024 threads an SM: 32 warps x 4 row pairs of loads in flight
constexpr int kNormRowsInFlight = 4;  // per half-warp
constexpr int kNormHeadDim = 128;

struct NormTensor {
    const uint4* x;   // [rows][16] chunks of 8 bf16
    uint4* y;         // same layout; may equal x
    const float* w;   // [H][128] fp32, or nullptr for weight 1
    long long rows;   // B * S * H
};

__device__ __forceinline__ void norm_chunk(uint4& c, float rs, const float* w_row, int sub) {
    __nv_bfloat162* x = reinterpret_cast<__nv_bfloat162*>(&c);
    float wv[8];
    if (w_row != nullptr) {
        const float4 w0 = *reinterpret_cast<const float4*>(w_row + sub * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(w_row + sub * 8 + 4);
        wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
        wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) wv[e] = 1.0f;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(x[e]);
        x[e] = __floats2bfloat162_rn(f.x * rs * wv[2 * e], f.y * rs * wv[2 * e + 1]);
    }
}

__device__ __forceinline__ float sum_squares(const uint4& c) {
    const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&c);
    float ss = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(x[e]);
        ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
    return ss;
}

// Rows 0 .. a.rows-1 are tensor a's, the next b.rows are tensor b's.  A grid
// of at most one wave strides over them, kNormRowsInFlight row pairs per warp
// and pass.
__global__ void __launch_bounds__(kNormThreads, kNormMinBlocks)
    qk_rms_norm_kernel(const NormTensor a, const NormTensor b, int H, float eps) {
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int sub = lane & 15;   // which 16-byte chunk of the row
    const int half = lane >> 4;  // which of the pass's two rows
    const long long total = a.rows + b.rows;
    const long long warp = (static_cast<long long>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * kNormThreads) >> 5;
    constexpr int kRowsPerPass = 2 * kNormRowsInFlight;
    for (long long base = warp * kRowsPerPass; base < total; base += n_warps * kRowsPerPass) {
        uint4 c[kNormRowsInFlight];
        float ss[kNormRowsInFlight];
#pragma unroll
        for (int u = 0; u < kNormRowsInFlight; ++u) {
            const long long r = base + 2 * u + half;
            c[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < a.rows)
                c[u] = __ldcs(a.x + r * 16 + sub);
            else if (r < total)
                c[u] = __ldcs(b.x + (r - a.rows) * 16 + sub);
        }
#pragma unroll
        for (int u = 0; u < kNormRowsInFlight; ++u) {
            ss[u] = sum_squares(c[u]);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
        }
#pragma unroll
        for (int u = 0; u < kNormRowsInFlight; ++u) {
            const long long r = base + 2 * u + half;
            if (r >= total) continue;
            const float rs = rsqrtf(ss[u] * (1.0f / kNormHeadDim) + eps);
            const bool in_a = r < a.rows;
            const long long rr = in_a ? r : r - a.rows;
            const NormTensor& t = in_a ? a : b;
            const int h = static_cast<int>(rr % H);
            norm_chunk(c[u], rs, t.w != nullptr ? t.w + static_cast<long long>(h) * kNormHeadDim : nullptr, sub);
            t.y[rr * 16 + sub] = c[u];
        }
    }
}

}  // namespace vdit
