// attn_merge.cuh -- merge of two partial attention results over disjoint key
// sets, through their log-sum-exp.
//
// For one query row, if O_a, LSE_a are attention over key set A and O_b,
// LSE_b over a disjoint set B, then over A u B
//   LSE = ln(e^LSE_a + e^LSE_b),   O = e^(LSE_a - LSE) O_a + e^(LSE_b - LSE) O_b.
// This is what passing K/V blocks around a ring of GPUs needs (the ring
// context parallelism of the Wave Forcing digest (airadar.tv), which compares
// Wave Parallelism with Ulysses and Ring context parallelism): each step
// attends to one K/V block and folds the partial result into the running one.
// An empty partial (LSE = -inf) leaves the other unchanged.
//
// HBM-bound.  A warp takes 32 consecutive query rows i of one (b, h): each
// lane reads the two LSE values of one row (coalesced) and computes that
// row's merge weights once, then the warp walks the 32 rows, every lane
// handling 4 of the 128 head dims (256 B per bf16 row, 512 B per fp32 row),
// with the weights broadcast by shuffle.  Per row it reads two O rows and two
// LSE values and writes one of each (plus the bf16 output row, if asked).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace vdit {

constexpr int kMergeWarpsPerBlock = 8;
constexpr int kMergeRowsPerWarp = 32;

// Four consecutive head dims of a running O row, as floats: bf16 (8 bytes) or
// fp32 (16 bytes) storage.
__device__ __forceinline__ void merge_load4(const __nv_bfloat16* p, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
__device__ __forceinline__ void merge_load4(const float* p, float (&x)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
}
__device__ __forceinline__ void merge_store4(__nv_bfloat16* p, const float (&x)[4]) {
    uint2 u;
    *reinterpret_cast<__nv_bfloat162*>(&u.x) = __floats2bfloat162_rn(x[0], x[1]);
    *reinterpret_cast<__nv_bfloat162*>(&u.y) = __floats2bfloat162_rn(x[2], x[3]);
    *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void merge_store4(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

// AccT: the running O's storage, bf16 or fp32.  An fp32 running O keeps a
// ring of N partial results from being rounded to bf16 N - 1 times; o_out,
// when not null, also receives the merged O rounded once to bf16 (the last
// fold of a ring writes the final output this way).
template <typename AccT>
__global__ void __launch_bounds__(kMergeWarpsPerBlock * 32)
    attn_merge_kernel(AccT* __restrict__ o_acc, float* __restrict__ lse_acc,
                      const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part,
                      __nv_bfloat16* __restrict__ o_out, int B, int H, int S) {
    const int lane = threadIdx.x & 31;
    const long long chunks = (S + kMergeRowsPerWarp - 1) / kMergeRowsPerWarp;
    const long long wid = static_cast<long long>(blockIdx.x) * kMergeWarpsPerBlock + (threadIdx.x >> 5);
    if (wid >= static_cast<long long>(B) * H * chunks) return;
    const long long bh = wid / chunks;  // b * H + h
    const int i0 = static_cast<int>(wid - bh * chunks) * kMergeRowsPerWarp;
    const int b = static_cast<int>(bh / H);
    const int h = static_cast<int>(bh - static_cast<long long>(b) * H);
    const int n = min(kMergeRowsPerWarp, S - i0);

    // lane l: weights of row i0 + l
    float wa = 0.0f, wp = 0.0f;
    if (lane < n) {
        const long long li = bh * S + i0 + lane;
        const float la = lse_acc[li];
        const float lp = lse_part[li];
        const float mx = fmaxf(la, lp);
        float lse = -INFINITY;
        if (mx != -INFINITY) {
            const float ea = expf(la - mx);
            const float ep = expf(lp - mx);
            const float inv = 1.0f / (ea + ep);
            wa = ea * inv;
            wp = ep * inv;
            lse = mx + logf(ea + ep);
        }
        lse_acc[li] = lse;
    }
    // O row (b, i, h) at ((b * S + i) * H + h) * 128
    const size_t row0 = (static_cast<size_t>(b) * S + i0) * H + h;
    const size_t stride = static_cast<size_t>(H) * 128;
    for (int r0 = 0; r0 < n; r0 += 4) {
        float a[4][4], p[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (r0 + u < n) {
                const size_t off = (row0 * 128) + (r0 + u) * stride + lane * 4;
                merge_load4(o_acc + off, a[u]);
                merge_load4(o_part + off, p[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float ra = __shfl_sync(0xffffffffu, wa, (r0 + u) & 31);
            const float rp = __shfl_sync(0xffffffffu, wp, (r0 + u) & 31);
            if (r0 + u < n) {
                float m[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) m[k] = ra * a[u][k] + rp * p[u][k];
                const size_t off = (row0 * 128) + (r0 + u) * stride + lane * 4;
                merge_store4(o_acc + off, m);
                if (o_out != nullptr) merge_store4(o_out + off, m);
            }
        }
    }
}

}  // namespace vdit
