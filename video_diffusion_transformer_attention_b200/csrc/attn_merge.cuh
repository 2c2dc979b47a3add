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
// handling 4 of the 128 head dims (8-byte accesses, 256 B per row), with the
// weights broadcast by shuffle.  Per row it reads two O rows and two LSE
// values and writes one of each.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace vdit {

constexpr int kMergeWarpsPerBlock = 8;
constexpr int kMergeRowsPerWarp = 32;

__global__ void __launch_bounds__(kMergeWarpsPerBlock * 32)
    attn_merge_kernel(__nv_bfloat16* __restrict__ o_acc, float* __restrict__ lse_acc,
                      const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part, int B, int H,
                      int S) {
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
        uint2 a[4], p[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (r0 + u < n) {
                const size_t off = (row0 * 128) + (r0 + u) * stride + lane * 4;
                a[u] = *reinterpret_cast<const uint2*>(o_acc + off);
                p[u] = __ldg(reinterpret_cast<const uint2*>(o_part + off));
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float ra = __shfl_sync(0xffffffffu, wa, (r0 + u) & 31);
            const float rp = __shfl_sync(0xffffffffu, wp, (r0 + u) & 31);
            if (r0 + u < n) {
                const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&p[u]);
                uint2 out;
                __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float2 fa = __bfloat1622float2(a2[k]);
                    const float2 fp = __bfloat1622float2(p2[k]);
                    o2[k] = __floats2bfloat162_rn(ra * fa.x + rp * fp.x, ra * fa.y + rp * fp.y);
                }
                *reinterpret_cast<uint2*>(o_acc + (row0 * 128) + (r0 + u) * stride + lane * 4) = out;
            }
        }
    }
}

}  // namespace vdit
