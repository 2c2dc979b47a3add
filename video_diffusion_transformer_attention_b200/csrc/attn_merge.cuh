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
// HBM-bound: one warp per (b, i, h) row, each lane 4 of the 128 head dims
// (8-byte loads and stores, coalesced 256 B per warp); per row it reads two
// O rows and two LSE values and writes one of each.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace vdit {

constexpr int kMergeWarpsPerBlock = 8;

__global__ void __launch_bounds__(kMergeWarpsPerBlock * 32)
    attn_merge_kernel(__nv_bfloat16* __restrict__ o_acc, float* __restrict__ lse_acc,
                      const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part, int B, int H,
                      int S) {
    const long long rows = static_cast<long long>(B) * S * H;
    const long long r = static_cast<long long>(blockIdx.x) * kMergeWarpsPerBlock + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    // O row r = (b * S + i) * H + h; LSE index (b * H + h) * S + i
    const long long bs = r / H;
    const int h = static_cast<int>(r - bs * H);
    const long long b = bs / S;
    const int i = static_cast<int>(bs - b * S);
    const long long li = (b * H + h) * S + i;
    const float la = lse_acc[li];
    const float lp = lse_part[li];
    const float mx = fmaxf(la, lp);
    float wa = 0.0f, wp = 0.0f, lse = -INFINITY;
    if (mx != -INFINITY) {
        const float ea = expf(la - mx);
        const float ep = expf(lp - mx);
        const float sum = ea + ep;
        wa = ea / sum;
        wp = ep / sum;
        lse = mx + logf(sum);
    }
    const size_t off = static_cast<size_t>(r) * 128 + lane * 4;
    const uint2 a = *reinterpret_cast<const uint2*>(o_acc + off);
    const uint2 p = *reinterpret_cast<const uint2*>(o_part + off);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&p);
    uint2 out;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float2 fa = __bfloat1622float2(a2[k]);
        const float2 fp = __bfloat1622float2(p2[k]);
        o2[k] = __floats2bfloat162_rn(wa * fa.x + wp * fp.x, wa * fa.y + wp * fp.y);
    }
    *reinterpret_cast<uint2*>(o_acc + off) = out;
    if (lane == 0) lse_acc[li] = lse;
}

}  // namespace vdit
