// vsmooth_group.cuh -- V-Smooth's "Group" step: online k-means over the value
// tokens of each (batch, head), and the joint permutation of K and V that
// puts each cluster's tokens next to each other.
//
// "VC-Attention: revolution in video generation speed without retraining"
// (aikraft.ru), section 02: value tokens are clustered per batch and head
// with an online k-means; keys and values are permuted together, which leaves
// non-causal attention unchanged, and the 128-token blocks of the permuted
// sequence then have block means that remove much more of V before
// quantisation.  Grouping runs on the first quarter of the denoising steps
// and a permutation is reused for four neighbouring steps, so the centroids
// are warm-started from the caller's (the previous step's).
//
// Lloyd iterations: assign every token to its nearest centroid (squared
// Euclidean distance, lowest index on ties), then move every centroid to the
// mean of its tokens (a centroid without tokens stays).  After the last
// iteration the tokens are assigned once more and stably sorted by cluster.
//
//   group_assign_kernel      one token per thread, its 128 values in registers,
//                            the centroids and their squared norms in shared
//                            memory; distance = |c|^2 - 2 v.c (|v|^2 is the
//                            same for every centroid)
//   group_accumulate_kernel  per 128-token block, thread d sums channel d of
//                            each cluster in shared memory, then adds the
//                            block's sums and counts to the head's with atomics
//   group_finalize_kernel    centroid = sum / count
//   group_sort_kernel        one CTA per head: cluster offsets from the counts,
//                            then 1024 tokens at a time, ranks within a warp by
//                            __match_any_sync and across warps by prefix counts
//                            -- a stable counting sort, so the permutation is
//                            unique given the labels
//   permute_rows_kernel      out[b, i, h, :] = in[b, perm[b, h, i], h, :]
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace vdit {

constexpr int kGroupMaxClusters = 64;
constexpr int kGroupTokens = 128;   // tokens per CTA in assign / accumulate
constexpr int kSortThreads = 1024;

__global__ void __launch_bounds__(kGroupTokens)
    group_assign_kernel(const __nv_bfloat16* __restrict__ v, const float* __restrict__ centroids,
                        int32_t* __restrict__ labels, int H, int S, int C) {
    __shared__ __align__(16) float cent[kGroupMaxClusters * 128];
    __shared__ float cnorm[kGroupMaxClusters];
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = static_cast<size_t>(b) * H + h;
    const float* cb = centroids + bh * C * 128;
    for (int i = threadIdx.x; i < C * 32; i += kGroupTokens)
        reinterpret_cast<float4*>(cent)[i] = reinterpret_cast<const float4*>(cb)[i];
    __syncthreads();
    if (threadIdx.x < C) {
        float s = 0.0f;
        for (int d = 0; d < 128; ++d) s = fmaf(cent[threadIdx.x * 128 + d], cent[threadIdx.x * 128 + d], s);
        cnorm[threadIdx.x] = s;
    }
    __syncthreads();
    const int t = blockIdx.x * kGroupTokens + threadIdx.x;
    if (t >= S) return;
    float x[128];
    const uint4* row = reinterpret_cast<const uint4*>(v + ((static_cast<size_t>(b) * S + t) * H + h) * 128);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint4 u = row[i];
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p[e]);
            x[i * 8 + 2 * e] = f.x;
            x[i * 8 + 2 * e + 1] = f.y;
        }
    }
    float best = INFINITY;
    int best_c = 0;
    for (int c = 0; c < C; ++c) {
        const float4* cc = reinterpret_cast<const float4*>(cent + c * 128);
        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float4 w = cc[i];
            a0 = fmaf(x[4 * i], w.x, a0);
            a1 = fmaf(x[4 * i + 1], w.y, a1);
            a2 = fmaf(x[4 * i + 2], w.z, a2);
            a3 = fmaf(x[4 * i + 3], w.w, a3);
        }
        const float dist = cnorm[c] - 2.0f * ((a0 + a1) + (a2 + a3));
        if (dist < best) {
            best = dist;
            best_c = c;
        }
    }
    labels[bh * S + t] = best_c;
}

// sums [B][H][C][128] and counts [B][H][C] must be zero before the launch.
__global__ void __launch_bounds__(128)
    group_accumulate_kernel(const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ labels,
                            float* __restrict__ sums, int32_t* __restrict__ counts, int H, int S, int C) {
    __shared__ float acc[kGroupMaxClusters * 128];
    __shared__ int cnt[kGroupMaxClusters];
    __shared__ int lab[kGroupTokens];
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = static_cast<size_t>(b) * H + h;
    const int d = threadIdx.x;
    const int t0 = blockIdx.x * kGroupTokens;
    const int n = min(kGroupTokens, S - t0);
    for (int c = 0; c < C; ++c) acc[c * 128 + d] = 0.0f;
    if (d < C) cnt[d] = 0;
    if (d < n) lab[d] = labels[bh * S + t0 + d];
    __syncthreads();
    if (d == 0)
        for (int i = 0; i < n; ++i) ++cnt[lab[i]];
    const __nv_bfloat16* col = v + ((static_cast<size_t>(b) * S + t0) * H + h) * 128 + d;
    const size_t stride = static_cast<size_t>(H) * 128;
#pragma unroll 8
    for (int i = 0; i < n; ++i) acc[lab[i] * 128 + d] += __bfloat162float(col[i * stride]);
    __syncthreads();
    for (int c = 0; c < C; ++c) {
        if (cnt[c] == 0) continue;
        atomicAdd(sums + (bh * C + c) * 128 + d, acc[c * 128 + d]);
        if (d == 0) atomicAdd(counts + bh * C + c, cnt[c]);
    }
}

__global__ void __launch_bounds__(128)
    group_finalize_kernel(const float* __restrict__ sums, const int32_t* __restrict__ counts,
                          float* __restrict__ centroids, int C) {
    const size_t bhc = blockIdx.x;  // (b * H + h) * C + c
    const int n = counts[bhc];
    if (n > 0) centroids[bhc * 128 + threadIdx.x] = sums[bhc * 128 + threadIdx.x] / static_cast<float>(n);
}

__global__ void __launch_bounds__(kSortThreads)
    group_sort_kernel(const int32_t* __restrict__ labels, int32_t* __restrict__ perm, int S, int C) {
    constexpr int kWarps = kSortThreads / 32;
    __shared__ int base[kGroupMaxClusters];            // next free position of each cluster
    __shared__ int total[kGroupMaxClusters];           // this chunk's tokens per cluster
    __shared__ int wpre[kWarps][kGroupMaxClusters];    // per warp: count, then exclusive prefix over warps
    const size_t bh = blockIdx.x;
    const int32_t* lab = labels + bh * S;
    int32_t* out = perm + bh * S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < C) base[threadIdx.x] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < S; t += kSortThreads) atomicAdd(&base[lab[t]], 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int c = 0; c < C; ++c) {
            const int k = base[c];
            base[c] = run;
            run += k;
        }
    }
    for (int t0 = 0; t0 < S; t0 += kSortThreads) {
        const int t = t0 + threadIdx.x;
        const int l = t < S ? lab[t] : -1;
        for (int i = threadIdx.x; i < kWarps * kGroupMaxClusters; i += kSortThreads) (&wpre[0][0])[i] = 0;
        __syncthreads();
        const unsigned peers = __match_any_sync(0xffffffffu, l);
        const int rank = __popc(peers & ((1u << lane) - 1u));   // earlier lanes of the same cluster
        if (l >= 0 && rank == 0) wpre[warp][l] = __popc(peers);
        __syncthreads();
        if (threadIdx.x < C) {
            int run = 0;
            for (int w = 0; w < kWarps; ++w) {
                const int k = wpre[w][threadIdx.x];
                wpre[w][threadIdx.x] = run;
                run += k;
            }
            total[threadIdx.x] = run;
        }
        __syncthreads();
        if (l >= 0) out[base[l] + wpre[warp][l] + rank] = t;
        __syncthreads();
        if (threadIdx.x < C) base[threadIdx.x] += total[threadIdx.x];
    }
}

// out[b, i, h, :] = in[b, perm[b, h, i], h, :] for K and V; 16 lanes per 256-byte row.
__global__ void __launch_bounds__(256)
    permute_rows_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ perm,
                        uint4* __restrict__ k_out, uint4* __restrict__ v_out, int H, int S, long long rows) {
    const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
    const int sub = threadIdx.x & 15;
    if (r >= rows) return;
    // r enumerates (b, h, i)
    const long long bh = r / S;
    const int i = static_cast<int>(r - bh * S);
    const int h = static_cast<int>(bh % H);
    const long long b = bh / H;
    const int src = perm[r];
    const size_t dst_off = ((static_cast<size_t>(b) * S + i) * H + h) * 16 + sub;
    const size_t src_off = ((static_cast<size_t>(b) * S + src) * H + h) * 16 + sub;
    k_out[dst_off] = k[src_off];
    v_out[dst_off] = v[src_off];
}

}  // namespace vdit
