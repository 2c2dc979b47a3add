/*
 * vdit_attn.h -- C ABI of the bf16 video-DiT attention forward library
 * (libvdit_attn.so, sm_100a / B200).
 *
 * The operation is the forward multi-head attention over the flattened
 * spatiotemporal latent tokens of a video diffusion transformer:
 *
 *   O[b,i,h,:] = sum_{j in A(i)} softmax_j(scale * q[b,i,h,:] . k[b,j,h,:]) v[b,j,h,:]
 *   LSE[b,h,i] = ln sum_{j in A(i)} exp(scale * q[b,i,h,:] . k[b,j,h,:])
 *
 * Sources for the operation:
 *  - "VC-Attention" (aikraft.ru), section 01 "Why attention became the
 *    bottleneck": the clip is flattened into one sequence of spatiotemporal
 *    tokens and full self-attention runs in every transformer layer; on B200
 *    the FP32 exp + cast between the two matrix products is the longest
 *    stage.
 *  - "Realtime video generation: FLOPS calculation and optimizations"
 *    (sudonull.com), FLOP list: self-attention (~82% of the layer at
 *    S = 75,600) and text->video cross-attention in each of the 40 layers;
 *    the FlashAttention bullet: no 75K x 75K score matrix is materialised.
 *  - Wave Forcing digest (airadar.tv), summary: block-causal attention in
 *    which later chunks read the K/V of earlier chunks.
 *
 * Conventions shared by every entry point:
 *  - Layout BSHD, contiguous: q and o are [B][Sq][H][D], k and v are
 *    [B][Skv][H][D], all bf16 (IEEE binary16 "brain" format, raw 2-byte
 *    elements).  lse is [B][H][Sq] fp32, natural log, unnormalised
 *    (LSE = max + ln(sum exp(logit - max))).
 *  - D must be 128.
 *  - Pointers are DEVICE pointers on the current CUDA device, 16-byte
 *    aligned, owned by the caller; the library never frees, keeps or
 *    allocates device memory on behalf of a call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream.
 *  - Argument errors are detected on the host before any launch and return
 *    a status with nothing launched.  No C++ exception crosses the ABI.
 *  - The library keeps no mutable per-call host state; concurrent calls from
 *    several host threads are safe.
 */
#ifndef VDIT_ATTN_H
#define VDIT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VDIT_ATTN_ABI_VERSION 1

/* Mask kinds.  A(i) is the set of keys query row i may attend to. */
typedef enum {
    /* A(i) = all keys j < Skv.  Bidirectional self-attention. */
    VDIT_MASK_FULL = 0,
    /* A(i) = { j : floor(j / c) <= floor(i / c) }, c = chunk_tokens.
     * Chunks are contiguous from token 0; the last may be partial.  Requires
     * Sq == Skv.  Keys of later chunks are skipped, not just masked. */
    VDIT_MASK_BLOCK_CAUSAL = 1,
    /* Same arithmetic as FULL; the caller says the keys are a short text
     * sequence (Skv << Sq), e.g. 512 text tokens, and the launch takes the
     * short-key schedule: persistent CTAs, two per SM, each taking one
     * 128-row query tile at a time and loading the next tile's Q while it
     * finishes the current one.  Any Skv is correct; long key sequences run
     * faster as FULL. */
    VDIT_MASK_CROSS = 2,
    /* A(i) = { j : mask[b][h][i / 128][j / 128] != 0 }, a caller-given byte
     * per (128-query, 128-key) block pair; key blocks no query of a tile pair
     * attends to are skipped.  Only through vdit_attn_fwd_block_sparse (and
     * vdit_attn_plan).  Skv <= 262,144. */
    VDIT_MASK_BLOCK_SPARSE = 3
} vdit_mask_kind;

typedef enum {
    VDIT_OK = 0,
    VDIT_ERR_INVALID_ARG = 1,  /* null pointer, negative size, Skv == 0,
                                  bad mask_kind, chunk_tokens < 1 with
                                  BLOCK_CAUSAL, Sq != Skv with BLOCK_CAUSAL,
                                  scale not finite or <= 0, H or B > 65535 */
    VDIT_ERR_UNSUPPORTED = 2,  /* D != 128, or the device is not sm_100 */
    VDIT_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
    VDIT_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
    VDIT_ERR_TIMEOUT = 5,      /* a kernel gave up waiting on one of its own
                                  pipeline barriers (reported by
                                  vdit_get_device_status) */
    VDIT_ERR_WORKSPACE = 6     /* workspace missing or too small */
} vdit_status;

/*
 * vdit_attn_plan -- host-only query, touches no device.
 * Writes the workspace size the _ws entry point needs (0 for every shape in
 * this version) and, if grid_ctas is non-NULL, the number of CTAs the
 * forward launches: B * H * ceil(Sq / 256), or for CROSS the number of
 * 128-row query tiles, B * H * ceil(Sq / 128), which the launch shares out
 * over at most two persistent CTAs per SM.  Same argument rules as
 * vdit_attn_fwd, except that pointers are not involved.
 */
vdit_status vdit_attn_plan(int B, int H, int Sq, int Skv, int D, int mask_kind,
                           int chunk_tokens, size_t* workspace_bytes,
                           int* grid_ctas);

/*
 * vdit_attn_fwd -- launch the attention forward on `stream`.
 *   q, k, v : device bf16 inputs (see conventions above).
 *   o       : device bf16 output, [B][Sq][H][D]; must not alias q/k/v.
 *   lse     : device fp32 output [B][H][Sq], or NULL to skip it.
 *   scale   : multiplies q.k before the softmax (1/sqrt(D) for the Wan
 *             configurations); finite and > 0.
 *   mask_kind, chunk_tokens : see vdit_mask_kind; chunk_tokens is ignored
 *             unless mask_kind == VDIT_MASK_BLOCK_CAUSAL.  mask_kind
 *             VDIT_MASK_BLOCK_SPARSE is rejected here (INVALID_ARG): it needs
 *             vdit_attn_fwd_block_sparse.
 * B == 0, H == 0 or Sq == 0 is a valid empty call: VDIT_OK, nothing launched.
 * Returns VDIT_ERR_CUDA if the launch itself fails.  Timeouts inside the
 * kernel are reported later by vdit_get_device_status.
 */
vdit_status vdit_attn_fwd(const void* q, const void* k, const void* v, void* o,
                          float* lse, int B, int H, int Sq, int Skv, int D,
                          float scale, int mask_kind, int chunk_tokens,
                          void* stream);

/*
 * vdit_attn_fwd_block_sparse -- block-sparse attention: the "Sparse attention
 * (VSA / Block Sparse): skips unimportant token pairs" item of the
 * optimisation list in "Realtime video generation: FLOPS calculation and
 * optimizations" (sudonull.com).
 *   block_mask : device bytes [B][H][ceil(Sq/128)][ceil(Skv/128)], row-major;
 *                nonzero = query block i/128 attends to key block j/128.
 *                Caller-owned, read-only, any alignment.
 *   other arguments as vdit_attn_fwd.
 * A query row whose blocks attend to no key gets O = 0 and LSE = -inf.
 * VDIT_ERR_INVALID_ARG for a NULL mask or Skv > 262,144.
 */
vdit_status vdit_attn_fwd_block_sparse(const void* q, const void* k,
                                       const void* v, void* o, float* lse,
                                       const uint8_t* block_mask, int B, int H,
                                       int Sq, int Skv, int D, float scale,
                                       void* stream);

/*
 * vdit_qk_rms_norm -- per-head RMS norm of the query and key tensors, in one
 * launch:
 *     y[b,s,h,:] = x * rsqrt(mean_d(x^2) + eps) * w[h][:]   (fp32, rounded to bf16)
 * for x the rows of q (weight q_norm_weight) and of k (k_norm_weight).  This
 * is the query/key normalisation of the Wan2.x blocks that the gonka
 * DiT-support discussion (#1155) proposes to serve; its "Pricing policy"
 * section counts normalisation among the parts of a forward pass that grow
 * linearly with the number of latent patches.
 *   q, k          : device bf16 [B][Sq][H][D] and [B][Skv][H][D]; either may
 *                   be absent (NULL) when its token count is 0.
 *   q_out, k_out  : device bf16, same shapes; each is either exactly its
 *                   input (in place) or overlaps no other buffer.
 *   q_norm_weight, k_norm_weight : device fp32 [H][D], or NULL for all ones.
 *   eps           : finite and > 0.
 * D must be 128; every pointer 16-byte aligned (VDIT_ERR_MISALIGNED).
 * Asynchronous on `stream`; HBM-bound (256 bytes read and written per row).
 */
vdit_status vdit_qk_rms_norm(const void* q, const void* k, void* q_out,
                             void* k_out, const float* q_norm_weight,
                             const float* k_norm_weight, float eps, int B,
                             int H, int Sq, int Skv, int D, void* stream);

/*
 * vdit_attn_qknorm_plan -- host-only: the workspace size, in bytes, that
 * vdit_attn_fwd_qknorm needs for this shape (the normalised Q and K).
 * Same shape rules as vdit_attn_plan; VDIT_MASK_BLOCK_SPARSE is not
 * accepted.
 */
vdit_status vdit_attn_qknorm_plan(int B, int H, int Sq, int Skv, int D,
                                  int mask_kind, int chunk_tokens,
                                  size_t* workspace_bytes);

/*
 * vdit_attn_fwd_qknorm -- vdit_attn_fwd on raw Q and K: first
 * vdit_qk_rms_norm of q and k into `workspace`, then the attention on the
 * normalised tensors, queued as a programmatic dependent launch so that its
 * CTAs start while the norm drains (its loads of Q and K wait for the norm
 * to complete).  q and k are not modified.
 *   q_norm_weight, k_norm_weight, eps : as vdit_qk_rms_norm.
 *   workspace     : caller-owned device memory of at least the size
 *                   vdit_attn_qknorm_plan reports, 256-byte aligned, not
 *                   overlapping any other argument (VDIT_ERR_WORKSPACE when
 *                   NULL or too small).
 * Other arguments as vdit_attn_fwd; VDIT_MASK_BLOCK_SPARSE is not accepted
 * (normalise with vdit_qk_rms_norm, then call vdit_attn_fwd_block_sparse).
 */
vdit_status vdit_attn_fwd_qknorm(const void* q, const void* k, const void* v,
                                 void* o, float* lse, const float* q_norm_weight,
                                 const float* k_norm_weight, float eps, int B,
                                 int H, int Sq, int Skv, int D, float scale,
                                 int mask_kind, int chunk_tokens,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * vdit_attn_fwd_qknorm_noalloc -- vdit_attn_fwd_qknorm for callers that
 * cannot allocate device memory: the normalised Q and K go to a scratch
 * buffer built into the library (VDIT_NOALLOC_SCRATCH_BYTES, a fixed
 * device-memory array that every GPU loading the library holds until the
 * process exits) instead of a workspace passed in.  The pages this library
 * follows have no counterpart of this entry point.
 *
 * It exists for code that must not call cudaMalloc: a plugin inside a host
 * application that owns all of the GPU's memory through its own pool (a raw
 * cudaMalloc there bypasses the pool's accounting and can fail once the pool
 * has reserved the rest of the device), and latency-critical loops where
 * cudaMalloc / cudaFree may synchronise the device and stall other work.
 * The entry point itself calls neither.
 *
 * Arguments, layouts and results are those of vdit_attn_fwd_qknorm, minus
 * the workspace.  Shapes whose normalised Q and K need more than
 * VDIT_NOALLOC_SCRATCH_BYTES (vdit_attn_qknorm_plan gives the need) return
 * VDIT_ERR_WORKSPACE with nothing launched.
 *
 * The first call on a device looks up the scratch's device address (once
 * per device, with that device current); make that first call before any
 * stream capture.  Only a lookup that succeeded is kept, so a first call
 * that failed is retried by the next one.  The address stays valid until the
 * device is reset (cudaDeviceReset unloads the library's device code, as it
 * does the kernel attributes the library sets once per device); do not reset
 * a device while the library is in use on it.  Arguments are checked in the
 * order vdit_attn_fwd_qknorm checks them, so both accept the same calls; on
 * a GPU that is not sm_100 the call returns VDIT_ERR_UNSUPPORTED.
 * All calls on a device share the one scratch buffer and it
 * keeps the last call's contents (nothing in it needs to start at zero), so
 * calls whose work overlaps on the GPU (other streams, or other host threads
 * without ordering between their streams) race on it: order them.
 */
#define VDIT_NOALLOC_SCRATCH_BYTES (64u << 20) /* 64 MiB */

vdit_status vdit_attn_fwd_qknorm_noalloc(const void* q, const void* k,
                                         const void* v, void* o, float* lse,
                                         const float* q_norm_weight,
                                         const float* k_norm_weight, float eps,
                                         int B, int H, int Sq, int Skv, int D,
                                         float scale, int mask_kind,
                                         int chunk_tokens, void* stream);

/*
 * 8-bit path: "VC-Attention: revolution in video generation speed without
 * retraining" (aikraft.ru), sections 02 (V-Smooth) and 03 (ExpCast-FP8).
 *
 *  - Q and K become E4M3 codes per 128-token block of one (b, h), scale =
 *    block absmax / 448.
 *  - V-Smooth: per 128-token block the mean is subtracted; the residual is
 *    quantised to E4M3 with one scale per (b, h, channel) = max(max |residual|,
 *    2^-8 max |block mean|) / 448; the block mean is added back through the
 *    softmax row sum.
 *  - ExpCast-FP8: each probability's E4M3 byte is written from the
 *    log-domain score as rint(8 log2(p 2^5) + 56 - 0.35) with one FMA, no
 *    exponential; the reference maximum is kept on the grid N + 0.65 (code
 *    units, 8 x log2) and raised only when a tile's max exceeds it by more
 *    than 24 codes.
 * O is bf16 and LSE fp32 as in vdit_attn_fwd; the result differs from
 * vdit_attn_fwd by the 8-bit quantisation (a few percent relative RMS on
 * iid data).  Masks: FULL, BLOCK_CAUSAL, CROSS; as in vdit_attn_fwd, CROSS
 * takes the short-key schedule (persistent CTAs, two per SM, one 128-row
 * query tile at a time) with the same per-row arithmetic.  D must be 128.
 *
 * The caller owns a device workspace (256-byte aligned, size from
 * vdit_attn_fp8_plan) that holds the codes; its parts, in this order, are
 * located by vdit_fp8_layout:
 */
enum {
    VDIT_FP8_PART_Q = 0,       /* uint8 [B][Sq][H][128]  E4M3 codes of Q        */
    VDIT_FP8_PART_K = 1,       /* uint8 [B][Skv][H][128] E4M3 codes of K        */
    VDIT_FP8_PART_VT = 2,      /* uint8 [B][H][nkb][128 ch][128 tok] V residual codes, per block transposed */
    VDIT_FP8_PART_MU_IMG = 3,  /* [B][H][nkb] 4 KB restore tiles (bf16 block mean / channel scale, hi/lo) */
    VDIT_FP8_PART_Q_SCALE = 4, /* fp32 [B][H][nqb]                            */
    VDIT_FP8_PART_K_SCALE = 5, /* fp32 [B][H][nkb]                            */
    VDIT_FP8_PART_V_SCALE = 6, /* fp32 [B][H][128]                            */
    VDIT_FP8_PART_V_AMAX = 7,  /* scratch of the V statistics                 */
    VDIT_FP8_PART_MU = 8,      /* fp32 [B][H][nkb][128] block means of V      */
    VDIT_FP8_NUM_PARTS = 9
};

/* Host-only: offsets[0..8] = byte offset of each part, offsets[9] = total. */
vdit_status vdit_fp8_layout(int B, int H, int Sq, int Skv, int D, size_t* offsets);

/* Host-only: workspace bytes of the 8-bit path for this shape. */
vdit_status vdit_attn_fp8_plan(int B, int H, int Sq, int Skv, int D,
                               int mask_kind, int chunk_tokens,
                               size_t* workspace_bytes);

/* Quantise bf16 q, k, v into the workspace (four launches on `stream`). */
vdit_status vdit_fp8_quantize(const void* q, const void* k, const void* v,
                              int B, int H, int Sq, int Skv, int D,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/* The 8-bit attention on a workspace that vdit_fp8_quantize filled. */
vdit_status vdit_attn_fwd_fp8_quantized(void* o, float* lse, int B, int H,
                                        int Sq, int Skv, int D, float scale,
                                        int mask_kind, int chunk_tokens,
                                        const void* workspace,
                                        size_t workspace_bytes, void* stream);

/* vdit_fp8_quantize, then the 8-bit attention as a programmatic dependent
 * launch.  Errors as vdit_attn_fwd, plus VDIT_ERR_WORKSPACE. */
vdit_status vdit_attn_fwd_fp8(const void* q, const void* k, const void* v,
                              void* o, float* lse, int B, int H, int Sq,
                              int Skv, int D, float scale, int mask_kind,
                              int chunk_tokens, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * V-Smooth "Group" (VC-Attention (aikraft.ru), section 02): cluster the value
 * tokens of every (batch, head) with a k-means warm-started from the caller's
 * centroids (the previous denoising step's), then permute K and V together
 * so that each cluster's tokens are adjacent.  A joint K/V permutation leaves
 * non-causal attention (FULL, CROSS) unchanged, and the 128-token blocks of
 * the permuted sequence have block means that remove more of V before the
 * 8-bit path quantises it.  Not for BLOCK_CAUSAL.
 *
 * vdit_vsmooth_group runs `iters` Lloyd iterations (assign each token to its
 * nearest centroid in squared Euclidean distance, lowest index on ties; move
 * each centroid to the mean of its tokens, keeping centroids without tokens),
 * then assigns once more and sorts stably by cluster:
 *   v          device bf16 [B][S][H][128]
 *   centroids  device fp32 [B][H][C][128], read and updated in place
 *   labels     device int32 [B][H][S], the final assignment
 *   perm       device int32 [B][H][S]: perm[b][h][i] = the token at position i
 *   C          1 .. 64 clusters
 *   workspace  device, vdit_vsmooth_group_plan bytes, 256-byte aligned (may be
 *              NULL when iters == 0)
 * Centroid sums use float atomics, so centroids may differ in the last bits
 * from run to run; labels and perm are then the exact consequence of them.
 */
vdit_status vdit_vsmooth_group_plan(int B, int H, int S, int D, int C,
                                    size_t* workspace_bytes);
vdit_status vdit_vsmooth_group(const void* v, float* centroids,
                               int32_t* labels, int32_t* perm, int B, int H,
                               int S, int D, int C, int iters,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* k_out[b][i][h][:] = k[b][perm[b][h][i]][h][:], the same for v (bf16,
 * [B][S][H][128]).  Outputs must not overlap any input. */
vdit_status vdit_permute_kv(const void* k, const void* v, const int32_t* perm,
                            void* k_out, void* v_out, int B, int H, int S,
                            int D, void* stream);

/*
 * vdit_attn_fwd_ws -- vdit_attn_fwd with a caller-owned device workspace of
 * `workspace_bytes` bytes (at least what vdit_attn_plan reports; NULL is
 * accepted when that is 0).
 */
vdit_status vdit_attn_fwd_ws(const void* q, const void* k, const void* v,
                             void* o, float* lse, int B, int H, int Sq,
                             int Skv, int D, float scale, int mask_kind,
                             int chunk_tokens, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * vdit_attn_merge -- fold a partial attention result into a running one.
 * For each (b, h, i), with (o_acc, lse_acc) attention over one key set and
 * (o_part, lse_part) over a disjoint key set, writes attention over their
 * union into (o_acc, lse_acc):
 *   LSE = ln(e^lse_acc + e^lse_part),
 *   O   = e^(lse_acc - LSE) o_acc + e^(lse_part - LSE) o_part.
 * This is the combine step of ring context parallelism over K/V blocks (the
 * Wave Forcing digest (airadar.tv) compares Wave Parallelism with Ulysses and
 * Ring context parallelism); it is why vdit_attn_fwd returns LSE.
 *   o_acc, o_part     : device bf16 [B][S][H][D] (BSHD), D == 128
 *   lse_acc, lse_part : device fp32 [B][H][S], natural log
 * A row with lse = -inf contributes nothing; two -inf rows give O = 0,
 * LSE = -inf.  fp32 arithmetic, O rounded to bf16.  Buffers must not overlap
 * (except that o_acc and lse_acc are read and written in place); pointers
 * 16-byte aligned.  Asynchronous on `stream`.
 */
vdit_status vdit_attn_merge(void* o_acc, float* lse_acc, const void* o_part,
                            const float* lse_part, int B, int H, int S, int D,
                            void* stream);

/*
 * vdit_attn_merge_f32 -- vdit_attn_merge with the running O kept in fp32.
 * Same formula and rules, but o_acc is device fp32 [B][S][H][D], so a ring
 * of N ranks rounds its merged O to bf16 once instead of after each of its
 * N - 1 folds.  o_part stays bf16 (the forward's output).  o_out, when not
 * NULL, is a device bf16 [B][S][H][D] buffer that also receives the merged O
 * rounded to bf16 (round to nearest even); pass it on the last fold.
 * Start a ring with o_acc = 0 and lse_acc = -inf: the first fold then copies
 * the first partial exactly.  No buffer may overlap another except o_acc and
 * lse_acc with themselves; pointers 16-byte aligned.  Asynchronous on
 * `stream`.  The same passages define it as vdit_attn_merge.
 */
vdit_status vdit_attn_merge_f32(float* o_acc, float* lse_acc, const void* o_part,
                                const float* lse_part, void* o_out, int B,
                                int H, int S, int D, void* stream);

/*
 * vdit_get_device_status -- synchronises `stream`, then reads and clears the
 * current device's error word that the kernels set when a bounded wait on
 * one of their pipeline barriers runs out.  Returns VDIT_OK,
 * VDIT_ERR_TIMEOUT, or VDIT_ERR_CUDA if the synchronisation itself failed.
 * If `detail` is non-NULL it receives the raw error word (0 when clean).
 */
vdit_status vdit_get_device_status(void* stream, uint32_t* detail);

/* Static, human-readable name of a status code. */
const char* vdit_status_string(int status);

/* VDIT_ATTN_ABI_VERSION of the loaded library. */
int vdit_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VDIT_ATTN_H */
