/*
 * attn_oracle.c -- fp64 CPU oracle for the video-DiT attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * tests, the smoke check and the benchmark's CPU-baseline leg compare the CUDA
 * path against.  Nothing on the product path may link, load or call it, and it
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, no tiling, no online softmax):
 *
 *   Full self-attention over the flattened spatiotemporal token sequence, one
 *   softmax(scale * Q K^T) V per (batch, head) -- "VC-Attention" (aikraft.ru),
 *   section 01 "Why attention became the bottleneck": the clip is flattened
 *   into one long token sequence and full self-attention runs in every layer.
 *   The same core serves text->video cross-attention, where the keys/values
 *   are the text tokens -- "Realtime video generation: FLOPS calculation and
 *   optimizations" (sudonull.com), the per-layer block list (self-attention,
 *   cross-attention, FFN).
 *
 *   Block-causal attention over latent-frame chunks: later chunks read the
 *   earlier chunks' K/V, full attention inside a chunk -- the Wave Forcing
 *   digest (airadar.tv), summary paragraph ("block-causal attention") and the
 *   usage notes (num-frames divisible by 3, i.e. 3-latent-frame chunks).
 *
 * For every batch b, head h and query row i with allowed key set A(i):
 *
 *   l_ij  = scale * sum_d q[b,i,h,d] * k[b,j,h,d]        j in A(i)
 *   M_i   = max_j l_ij
 *   Z_i   = sum_j exp(l_ij - M_i)
 *   O[i]  = sum_j exp(l_ij - M_i) * v[b,j,h,:] / Z_i
 *   LSE_i = M_i + ln Z_i                                  (natural log)
 *
 *   A(i) = { j : 0 <= j < Skv }                       FULL (0) and CROSS (2)
 *   A(i) = { j : j < Skv and floor(j/c) <= floor(i/c) } BLOCK_CAUSAL (1)
 *   A(i) = { j : j < Skv and mask[b][h][i/128][j/128] }  BLOCK_SPARSE (3)
 *
 * BLOCK_SPARSE is the block-sparse attention of the sudonull.com page's
 * optimisation list ("Sparse attention (VSA / Block Sparse): skips unimportant
 * token pairs"): a caller-given byte per (128-query, 128-key) block says
 * whether the pair of blocks attends.
 *
 * An empty A(i) gives O = 0 and LSE = -inf.  Subtracting M_i before exp is the
 * textbook overflow guard; it changes nothing in exact arithmetic.
 *
 * Inputs are the raw bf16 bit patterns, layout [B][S][H][D] (BSHD); each value
 * is widened exactly to double.  All arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MASK_FULL 0
#define ORACLE_MASK_BLOCK_CAUSAL 1
#define ORACLE_MASK_CROSS 2
#define ORACLE_MASK_BLOCK_SPARSE 3
#define ORACLE_SPARSE_BLOCK 128

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double widen_bf16(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Keys j < n are candidates: the allowed set of FULL, CROSS and
 * BLOCK_CAUSAL is exactly the prefix [0, n); BLOCK_SPARSE further needs the
 * block bit (key_allowed). */
static int64_t allowed_prefix(int mask_kind, int64_t i, int64_t Skv, int64_t chunk) {
    if (mask_kind == ORACLE_MASK_BLOCK_CAUSAL) {
        int64_t end = (i / chunk + 1) * chunk; /* first key of the next chunk */
        return end < Skv ? end : Skv;
    }
    return Skv;
}

static int key_allowed(int mask_kind, const uint8_t* mask_row, int64_t j) {
    if (mask_kind != ORACLE_MASK_BLOCK_SPARSE) return 1;
    return mask_row[j / ORACLE_SPARSE_BLOCK] != 0;
}

/* One query row.  logits: scratch of Skv doubles.  mask_row: the row's
 * block-mask row (BLOCK_SPARSE only). */
static void oracle_row(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       int64_t H, int64_t Sq, int64_t Skv, int64_t D,
                       double scale, int mask_kind, int64_t chunk, const uint8_t* mask_row,
                       int64_t b, int64_t h, int64_t i,
                       double* logits, double* o_row, double* lse_out) {
    const uint16_t* qi = q + ((b * Sq + i) * H + h) * D;
    int64_t n = allowed_prefix(mask_kind, i, Skv, chunk);
    for (int64_t d = 0; d < D; ++d) o_row[d] = 0.0;
    /* l_ij = scale * <q_i, k_j> for the allowed keys */
    double M = -INFINITY;
    int64_t count = 0;
    for (int64_t j = 0; j < n; ++j) {
        if (!key_allowed(mask_kind, mask_row, j)) continue;
        const uint16_t* kj = k + ((b * Skv + j) * H + h) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += widen_bf16(qi[d]) * widen_bf16(kj[d]);
        logits[j] = scale * dot;
        if (logits[j] > M) M = logits[j];
        ++count;
    }
    if (count == 0) {
        *lse_out = -INFINITY;
        return;
    }
    /* Z_i and the unnormalised weighted sum of V rows */
    double Z = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        if (!key_allowed(mask_kind, mask_row, j)) continue;
        const uint16_t* vj = v + ((b * Skv + j) * H + h) * D;
        double w = exp(logits[j] - M);
        Z += w;
        for (int64_t d = 0; d < D; ++d) o_row[d] += w * widen_bf16(vj[d]);
    }
    for (int64_t d = 0; d < D; ++d) o_row[d] /= Z;
    *lse_out = M + log(Z);
}

/*
 * vdit_oracle_attn -- rows selected by `sel` (nsel triples b,h,i), or every row
 * in (b, h, i) order when sel == NULL (then nsel is ignored and B*H*Sq rows are
 * written).  o: [rows][D] doubles, lse: [rows] doubles.  block_mask: for
 * BLOCK_SPARSE, [B][H][ceil(Sq/128)][ceil(Skv/128)] bytes (nonzero = the
 * blocks attend), else ignored.  nthreads <= 0 uses the OpenMP default.
 * Returns 0, or -1 on a bad argument.
 */
int vdit_oracle_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int64_t B, int64_t H, int64_t Sq, int64_t Skv, int64_t D,
                     double scale, int mask_kind, int64_t chunk, const uint8_t* block_mask,
                     const int64_t* sel, int64_t nsel,
                     double* o, double* lse, int nthreads) {
    if (!q || !k || !v || !o || !lse) return -1;
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D <= 0) return -1;
    if (mask_kind != ORACLE_MASK_FULL && mask_kind != ORACLE_MASK_BLOCK_CAUSAL &&
        mask_kind != ORACLE_MASK_CROSS && mask_kind != ORACLE_MASK_BLOCK_SPARSE)
        return -1;
    if (mask_kind == ORACLE_MASK_BLOCK_CAUSAL && chunk <= 0) return -1;
    if (mask_kind == ORACLE_MASK_BLOCK_SPARSE && !block_mask) return -1;
    const int64_t nqb = (Sq + ORACLE_SPARSE_BLOCK - 1) / ORACLE_SPARSE_BLOCK;
    const int64_t nkb = (Skv + ORACLE_SPARSE_BLOCK - 1) / ORACLE_SPARSE_BLOCK;
    int64_t rows = sel ? nsel : B * H * Sq;
    if (sel) {
        for (int64_t r = 0; r < rows; ++r) {
            int64_t b = sel[3 * r], h = sel[3 * r + 1], i = sel[3 * r + 2];
            if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Sq) return -1;
        }
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!logits) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < rows; ++r) {
                int64_t b, h, i;
                if (sel) {
                    b = sel[3 * r];
                    h = sel[3 * r + 1];
                    i = sel[3 * r + 2];
                } else {
                    b = r / (H * Sq);
                    h = (r / Sq) % H;
                    i = r % Sq;
                }
                const uint8_t* mask_row =
                    mask_kind == ORACLE_MASK_BLOCK_SPARSE
                        ? block_mask + ((b * H + h) * nqb + i / ORACLE_SPARSE_BLOCK) * nkb
                        : NULL;
                oracle_row(q, k, v, H, Sq, Skv, D, scale, mask_kind, chunk, mask_row, b, h, i,
                           logits, o + r * D, lse + r);
            }
            free(logits);
        }
    }
    return failed ? -1 : 0;
}

/* Threads the OpenMP runtime will use by default (for reporting). */
int vdit_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
