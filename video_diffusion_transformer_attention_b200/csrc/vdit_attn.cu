// vdit_attn.cu -- host side of libvdit_attn.so: argument validation, TMA
// tensor maps, launch, and the device status word.  The C ABI is declared in
// include/vdit_attn.h; every entry point returns a status code and lets no
// C++ exception escape.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "vdit_attn.h"
#include "vdit_attn_testing.h"
#include "attn_fwd_sm100.cuh"
#include "attn_cross_sm100.cuh"
#include "attn_cross_fp8_sm100.cuh"
#include "attn_merge.cuh"
#include "qk_norm.cuh"
#include "fp8_quant.cuh"
#include "attn_fwd_fp8_sm100.cuh"
#include "vsmooth_group.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitTimeoutNs = 2000000000ull;  // 2 s per barrier wait

// ------------------------------------------------------------ argument checks

struct Shape {
    int B, H, Sq, Skv, D, mask_kind, chunk;
};

vdit_status check_shape(const Shape& s, bool check_scale, float scale) {
    if (s.B < 0 || s.H < 0 || s.Sq < 0 || s.Skv < 1 || s.D < 1) return VDIT_ERR_INVALID_ARG;
    if (s.mask_kind != VDIT_MASK_FULL && s.mask_kind != VDIT_MASK_BLOCK_CAUSAL && s.mask_kind != VDIT_MASK_CROSS &&
        s.mask_kind != VDIT_MASK_BLOCK_SPARSE)
        return VDIT_ERR_INVALID_ARG;
    if (s.mask_kind == VDIT_MASK_BLOCK_SPARSE &&
        (s.Skv + vdit::kSparseBlock - 1) / vdit::kSparseBlock > vdit::kMaxSparseKvBlocks)
        return VDIT_ERR_INVALID_ARG;
    if (s.D != vdit::kHeadDim) return VDIT_ERR_UNSUPPORTED;
    if (s.mask_kind == VDIT_MASK_BLOCK_CAUSAL && (s.chunk < 1 || s.Sq != s.Skv)) return VDIT_ERR_INVALID_ARG;
    if (s.B > 65535 || s.H > 65535) return VDIT_ERR_INVALID_ARG;
    if (check_scale && !(std::isfinite(scale) && scale > 0.0f)) return VDIT_ERR_INVALID_ARG;
    return VDIT_OK;
}

int grid_x(int Sq) {
    const long long rows = vdit::kQTiles * vdit::kBlockM;  // query rows per CTA; no int overflow near INT_MAX
    return static_cast<int>((static_cast<long long>(Sq) + rows - 1) / rows);
}

// 128-row query tiles per (batch, head): the cross-attention work items
int cross_tiles(int Sq) { return static_cast<int>((static_cast<long long>(Sq) + vdit::kBlockM - 1) / vdit::kBlockM); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// ------------------------------------------------------------ per-device setup

struct DeviceState {
    std::once_flag once;
    vdit_status status = VDIT_ERR_CUDA;
    int norm_grid = 0;   // one full wave of qk_rms_norm_kernel blocks
    int cross_grid = 0;  // the persistent cross-attention grid: two CTAs per SM
};
DeviceState g_devices[kMaxDevices];

void init_device(int dev, DeviceState* st) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        st->status = VDIT_ERR_CUDA;
        return;
    }
    if (major != 10 || minor != 0) {
        st->status = VDIT_ERR_UNSUPPORTED;
        return;
    }
    if (cudaFuncSetAttribute(vdit::attn_fwd_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_fwd_sm100_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kSmemBytesSparse) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_fwd_sm100_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_cross_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kCrossSmemBytes) != cudaSuccess ||
        // all of the unified L1 / shared storage as shared memory: two CTAs fit
        cudaFuncSetAttribute(vdit::attn_cross_sm100_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_fwd_fp8_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kF8SmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_fwd_fp8_sm100_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kF8SmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_cross_fp8_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             vdit::kF8CrossSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(vdit::attn_cross_fp8_sm100_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
        st->status = VDIT_ERR_CUDA;
        return;
    }
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, vdit::qk_rms_norm_kernel, vdit::kNormThreads, 0) !=
            cudaSuccess ||
        sms < 1 || per_sm < 1) {
        st->status = VDIT_ERR_CUDA;
        return;
    }
    st->norm_grid = sms * per_sm;
    // Two CTAs per SM: what the cross kernel's TMEM (256 of 512 columns),
    // registers (2 x 192 x 168) and shared memory (2 x 97 KB) allow.  The
    // occupancy query reports one for this kernel, but two run side by side
    // (measured: 1.02 vs 1.68 ms at Sq = 75,600, H = 40, Skv = 512).  The CTAs
    // never wait on one another, so the grid is correct at any residency.
    st->cross_grid = sms * 2;
    st->status = VDIT_OK;
}

vdit_status ensure_device(int* dev_out, const DeviceState** state_out = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return VDIT_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return VDIT_ERR_UNSUPPORTED;
    DeviceState* st = &g_devices[dev];
    std::call_once(st->once, init_device, dev, st);
    *dev_out = dev;
    if (state_out != nullptr) *state_out = st;
    return st->status;
}

// ------------------------------------------------------------ TMA tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
    if (f == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        fn.store(f);
    }
    return f;
}

// [B][S][H][D] bf16 viewed as a 4-D tensor (D, H, S, B), innermost first; a
// box is 64 head dims x 1 head x 128 tokens x 1 batch, 128-byte swizzled, so
// each box lands as 128 rows of 128 bytes (one K-major / MN-major SW128 atom
// column).  Rows past S read as zero.
bool encode_bshd(CUtensorMap* map, const void* base, int B, int S, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 f = encode_fn();
    if (f == nullptr) return false;
    const cuuint64_t D = vdit::kHeadDim;
    cuuint64_t dims[4] = {D, cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
    cuuint64_t strides[3] = {D * 2, cuuint64_t(H) * D * 2, cuuint64_t(S) * cuuint64_t(H) * D * 2};
    cuuint32_t box[4] = {64, 1, cuuint32_t(vdit::kBlockM), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The output O as a store target for the cross-attention epilogue: the same
// 4-D view, boxes of 64 head dims x 32 tokens (a warp's rows, 128 bytes each),
// 128-byte swizzled.  Rows past S are not written.
static_assert(vdit::kStageCols == vdit::kCrossStageCols && vdit::kStageRows == vdit::kCrossStageRows,
              "the dense and cross epilogues store O in the same 64-dim x 32-row boxes");

bool encode_bshd_store(CUtensorMap* map, void* base, int B, int S, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 f = encode_fn();
    if (f == nullptr) return false;
    const cuuint64_t D = vdit::kHeadDim;
    cuuint64_t dims[4] = {D, cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
    cuuint64_t strides[3] = {D * 2, cuuint64_t(H) * D * 2, cuuint64_t(S) * cuuint64_t(H) * D * 2};
    cuuint32_t box[4] = {cuuint32_t(vdit::kCrossStageCols), 1, cuuint32_t(vdit::kCrossStageRows), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

vdit_status launch(const void* q, const void* k, const void* v, void* o, float* lse, const uint8_t* block_mask,
                   const Shape& s, float scale, int debug_flags, unsigned long long timeout_ns, cudaStream_t stream,
                   bool after_norm, unsigned long long* cta_spans = nullptr, int max_span_ctas = 0) {
    int dev = 0;
    const DeviceState* ds = nullptr;
    vdit_status st = ensure_device(&dev, &ds);
    if (st != VDIT_OK) return st;
    CUtensorMap tq, tk, tv;
    if (!encode_bshd(&tq, q, s.B, s.Sq, s.H) || !encode_bshd(&tk, k, s.B, s.Skv, s.H) ||
        !encode_bshd(&tv, v, s.B, s.Skv, s.H))
        return VDIT_ERR_CUDA;
    vdit::FwdParams p{};
    p.B = s.B;
    p.H = s.H;
    p.Sq = s.Sq;
    p.Skv = s.Skv;
    p.mask_kind = s.mask_kind;
    p.chunk = s.mask_kind == VDIT_MASK_BLOCK_CAUSAL ? s.chunk : 1;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.timeout_ns = timeout_ns;
    p.debug_flags = debug_flags;
    p.block_mask = block_mask;
    p.n_qb = (s.Sq + vdit::kSparseBlock - 1) / vdit::kSparseBlock;
    p.n_kvb = (s.Skv + vdit::kSparseBlock - 1) / vdit::kSparseBlock;
    CUtensorMap to;
    if (!encode_bshd_store(&to, o, s.B, s.Sq, s.H)) return VDIT_ERR_CUDA;
    if (s.mask_kind == VDIT_MASK_CROSS) {
        // Short key sequence: persistent, two CTAs per SM, one 128-row query tile per item.
        const long long items = static_cast<long long>(p.n_qb) * s.H * s.B;
        const dim3 grid(static_cast<unsigned>(items < ds->cross_grid ? items : ds->cross_grid));
        const vdit::CrossSpans rec{cta_spans, max_span_ctas};
        if (!after_norm) {
            vdit::attn_cross_sm100_kernel<<<grid, vdit::kCrossThreads, vdit::kCrossSmemBytes, stream>>>(tq, tk, tv, to,
                                                                                                      p, rec);
            return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
        }
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(vdit::kCrossThreads);
        cfg.dynamicSmemBytes = vdit::kCrossSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, vdit::attn_cross_sm100_kernel, tq, tk, tv, to, p, rec) == cudaSuccess
                   ? VDIT_OK
                   : VDIT_ERR_CUDA;
    }
    dim3 grid(grid_x(s.Sq), s.H, s.B);
    if (!after_norm) {
        if (s.mask_kind == VDIT_MASK_BLOCK_SPARSE)
            vdit::attn_fwd_sm100_kernel<true><<<grid, vdit::kNumThreads, vdit::kSmemBytesSparse, stream>>>(tq, tk, tv,
                                                                                                         to, p);
        else if (s.mask_kind == VDIT_MASK_BLOCK_CAUSAL)
            vdit::attn_fwd_sm100_kernel<false, true><<<grid, vdit::kNumThreads, vdit::kSmemBytes, stream>>>(tq, tk, tv,
                                                                                                         to, p);
        else
            vdit::attn_fwd_sm100_kernel<false><<<grid, vdit::kNumThreads, vdit::kSmemBytes, stream>>>(tq, tk, tv, to,
                                                                                                   p);
        return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
    }
    // Programmatic dependent of the Q/K norm kernel just queued on this
    // stream: CTAs may start while it drains; the TMA producer waits for it
    // (griddepcontrol.wait) before loading Q or K.
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(vdit::kNumThreads);
    cfg.dynamicSmemBytes = vdit::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (s.mask_kind == VDIT_MASK_BLOCK_CAUSAL)
        return cudaLaunchKernelEx(&cfg, vdit::attn_fwd_sm100_kernel<false, true>, tq, tk, tv, to, p) == cudaSuccess
                   ? VDIT_OK
                   : VDIT_ERR_CUDA;
    return cudaLaunchKernelEx(&cfg, vdit::attn_fwd_sm100_kernel<false>, tq, tk, tv, to, p) == cudaSuccess
               ? VDIT_OK
               : VDIT_ERR_CUDA;
}

vdit_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                     int Skv, int D, float scale, int mask_kind, int chunk_tokens, void* workspace,
                     size_t workspace_bytes, void* stream, int debug_flags = 0,
                     unsigned long long timeout_ns = kDefaultWaitTimeoutNs,
                     const uint8_t* block_mask = nullptr, bool after_norm = false,
                     unsigned long long* cta_spans = nullptr, int max_span_ctas = 0) {
    (void)workspace;
    (void)workspace_bytes;  // no shape needs a workspace in this version
    const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
    vdit_status st = check_shape(s, true, scale);
    if (st != VDIT_OK) return st;
    if (B == 0 || H == 0 || Sq == 0) return VDIT_OK;
    if ((mask_kind == VDIT_MASK_BLOCK_SPARSE) != (block_mask != nullptr)) return VDIT_ERR_INVALID_ARG;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return VDIT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return VDIT_ERR_MISALIGNED;
    const size_t row_bytes = size_t(H) * size_t(D) * 2;
    const size_t q_bytes = size_t(B) * size_t(Sq) * row_bytes;
    const size_t kv_bytes = size_t(B) * size_t(Skv) * row_bytes;
    if (overlaps(o, q_bytes, q, q_bytes) || overlaps(o, q_bytes, k, kv_bytes) || overlaps(o, q_bytes, v, kv_bytes))
        return VDIT_ERR_INVALID_ARG;
    if (lse != nullptr) {
        const size_t lse_bytes = size_t(B) * size_t(H) * size_t(Sq) * 4;
        if (overlaps(lse, lse_bytes, o, q_bytes) || overlaps(lse, lse_bytes, q, q_bytes) ||
            overlaps(lse, lse_bytes, k, kv_bytes) || overlaps(lse, lse_bytes, v, kv_bytes))
            return VDIT_ERR_INVALID_ARG;
    }
    if (block_mask != nullptr) {
        const size_t mask_bytes = size_t(B) * size_t(H) * size_t((Sq + vdit::kSparseBlock - 1) / vdit::kSparseBlock) *
                                  size_t((Skv + vdit::kSparseBlock - 1) / vdit::kSparseBlock);
        if (overlaps(block_mask, mask_bytes, o, q_bytes) ||
            (lse != nullptr && overlaps(block_mask, mask_bytes, lse, size_t(B) * size_t(H) * size_t(Sq) * 4)))
            return VDIT_ERR_INVALID_ARG;
    }
    return launch(q, k, v, o, lse, block_mask, s, scale, debug_flags, timeout_ns, static_cast<cudaStream_t>(stream),
                  after_norm, cta_spans, max_span_ctas);
}

// ------------------------------------------------------------ Q/K RMS norm

constexpr size_t kWorkspaceAlign = 256;

size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

// Validates and queues the per-head RMS norm of q (B*Sq*H rows) and k
// (B*Skv*H rows) into q_out / k_out.  Each output is the same address as its
// input or disjoint from every input and output.
vdit_status qk_norm_impl(const void* q, const void* k, void* q_out, void* k_out, const float* q_w, const float* k_w,
                         float eps, int B, int H, int Sq, int Skv, int D, cudaStream_t stream) {
    if (B < 0 || H < 0 || Sq < 0 || Skv < 0 || D < 1) return VDIT_ERR_INVALID_ARG;
    if (D != vdit::kNormHeadDim) return VDIT_ERR_UNSUPPORTED;
    if (!(std::isfinite(eps) && eps > 0.0f)) return VDIT_ERR_INVALID_ARG;
    const long long q_rows = (long long)B * Sq * H, k_rows = (long long)B * Skv * H;
    if (q_rows == 0 && k_rows == 0) return VDIT_OK;
    if ((q_rows > 0 && (q == nullptr || q_out == nullptr)) || (k_rows > 0 && (k == nullptr || k_out == nullptr)))
        return VDIT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_w) ||
        !aligned16(k_w))
        return VDIT_ERR_MISALIGNED;
    const size_t qb = size_t(q_rows) * 256, kb = size_t(k_rows) * 256;
    const size_t wb = size_t(H) * vdit::kNormHeadDim * 4;
    auto clash = [](const void* a, size_t na, const void* b, size_t nb) {  // overlap other than identity
        return na > 0 && nb > 0 && a != b && overlaps(a, na, b, nb);
    };
    if (clash(q_out, qb, q, qb) || clash(k_out, kb, k, kb) || (qb > 0 && kb > 0 &&
        (overlaps(q_out, qb, k, kb) || overlaps(k_out, kb, q, qb) || overlaps(q_out, qb, k_out, kb))))
        return VDIT_ERR_INVALID_ARG;
    if ((q_w != nullptr && ((qb > 0 && overlaps(q_w, wb, q_out, qb)) || (kb > 0 && overlaps(q_w, wb, k_out, kb)))) ||
        (k_w != nullptr && ((qb > 0 && overlaps(k_w, wb, q_out, qb)) || (kb > 0 && overlaps(k_w, wb, k_out, kb)))))
        return VDIT_ERR_INVALID_ARG;
    int dev = 0;
    const DeviceState* ds = nullptr;
    const vdit_status st = ensure_device(&dev, &ds);
    if (st != VDIT_OK) return st;
    const long long passes = (q_rows + k_rows + 2 * vdit::kNormRowsInFlight - 1) / (2 * vdit::kNormRowsInFlight);
    const long long want = (passes + vdit::kNormThreads / 32 - 1) / (vdit::kNormThreads / 32);
    const unsigned grid = unsigned(want < ds->norm_grid ? want : ds->norm_grid);
    const vdit::NormTensor a{static_cast<const uint4*>(q), static_cast<uint4*>(q_out), q_w, q_rows};
    const vdit::NormTensor b{static_cast<const uint4*>(k), static_cast<uint4*>(k_out), k_w, k_rows};
    vdit::qk_rms_norm_kernel<<<grid, vdit::kNormThreads, 0, stream>>>(a, b, H, eps);
    return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
}

size_t qknorm_workspace_bytes(int B, int H, int Sq, int Skv, int D) {
    const size_t row = size_t(H) * size_t(D) * 2;
    return round_up(size_t(B) * size_t(Sq) * row, kWorkspaceAlign) + size_t(B) * size_t(Skv) * row;
}

// ------------------------------------------------------------ 8-bit path

// Byte offsets of the 8-bit path's workspace parts (the order of
// VDIT_FP8_PART_* in the header), each 256-byte aligned; [VDIT_FP8_NUM_PARTS]
// is the total.
void fp8_layout(int B, int H, int Sq, int Skv, size_t* off) {
    const size_t bh = size_t(B) * size_t(H);
    const size_t nqb = size_t((Sq + vdit::kQuantBlock - 1) / vdit::kQuantBlock);
    const size_t nkb = size_t((Skv + vdit::kQuantBlock - 1) / vdit::kQuantBlock);
    const size_t sizes[VDIT_FP8_NUM_PARTS] = {
        size_t(B) * size_t(Sq) * size_t(H) * 128,  // q8
        size_t(B) * size_t(Skv) * size_t(H) * 128, // k8
        bh * nkb * 128 * 128,                      // vt8
        bh * nkb * vdit::kMuImgBytes,              // mu_img
        bh * nqb * 4,                              // q_scale
        bh * nkb * 4,                              // k_scale
        bh * 128 * 4,                              // v_scale
        bh * 128 * 4 * 2,                          // v_amax_r, v_amax_mu (zeroed together)
        bh * nkb * 128 * 4,                        // mu
    };
    size_t at = 0;
    for (int i = 0; i < VDIT_FP8_NUM_PARTS; ++i) {
        off[i] = at;
        at = round_up(at + sizes[i], kWorkspaceAlign);
    }
    off[VDIT_FP8_NUM_PARTS] = at;
}

vdit::Fp8Tensors fp8_tensors(void* ws, const size_t* off, int B, int H) {
    char* w = static_cast<char*>(ws);
    vdit::Fp8Tensors t;
    t.q8 = reinterpret_cast<uint8_t*>(w + off[VDIT_FP8_PART_Q]);
    t.k8 = reinterpret_cast<uint8_t*>(w + off[VDIT_FP8_PART_K]);
    t.vt8 = reinterpret_cast<uint8_t*>(w + off[VDIT_FP8_PART_VT]);
    t.mu_img = reinterpret_cast<uint8_t*>(w + off[VDIT_FP8_PART_MU_IMG]);
    t.q_scale = reinterpret_cast<float*>(w + off[VDIT_FP8_PART_Q_SCALE]);
    t.k_scale = reinterpret_cast<float*>(w + off[VDIT_FP8_PART_K_SCALE]);
    t.v_scale = reinterpret_cast<float*>(w + off[VDIT_FP8_PART_V_SCALE]);
    t.v_amax_r = reinterpret_cast<uint32_t*>(w + off[VDIT_FP8_PART_V_AMAX]);
    t.v_amax_mu = t.v_amax_r + size_t(B) * size_t(H) * 128;
    t.mu = reinterpret_cast<float*>(w + off[VDIT_FP8_PART_MU]);
    return t;
}

// Shape and workspace checks shared by the 8-bit entry points.
vdit_status fp8_check(const Shape& s, bool check_scale, float scale, void* workspace, size_t workspace_bytes,
                      size_t* off) {
    if (s.mask_kind == VDIT_MASK_BLOCK_SPARSE) return VDIT_ERR_INVALID_ARG;
    vdit_status st = check_shape(s, check_scale, scale);
    if (st != VDIT_OK) return st;
    fp8_layout(s.B, s.H, s.Sq, s.Skv, off);
    if (s.B == 0 || s.H == 0 || s.Sq == 0) return VDIT_OK;
    if (workspace == nullptr || workspace_bytes < off[VDIT_FP8_NUM_PARTS]) return VDIT_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWorkspaceAlign - 1)) != 0) return VDIT_ERR_MISALIGNED;
    return VDIT_OK;
}

vdit_status fp8_quantize_impl(const void* q, const void* k, const void* v, const Shape& s, void* workspace,
                              const size_t* off, cudaStream_t stream) {
    if (q == nullptr || k == nullptr || v == nullptr) return VDIT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return VDIT_ERR_MISALIGNED;
    const size_t row = size_t(s.H) * 256;
    const size_t qb = size_t(s.B) * size_t(s.Sq) * row, kb = size_t(s.B) * size_t(s.Skv) * row;
    const size_t wb = off[VDIT_FP8_NUM_PARTS];
    if (overlaps(workspace, wb, q, qb) || overlaps(workspace, wb, k, kb) || overlaps(workspace, wb, v, kb))
        return VDIT_ERR_INVALID_ARG;
    int dev = 0;
    vdit_status st = ensure_device(&dev);
    if (st != VDIT_OK) return st;
    const vdit::Fp8Tensors t = fp8_tensors(workspace, off, s.B, s.H);
    const long long nqb = (s.Sq + vdit::kQuantBlock - 1) / vdit::kQuantBlock;
    const long long nkb = (s.Skv + vdit::kQuantBlock - 1) / vdit::kQuantBlock;
    const long long bh = (long long)s.B * s.H;
    if (bh * (nqb + nkb) > 0x7fffffffLL) return VDIT_ERR_INVALID_ARG;
    if (cudaMemsetAsync(t.v_amax_r, 0, size_t(bh) * 128 * 4 * 2, stream) != cudaSuccess) return VDIT_ERR_CUDA;
    vdit::qk_quant_kernel<<<unsigned(bh * (nqb + nkb)), vdit::kQuantThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), t, s.B, s.H, s.Sq, s.Skv);
    vdit::v_stats_kernel<<<unsigned(bh * nkb), vdit::kQuantThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), t, s.B, s.H,
                                                                 s.Skv);
    vdit::v_quant_kernel<<<unsigned(bh * nkb), vdit::kQuantThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), t, s.B, s.H,
                                                                 s.Skv);
    return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
}

// E4M3 [B][S][H][128] codes as a 4-D tensor (128 bytes, H, S, B); a box is one
// 128-token tile of one head, 128-byte swizzled.
bool encode_bshd_u8(CUtensorMap* map, const void* base, int B, int S, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 f = encode_fn();
    if (f == nullptr) return false;
    cuuint64_t dims[4] = {128, cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
    cuuint64_t strides[3] = {128, cuuint64_t(H) * 128, cuuint64_t(S) * cuuint64_t(H) * 128};
    cuuint32_t box[4] = {128, 1, cuuint32_t(vdit::kBlockM), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The transposed V codes [blocks][128 channels][128 tokens] as a 3-D tensor.
bool encode_vt_u8(CUtensorMap* map, const void* base, long long blocks) {
    PFN_cuTensorMapEncodeTiled_v12000 f = encode_fn();
    if (f == nullptr) return false;
    cuuint64_t dims[3] = {128, 128, cuuint64_t(blocks)};
    cuuint64_t strides[2] = {128, 128 * 128};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

vdit_status fp8_attention_impl(void* o, float* lse, const Shape& s, float scale, void* workspace,
                               const size_t* off, cudaStream_t stream, bool after_quantize) {
    if (o == nullptr) return VDIT_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(lse)) return VDIT_ERR_MISALIGNED;
    const size_t ob = size_t(s.B) * size_t(s.Sq) * size_t(s.H) * 256;
    const size_t wb = off[VDIT_FP8_NUM_PARTS];
    if (overlaps(o, ob, workspace, wb) ||
        (lse != nullptr && (overlaps(lse, size_t(s.B) * s.H * s.Sq * 4, workspace, wb) ||
                            overlaps(lse, size_t(s.B) * s.H * s.Sq * 4, o, ob))))
        return VDIT_ERR_INVALID_ARG;
    int dev = 0;
    vdit_status st = ensure_device(&dev);
    if (st != VDIT_OK) return st;
    const vdit::Fp8Tensors t = fp8_tensors(workspace, off, s.B, s.H);
    const int nqb = (s.Sq + vdit::kQuantBlock - 1) / vdit::kQuantBlock;
    const int nkb = (s.Skv + vdit::kQuantBlock - 1) / vdit::kQuantBlock;
    CUtensorMap tq, tk, tvt;
    if (!encode_bshd_u8(&tq, t.q8, s.B, s.Sq, s.H) || !encode_bshd_u8(&tk, t.k8, s.B, s.Skv, s.H) ||
        !encode_vt_u8(&tvt, t.vt8, (long long)s.B * s.H * nkb))
        return VDIT_ERR_CUDA;
    vdit::Fp8FwdParams p{};
    p.B = s.B;
    p.H = s.H;
    p.Sq = s.Sq;
    p.Skv = s.Skv;
    p.mask_kind = s.mask_kind;
    p.chunk = s.mask_kind == VDIT_MASK_BLOCK_CAUSAL ? s.chunk : 1;
    p.c0 = static_cast<float>(8.0 * static_cast<double>(scale) * 1.4426950408889634);
    p.q_scale = t.q_scale;
    p.k_scale = t.k_scale;
    p.v_scale = t.v_scale;
    p.mu_img = t.mu_img;
    p.nqb = nqb;
    p.nkb = nkb;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.timeout_ns = kDefaultWaitTimeoutNs;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = after_quantize ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = stream;
    if (s.mask_kind == VDIT_MASK_CROSS) {
        // Short key sequence: persistent, two CTAs per SM, one 128-row query tile per item.
        const DeviceState* ds = nullptr;
        if (ensure_device(&dev, &ds) != VDIT_OK) return VDIT_ERR_CUDA;
        CUtensorMap to;
        if (!encode_bshd_store(&to, o, s.B, s.Sq, s.H)) return VDIT_ERR_CUDA;
        const long long items = static_cast<long long>(nqb) * s.H * s.B;
        cfg.gridDim = dim3(static_cast<unsigned>(items < ds->cross_grid ? items : ds->cross_grid));
        cfg.blockDim = dim3(vdit::kCrossThreads);
        cfg.dynamicSmemBytes = vdit::kF8CrossSmemBytes;
        return cudaLaunchKernelEx(&cfg, vdit::attn_cross_fp8_sm100_kernel, tq, tk, tvt, to, p) == cudaSuccess
                   ? VDIT_OK
                   : VDIT_ERR_CUDA;
    }
    cfg.gridDim = dim3(grid_x(s.Sq), s.H, s.B);
    cfg.blockDim = dim3(vdit::kNumThreads);
    cfg.dynamicSmemBytes = vdit::kF8SmemBytes;
    if (s.mask_kind == VDIT_MASK_BLOCK_CAUSAL)
        return cudaLaunchKernelEx(&cfg, vdit::attn_fwd_fp8_sm100_kernel<true>, tq, tk, tvt, p) == cudaSuccess
                   ? VDIT_OK
                   : VDIT_ERR_CUDA;
    return cudaLaunchKernelEx(&cfg, vdit::attn_fwd_fp8_sm100_kernel<false>, tq, tk, tvt, p) == cudaSuccess
               ? VDIT_OK
               : VDIT_ERR_CUDA;
}

// ------------------------------------------------------------ LSE merge

// Validates and queues one fold of (o_part, lse_part) into (o_acc, lse_acc);
// AccT is the running O's storage (bf16 or fp32), o_out an optional bf16
// copy of the merged O.
template <typename AccT>
vdit_status merge_impl(AccT* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                       int H, int S, int D, cudaStream_t stream) {
    if (B < 0 || H < 0 || S < 0 || D < 1) return VDIT_ERR_INVALID_ARG;
    if (D != vdit::kHeadDim) return VDIT_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || S == 0) return VDIT_OK;
    if (o_acc == nullptr || lse_acc == nullptr || o_part == nullptr || lse_part == nullptr)
        return VDIT_ERR_INVALID_ARG;
    if (!aligned16(o_acc) || !aligned16(o_part) || !aligned16(lse_acc) || !aligned16(lse_part) || !aligned16(o_out))
        return VDIT_ERR_MISALIGNED;
    const long long rows = (long long)B * S * H;
    const long long warps = (long long)B * H * ((S + vdit::kMergeRowsPerWarp - 1) / vdit::kMergeRowsPerWarp);
    const long long blocks = (warps + vdit::kMergeWarpsPerBlock - 1) / vdit::kMergeWarpsPerBlock;
    if (blocks > 0x7fffffffLL) return VDIT_ERR_INVALID_ARG;
    const size_t acc_bytes = size_t(rows) * size_t(D) * sizeof(AccT);
    const size_t o_bytes = size_t(rows) * size_t(D) * 2, l_bytes = size_t(rows) * 4;
    if (overlaps(o_acc, acc_bytes, o_part, o_bytes) || overlaps(lse_acc, l_bytes, lse_part, l_bytes) ||
        overlaps(o_acc, acc_bytes, lse_acc, l_bytes) || overlaps(o_acc, acc_bytes, lse_part, l_bytes) ||
        overlaps(lse_acc, l_bytes, o_part, o_bytes))
        return VDIT_ERR_INVALID_ARG;
    if (o_out != nullptr &&
        (overlaps(o_out, o_bytes, o_acc, acc_bytes) || overlaps(o_out, o_bytes, o_part, o_bytes) ||
         overlaps(o_out, o_bytes, lse_acc, l_bytes) || overlaps(o_out, o_bytes, lse_part, l_bytes)))
        return VDIT_ERR_INVALID_ARG;
    int dev = 0;
    const vdit_status st = ensure_device(&dev);
    if (st != VDIT_OK) return st;
    vdit::attn_merge_kernel<AccT><<<unsigned(blocks), vdit::kMergeWarpsPerBlock * 32, 0, stream>>>(
        o_acc, lse_acc, static_cast<const __nv_bfloat16*>(o_part), lse_part, static_cast<__nv_bfloat16*>(o_out), B,
        H, S);
    return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------ fixed scratch, no allocation
//
// Backing store of vdit_attn_fwd_qknorm_noalloc: the normalised Q and K live
// here instead of in a caller workspace.  Every GPU that loads the library
// holds these bytes until the process exits.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in symbol); the
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[VDIT_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoAllocScratch {
    std::mutex mu;
    void* ptr = nullptr;  // device address of g_noalloc_scratch on this device, once a lookup succeeded
};
NoAllocScratch g_noalloc[kMaxDevices];

// The scratch's device address on `dev`, which must be the current device.
// Only a successful lookup is cached, so a first call that failed (one made
// during a stream capture, say) is retried by the next call instead of
// failing for the rest of the process.  A cudaDeviceReset unloads the module
// that holds the array, after which the cached address is stale: like the
// per-device kernel attributes this library sets once, it assumes the device
// is not reset while the library is in use.
vdit_status noalloc_scratch(int dev, void** out) {
    NoAllocScratch* sc = &g_noalloc[dev];
    std::lock_guard<std::mutex> lock(sc->mu);
    if (sc->ptr == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();  // leave no error behind for the next launch check
            return VDIT_ERR_CUDA;
        }
        sc->ptr = p;
    }
    *out = sc->ptr;
    return VDIT_OK;
}

}  // namespace

extern "C" {

int vdit_abi_version(void) { return VDIT_ATTN_ABI_VERSION; }

const char* vdit_status_string(int status) {
    switch (status) {
        case VDIT_OK: return "VDIT_OK";
        case VDIT_ERR_INVALID_ARG: return "VDIT_ERR_INVALID_ARG";
        case VDIT_ERR_UNSUPPORTED: return "VDIT_ERR_UNSUPPORTED";
        case VDIT_ERR_MISALIGNED: return "VDIT_ERR_MISALIGNED";
        case VDIT_ERR_CUDA: return "VDIT_ERR_CUDA";
        case VDIT_ERR_TIMEOUT: return "VDIT_ERR_TIMEOUT";
        case VDIT_ERR_WORKSPACE: return "VDIT_ERR_WORKSPACE";
        default: return "VDIT_ERR_UNKNOWN";
    }
}

vdit_status vdit_attn_plan(int B, int H, int Sq, int Skv, int D, int mask_kind, int chunk_tokens,
                           size_t* workspace_bytes, int* grid_ctas) {
    try {
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        vdit_status st = check_shape(s, false, 1.0f);
        if (st != VDIT_OK) return st;
        if (workspace_bytes == nullptr) return VDIT_ERR_INVALID_ARG;
        *workspace_bytes = 0;
        if (grid_ctas != nullptr) {
            const long long per_bh = mask_kind == VDIT_MASK_CROSS ? cross_tiles(Sq) : grid_x(Sq);
            const long long n = (B == 0 || H == 0 || Sq == 0) ? 0 : per_bh * H * B;
            *grid_ctas = n > 0x7fffffffLL ? 0x7fffffff : int(n);
        }
        return VDIT_OK;
    } catch (...) {
        return VDIT_ERR_INVALID_ARG;
    }
}

vdit_status vdit_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                          int Skv, int D, float scale, int mask_kind, int chunk_tokens, void* stream) {
    try {
        return fwd_impl(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, nullptr, 0, stream);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int Sq, int Skv, int D, float scale, int mask_kind, int chunk_tokens, void* workspace,
                             size_t workspace_bytes, void* stream) {
    try {
        return fwd_impl(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, workspace,
                        workspace_bytes, stream);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                                       const uint8_t* block_mask, int B, int H, int Sq, int Skv, int D, float scale,
                                       void* stream) {
    try {
        if (B > 0 && H > 0 && Sq > 0 && block_mask == nullptr) return VDIT_ERR_INVALID_ARG;
        return fwd_impl(q, k, v, o, lse, B, H, Sq, Skv, D, scale, VDIT_MASK_BLOCK_SPARSE, 0, nullptr, 0, stream, 0,
                        kDefaultWaitTimeoutNs, block_mask);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_qk_rms_norm(const void* q, const void* k, void* q_out, void* k_out, const float* q_norm_weight,
                             const float* k_norm_weight, float eps, int B, int H, int Sq, int Skv, int D,
                             void* stream) {
    try {
        return qk_norm_impl(q, k, q_out, k_out, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D,
                            static_cast<cudaStream_t>(stream));
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_qknorm_plan(int B, int H, int Sq, int Skv, int D, int mask_kind, int chunk_tokens,
                                  size_t* workspace_bytes) {
    try {
        if (workspace_bytes == nullptr || mask_kind == VDIT_MASK_BLOCK_SPARSE) return VDIT_ERR_INVALID_ARG;
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        const vdit_status st = check_shape(s, false, 1.0f);
        if (st != VDIT_OK) return st;
        *workspace_bytes = qknorm_workspace_bytes(B, H, Sq, Skv, D);
        return VDIT_OK;
    } catch (...) {
        return VDIT_ERR_INVALID_ARG;
    }
}

vdit_status vdit_attn_fwd_qknorm(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const float* q_norm_weight, const float* k_norm_weight, float eps, int B, int H,
                                 int Sq, int Skv, int D, float scale, int mask_kind, int chunk_tokens, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    try {
        if (mask_kind == VDIT_MASK_BLOCK_SPARSE) return VDIT_ERR_INVALID_ARG;
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        vdit_status st = check_shape(s, true, scale);
        if (st != VDIT_OK) return st;
        if (!(std::isfinite(eps) && eps > 0.0f)) return VDIT_ERR_INVALID_ARG;
        if (!aligned16(q_norm_weight) || !aligned16(k_norm_weight)) return VDIT_ERR_MISALIGNED;
        if (B == 0 || H == 0 || Sq == 0) return VDIT_OK;
        const size_t need = qknorm_workspace_bytes(B, H, Sq, Skv, D);
        if (workspace == nullptr || workspace_bytes < need) return VDIT_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & (kWorkspaceAlign - 1)) != 0) return VDIT_ERR_MISALIGNED;
        const size_t row = size_t(H) * size_t(D) * 2;
        const size_t qb = size_t(B) * size_t(Sq) * row, kb = size_t(B) * size_t(Skv) * row;
        if (q == nullptr || k == nullptr || overlaps(workspace, need, q, qb) || overlaps(workspace, need, k, kb) ||
            (v != nullptr && overlaps(workspace, need, v, kb)) ||
            (lse != nullptr && overlaps(workspace, need, lse, size_t(B) * size_t(H) * size_t(Sq) * 4)))
            return VDIT_ERR_INVALID_ARG;
        void* q_n = workspace;
        void* k_n = static_cast<char*>(workspace) + round_up(qb, kWorkspaceAlign);
        if (v == nullptr || o == nullptr) return VDIT_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
            return VDIT_ERR_MISALIGNED;
        if (overlaps(o, qb, q, qb) || overlaps(o, qb, k, kb)) return VDIT_ERR_INVALID_ARG;
        st = qk_norm_impl(q, k, q_n, k_n, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D,
                          static_cast<cudaStream_t>(stream));
        if (st != VDIT_OK) return st;
        return fwd_impl(q_n, k_n, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, nullptr, 0, stream, 0,
                        kDefaultWaitTimeoutNs, nullptr, true);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_fwd_qknorm_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                         const float* q_norm_weight, const float* k_norm_weight, float eps, int B,
                                         int H, int Sq, int Skv, int D, float scale, int mask_kind,
                                         int chunk_tokens, void* stream) {
    try {
        // the argument checks of vdit_attn_fwd_qknorm, in its order, so that
        // the two entry points accept and reject the same calls
        if (mask_kind == VDIT_MASK_BLOCK_SPARSE) return VDIT_ERR_INVALID_ARG;
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        vdit_status st = check_shape(s, true, scale);
        if (st != VDIT_OK) return st;
        if (!(std::isfinite(eps) && eps > 0.0f)) return VDIT_ERR_INVALID_ARG;
        if (!aligned16(q_norm_weight) || !aligned16(k_norm_weight)) return VDIT_ERR_MISALIGNED;
        if (B == 0 || H == 0 || Sq == 0) return VDIT_OK;
        if (qknorm_workspace_bytes(B, H, Sq, Skv, D) > size_t(VDIT_NOALLOC_SCRATCH_BYTES))
            return VDIT_ERR_WORKSPACE;  // the shape does not fit the fixed scratch
        int dev = 0;
        st = ensure_device(&dev);  // an unsupported GPU reports VDIT_ERR_UNSUPPORTED before any lookup
        if (st != VDIT_OK) return st;
        void* scratch = nullptr;
        st = noalloc_scratch(dev, &scratch);
        if (st != VDIT_OK) return st;
        // Nothing in the scratch has to start at zero: the norm writes all of
        // the normalised Q and K before the attention reads them.
        return vdit_attn_fwd_qknorm(q, k, v, o, lse, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, scale,
                                    mask_kind, chunk_tokens, scratch, size_t(VDIT_NOALLOC_SCRATCH_BYTES), stream);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_fp8_layout(int B, int H, int Sq, int Skv, int D, size_t* offsets) {
    try {
        if (offsets == nullptr) return VDIT_ERR_INVALID_ARG;
        const Shape s{B, H, Sq, Skv, D, VDIT_MASK_FULL, 0};
        const vdit_status st = check_shape(s, false, 1.0f);
        if (st != VDIT_OK) return st;
        fp8_layout(B, H, Sq, Skv, offsets);
        return VDIT_OK;
    } catch (...) {
        return VDIT_ERR_INVALID_ARG;
    }
}

vdit_status vdit_attn_fp8_plan(int B, int H, int Sq, int Skv, int D, int mask_kind, int chunk_tokens,
                               size_t* workspace_bytes) {
    try {
        if (workspace_bytes == nullptr) return VDIT_ERR_INVALID_ARG;
        size_t off[VDIT_FP8_NUM_PARTS + 1];
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        const vdit_status st = fp8_check(s, false, 1.0f, nullptr, 0, off);
        if (st != VDIT_OK && st != VDIT_ERR_WORKSPACE) return st;
        *workspace_bytes = off[VDIT_FP8_NUM_PARTS];
        return VDIT_OK;
    } catch (...) {
        return VDIT_ERR_INVALID_ARG;
    }
}

vdit_status vdit_fp8_quantize(const void* q, const void* k, const void* v, int B, int H, int Sq, int Skv, int D,
                              void* workspace, size_t workspace_bytes, void* stream) {
    try {
        size_t off[VDIT_FP8_NUM_PARTS + 1];
        const Shape s{B, H, Sq, Skv, D, VDIT_MASK_FULL, 0};
        const vdit_status st = fp8_check(s, false, 1.0f, workspace, workspace_bytes, off);
        if (st != VDIT_OK || B == 0 || H == 0 || Sq == 0) return st;
        return fp8_quantize_impl(q, k, v, s, workspace, off, static_cast<cudaStream_t>(stream));
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_fwd_fp8_quantized(void* o, float* lse, int B, int H, int Sq, int Skv, int D, float scale,
                                        int mask_kind, int chunk_tokens, const void* workspace,
                                        size_t workspace_bytes, void* stream) {
    try {
        size_t off[VDIT_FP8_NUM_PARTS + 1];
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        void* ws = const_cast<void*>(workspace);
        const vdit_status st = fp8_check(s, true, scale, ws, workspace_bytes, off);
        if (st != VDIT_OK || B == 0 || H == 0 || Sq == 0) return st;
        return fp8_attention_impl(o, lse, s, scale, ws, off, static_cast<cudaStream_t>(stream), false);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                              int Sq, int Skv, int D, float scale, int mask_kind, int chunk_tokens, void* workspace,
                              size_t workspace_bytes, void* stream) {
    try {
        size_t off[VDIT_FP8_NUM_PARTS + 1];
        const Shape s{B, H, Sq, Skv, D, mask_kind, chunk_tokens};
        vdit_status st = fp8_check(s, true, scale, workspace, workspace_bytes, off);
        if (st != VDIT_OK || B == 0 || H == 0 || Sq == 0) return st;
        if (o == nullptr) return VDIT_ERR_INVALID_ARG;
        if (!aligned16(o) || !aligned16(lse)) return VDIT_ERR_MISALIGNED;
        const size_t ob = size_t(B) * size_t(Sq) * size_t(H) * 256;
        const size_t kb = size_t(B) * size_t(Skv) * size_t(H) * 256;
        if (overlaps(o, ob, q, ob) || overlaps(o, ob, k, kb) || overlaps(o, ob, v, kb)) return VDIT_ERR_INVALID_ARG;
        st = fp8_quantize_impl(q, k, v, s, workspace, off, static_cast<cudaStream_t>(stream));
        if (st != VDIT_OK) return st;
        return fp8_attention_impl(o, lse, s, scale, workspace, off, static_cast<cudaStream_t>(stream), true);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_vsmooth_group_plan(int B, int H, int S, int D, int C, size_t* workspace_bytes) {
    try {
        if (workspace_bytes == nullptr || B < 0 || H < 0 || S < 0 || D < 1) return VDIT_ERR_INVALID_ARG;
        if (D != 128) return VDIT_ERR_UNSUPPORTED;
        if (C < 1 || C > vdit::kGroupMaxClusters) return VDIT_ERR_INVALID_ARG;
        const size_t bhc = size_t(B) * size_t(H) * size_t(C);
        *workspace_bytes = round_up(bhc * 128 * 4, kWorkspaceAlign) + bhc * 4;
        return VDIT_OK;
    } catch (...) {
        return VDIT_ERR_INVALID_ARG;
    }
}

vdit_status vdit_vsmooth_group(const void* v, float* centroids, int32_t* labels, int32_t* perm, int B, int H, int S,
                               int D, int C, int iters, void* workspace, size_t workspace_bytes, void* stream) {
    try {
        size_t need = 0;
        vdit_status st = vdit_vsmooth_group_plan(B, H, S, D, C, &need);
        if (st != VDIT_OK) return st;
        if (iters < 0 || iters > 1000) return VDIT_ERR_INVALID_ARG;
        if (B > 65535 || H > 65535) return VDIT_ERR_INVALID_ARG;
        if (B == 0 || H == 0 || S == 0) return VDIT_OK;
        if (v == nullptr || centroids == nullptr || labels == nullptr || perm == nullptr)
            return VDIT_ERR_INVALID_ARG;
        if (!aligned16(v) || !aligned16(centroids) || (reinterpret_cast<uintptr_t>(labels) & 3) ||
            (reinterpret_cast<uintptr_t>(perm) & 3))
            return VDIT_ERR_MISALIGNED;
        if (iters > 0) {
            if (workspace == nullptr || workspace_bytes < need) return VDIT_ERR_WORKSPACE;
            if ((reinterpret_cast<uintptr_t>(workspace) & (kWorkspaceAlign - 1)) != 0) return VDIT_ERR_MISALIGNED;
        }
        const size_t bh = size_t(B) * size_t(H);
        const size_t vb = bh * size_t(S) * 256, cb = bh * size_t(C) * 512, lb = bh * size_t(S) * 4;
        if (overlaps(centroids, cb, v, vb) || overlaps(labels, lb, v, vb) || overlaps(perm, lb, v, vb) ||
            overlaps(labels, lb, perm, lb) || overlaps(labels, lb, centroids, cb) ||
            overlaps(perm, lb, centroids, cb) ||
            (iters > 0 && (overlaps(workspace, need, v, vb) || overlaps(workspace, need, centroids, cb) ||
                           overlaps(workspace, need, labels, lb) || overlaps(workspace, need, perm, lb))))
            return VDIT_ERR_INVALID_ARG;
        int dev = 0;
        st = ensure_device(&dev);
        if (st != VDIT_OK) return st;
        cudaStream_t sm = static_cast<cudaStream_t>(stream);
        const __nv_bfloat16* vv = static_cast<const __nv_bfloat16*>(v);
        float* sums = static_cast<float*>(workspace);
        int32_t* counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                                     round_up(bh * size_t(C) * 512, kWorkspaceAlign));
        const dim3 grid((S + vdit::kGroupTokens - 1) / vdit::kGroupTokens, H, B);
        for (int it = 0; it < iters; ++it) {
            vdit::group_assign_kernel<<<grid, vdit::kGroupTokens, 0, sm>>>(vv, centroids, labels, H, S, C);
            if (cudaMemsetAsync(workspace, 0, need, sm) != cudaSuccess) return VDIT_ERR_CUDA;
            vdit::group_accumulate_kernel<<<grid, 128, 0, sm>>>(vv, labels, sums, counts, H, S, C);
            vdit::group_finalize_kernel<<<unsigned(bh * size_t(C)), 128, 0, sm>>>(sums, counts, centroids, C);
        }
        vdit::group_assign_kernel<<<grid, vdit::kGroupTokens, 0, sm>>>(vv, centroids, labels, H, S, C);
        vdit::group_sort_kernel<<<unsigned(bh), vdit::kSortThreads, 0, sm>>>(labels, perm, S, C);
        return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_permute_kv(const void* k, const void* v, const int32_t* perm, void* k_out, void* v_out, int B,
                            int H, int S, int D, void* stream) {
    try {
        if (B < 0 || H < 0 || S < 0 || D < 1) return VDIT_ERR_INVALID_ARG;
        if (D != 128) return VDIT_ERR_UNSUPPORTED;
        if (B == 0 || H == 0 || S == 0) return VDIT_OK;
        if (k == nullptr || v == nullptr || perm == nullptr || k_out == nullptr || v_out == nullptr)
            return VDIT_ERR_INVALID_ARG;
        if (!aligned16(k) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out) ||
            (reinterpret_cast<uintptr_t>(perm) & 3))
            return VDIT_ERR_MISALIGNED;
        const size_t tb = size_t(B) * size_t(S) * size_t(H) * 256, pb = size_t(B) * size_t(H) * size_t(S) * 4;
        const void* ins[3] = {k, v, perm};
        const size_t in_b[3] = {tb, tb, pb};
        for (int i = 0; i < 3; ++i)
            if (overlaps(k_out, tb, ins[i], in_b[i]) || overlaps(v_out, tb, ins[i], in_b[i])) return VDIT_ERR_INVALID_ARG;
        if (overlaps(k_out, tb, v_out, tb)) return VDIT_ERR_INVALID_ARG;
        int dev = 0;
        const vdit_status st = ensure_device(&dev);
        if (st != VDIT_OK) return st;
        const long long rows = (long long)B * H * S;
        const long long blocks = (rows * 16 + 255) / 256;
        if (blocks > 0x7fffffffLL) return VDIT_ERR_INVALID_ARG;
        vdit::permute_rows_kernel<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
            static_cast<const uint4*>(k), static_cast<const uint4*>(v), perm, static_cast<uint4*>(k_out),
            static_cast<uint4*>(v_out), H, S, rows);
        return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA;
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_testing_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                  int Sq, int Skv, int D, float scale, int mask_kind, int chunk_tokens,
                                  int fault, unsigned long long wait_timeout_ns, void* stream) {
    try {
        if (fault != VDIT_TESTING_NO_FAULT && fault != VDIT_TESTING_WITHHOLD_KV) return VDIT_ERR_INVALID_ARG;
        if (wait_timeout_ns < 1000000ull || wait_timeout_ns > 10000000000ull) return VDIT_ERR_INVALID_ARG;
        const int flags = fault == VDIT_TESTING_WITHHOLD_KV ? vdit::kDebugWithholdKV : 0;
        return fwd_impl(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, nullptr, 0, stream, flags,
                        wait_timeout_ns);
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_testing_cross_cta_spans(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                         int H, int Sq, int Skv, int D, float scale, unsigned long long* spans,
                                         int max_ctas, int* grid_ctas, void* stream) {
    try {
        if (spans == nullptr || max_ctas < 1 || grid_ctas == nullptr) return VDIT_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(spans) & 7u) != 0) return VDIT_ERR_MISALIGNED;
        *grid_ctas = 0;
        const Shape s{B, H, Sq, Skv, D, VDIT_MASK_CROSS, 0};
        vdit_status st = check_shape(s, true, scale);
        if (st != VDIT_OK) return st;
        if (B == 0 || H == 0 || Sq == 0) return VDIT_OK;
        int dev = 0;
        const DeviceState* ds = nullptr;
        st = ensure_device(&dev, &ds);
        if (st != VDIT_OK) return st;
        const long long items = static_cast<long long>(cross_tiles(Sq)) * H * B;
        const int grid = static_cast<int>(items < ds->cross_grid ? items : ds->cross_grid);
        if (grid > max_ctas) return VDIT_ERR_INVALID_ARG;  // every CTA records its span
        st = fwd_impl(q, k, v, o, lse, B, H, Sq, Skv, D, scale, VDIT_MASK_CROSS, 0, nullptr, 0, stream, 0,
                      kDefaultWaitTimeoutNs, nullptr, false, spans, max_ctas);
        if (st == VDIT_OK) *grid_ctas = grid;
        return st;
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_merge(void* o_acc, float* lse_acc, const void* o_part, const float* lse_part, int B, int H,
                            int S, int D, void* stream) {
    try {
        return merge_impl(static_cast<__nv_bfloat16*>(o_acc), lse_acc, o_part, lse_part, nullptr, B, H, S, D,
                          static_cast<cudaStream_t>(stream));
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_attn_merge_f32(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                void* o_out, int B, int H, int S, int D, void* stream) {
    try {
        return merge_impl(o_acc, lse_acc, o_part, lse_part, static_cast<__nv_bfloat16*>(o_out), B, H, S, D,
                          static_cast<cudaStream_t>(stream));
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

vdit_status vdit_get_device_status(void* stream, uint32_t* detail) {
    try {
        if (detail != nullptr) *detail = 0;
        if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return VDIT_ERR_CUDA;
        uint32_t word = 0;
        if (cudaMemcpyFromSymbol(&word, vdit::g_status_word, sizeof(word)) != cudaSuccess) return VDIT_ERR_CUDA;
        if (word != 0) {
            const uint32_t zero = 0;
            if (cudaMemcpyToSymbol(vdit::g_status_word, &zero, sizeof(zero)) != cudaSuccess) return VDIT_ERR_CUDA;
        }
        if (detail != nullptr) *detail = word;
        return (word & vdit::kStatusTimeout) ? VDIT_ERR_TIMEOUT : VDIT_OK;
    } catch (...) {
        return VDIT_ERR_CUDA;
    }
}

}  // extern "C"
