"""ctypes binding of libvdit_attn.so: the C ABI of include/*.h, same names.

Argument marshalling only -- every step of the attention runs in the CUDA
library.  Functions accept raw integers (device addresses, a cudaStream_t
value) or torch tensors / streams, which are turned into those integers.
If the library has not been built, loading raises ``ImportError``; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvdit_attn.so")

VDIT_MASK_FULL = 0
VDIT_MASK_BLOCK_CAUSAL = 1
VDIT_MASK_CROSS = 2
VDIT_MASK_BLOCK_SPARSE = 3
SPARSE_BLOCK = 128

VDIT_OK = 0
VDIT_ERR_INVALID_ARG = 1
VDIT_ERR_UNSUPPORTED = 2
VDIT_ERR_MISALIGNED = 3
VDIT_ERR_CUDA = 4
VDIT_ERR_TIMEOUT = 5
VDIT_ERR_WORKSPACE = 6

VDIT_TESTING_NO_FAULT = 0
VDIT_TESTING_WITHHOLD_KV = 1

# every entry point declared in include/*.h
EXPORTS = (
    "vdit_attn_plan",
    "vdit_attn_fwd",
    "vdit_attn_fwd_ws",
    "vdit_attn_fwd_block_sparse",
    "vdit_attn_merge",
    "vdit_attn_merge_f32",
    "vdit_attn_fwd_qknorm",
    "vdit_attn_qknorm_plan",
    "vdit_qk_rms_norm",
    "vdit_attn_fwd_qknorm_noalloc",
    "vdit_fp8_layout",
    "vdit_attn_fp8_plan",
    "vdit_fp8_quantize",
    "vdit_attn_fwd_fp8_quantized",
    "vdit_attn_fwd_fp8",
    "vdit_vsmooth_group_plan",
    "vdit_vsmooth_group",
    "vdit_permute_kv",
    "vdit_get_device_status",
    "vdit_status_string",
    "vdit_abi_version",
    "vdit_testing_attn_fwd",
    "vdit_testing_cross_cta_spans",
)

_lock = threading.Lock()
_lib = None


class VditError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__(f"{what}: {vdit_status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load (once) and return the library handle."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing; build it with "
                    "`python -m video_diffusion_transformer_attention_b200.build`")
            h = ctypes.CDLL(LIB_PATH)
            c_int, c_float, c_size, vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
            h.vdit_attn_plan.restype = c_int
            h.vdit_attn_plan.argtypes = [c_int] * 7 + [ctypes.POINTER(c_size), ctypes.POINTER(c_int)]
            fwd_args = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int]
            h.vdit_attn_fwd.restype = c_int
            h.vdit_attn_fwd.argtypes = fwd_args + [vp]
            h.vdit_attn_fwd_ws.restype = c_int
            h.vdit_attn_fwd_ws.argtypes = fwd_args + [vp, c_size, vp]
            h.vdit_attn_fwd_block_sparse.restype = c_int
            h.vdit_attn_fwd_block_sparse.argtypes = [vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int,
                                                     c_float, vp]
            h.vdit_attn_fwd_qknorm.restype = c_int
            h.vdit_attn_fwd_qknorm.argtypes = [vp, vp, vp, vp, vp, vp, vp, c_float, c_int, c_int, c_int, c_int,
                                               c_int, c_float, c_int, c_int, vp, c_size, vp]
            h.vdit_attn_qknorm_plan.restype = c_int
            h.vdit_attn_qknorm_plan.argtypes = [c_int] * 7 + [ctypes.POINTER(c_size)]
            h.vdit_attn_fwd_qknorm_noalloc.restype = c_int
            h.vdit_attn_fwd_qknorm_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, c_float, c_int, c_int, c_int,
                                                       c_int, c_int, c_float, c_int, c_int, vp]
            h.vdit_fp8_layout.restype = c_int
            h.vdit_fp8_layout.argtypes = [c_int] * 5 + [ctypes.POINTER(c_size)]
            h.vdit_attn_fp8_plan.restype = c_int
            h.vdit_attn_fp8_plan.argtypes = [c_int] * 7 + [ctypes.POINTER(c_size)]
            h.vdit_fp8_quantize.restype = c_int
            h.vdit_fp8_quantize.argtypes = [vp, vp, vp] + [c_int] * 5 + [vp, c_size, vp]
            h.vdit_attn_fwd_fp8_quantized.restype = c_int
            h.vdit_attn_fwd_fp8_quantized.argtypes = [vp, vp] + [c_int] * 5 + [c_float, c_int, c_int, vp, c_size, vp]
            h.vdit_attn_fwd_fp8.restype = c_int
            h.vdit_attn_fwd_fp8.argtypes = fwd_args + [vp, c_size, vp]
            h.vdit_vsmooth_group_plan.restype = c_int
            h.vdit_vsmooth_group_plan.argtypes = [c_int] * 5 + [ctypes.POINTER(c_size)]
            h.vdit_vsmooth_group.restype = c_int
            h.vdit_vsmooth_group.argtypes = [vp, vp, vp, vp] + [c_int] * 6 + [vp, c_size, vp]
            h.vdit_permute_kv.restype = c_int
            h.vdit_permute_kv.argtypes = [vp] * 5 + [c_int] * 4 + [vp]
            h.vdit_qk_rms_norm.restype = c_int
            h.vdit_qk_rms_norm.argtypes = [vp, vp, vp, vp, vp, vp, c_float, c_int, c_int, c_int, c_int, c_int, vp]
            h.vdit_attn_merge.restype = c_int
            h.vdit_attn_merge.argtypes = [vp, vp, vp, vp, c_int, c_int, c_int, c_int, vp]
            h.vdit_attn_merge_f32.restype = c_int
            h.vdit_attn_merge_f32.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, vp]
            h.vdit_testing_attn_fwd.restype = c_int
            h.vdit_testing_attn_fwd.argtypes = fwd_args + [c_int, ctypes.c_ulonglong, vp]
            h.vdit_testing_cross_cta_spans.restype = c_int
            h.vdit_testing_cross_cta_spans.argtypes = [vp] * 5 + [c_int] * 5 + [c_float, vp, c_int,
                                                                              ctypes.POINTER(c_int), vp]
            h.vdit_get_device_status.restype = c_int
            h.vdit_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
            h.vdit_status_string.restype = ctypes.c_char_p
            h.vdit_status_string.argtypes = [c_int]
            h.vdit_abi_version.restype = c_int
            h.vdit_abi_version.argtypes = []
            _lib = h
    return _lib


def _addr(x) -> int | None:
    """A device address from a tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int | None:
    """A cudaStream_t value from a torch stream, an int, or None (current stream)."""
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def vdit_status_string(status: int) -> str:
    return lib().vdit_status_string(int(status)).decode()


def vdit_abi_version() -> int:
    return int(lib().vdit_abi_version())


def vdit_attn_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens):
    """Returns (workspace_bytes, grid_ctas); raises VditError on a bad shape."""
    ws = ctypes.c_size_t(0)
    grid = ctypes.c_int(0)
    st = lib().vdit_attn_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens, ctypes.byref(ws), ctypes.byref(grid))
    if st != VDIT_OK:
        raise VditError(st, "vdit_attn_plan")
    return int(ws.value), int(grid.value)


def vdit_attn_fwd(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, stream=None,
                  check=True) -> int:
    """Launch the forward; returns the status (raises VditError if check and not OK)."""
    st = lib().vdit_attn_fwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), B, H, Sq, Skv, D,
                             float(scale), mask_kind, chunk_tokens, _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd")
    return st


def vdit_attn_fwd_ws(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, workspace,
                     workspace_bytes, stream=None, check=True) -> int:
    st = lib().vdit_attn_fwd_ws(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), B, H, Sq, Skv, D,
                                float(scale), mask_kind, chunk_tokens, _addr(workspace),
                                int(workspace_bytes), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_ws")
    return st


def vdit_attn_fwd_block_sparse(q, k, v, o, lse, block_mask, B, H, Sq, Skv, D, scale, stream=None,
                               check=True) -> int:
    """Block-sparse forward; block_mask is a device uint8 [B, H, ceil(Sq/128), ceil(Skv/128)]."""
    st = lib().vdit_attn_fwd_block_sparse(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), _addr(block_mask),
                                          B, H, Sq, Skv, D, float(scale), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_block_sparse")
    return st


def vdit_qk_rms_norm(q, k, q_out, k_out, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, stream=None,
                     check=True) -> int:
    """Per-head RMS norm of q and k into q_out, k_out (see include/vdit_attn.h)."""
    st = lib().vdit_qk_rms_norm(_addr(q), _addr(k), _addr(q_out), _addr(k_out), _addr(q_norm_weight),
                                _addr(k_norm_weight), float(eps), B, H, Sq, Skv, D, _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_qk_rms_norm")
    return st


def vdit_attn_qknorm_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens):
    """Returns (status, workspace bytes) for vdit_attn_fwd_qknorm."""
    ws = ctypes.c_size_t(0)
    st = lib().vdit_attn_qknorm_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens, ctypes.byref(ws))
    return int(st), int(ws.value)


def vdit_attn_fwd_qknorm(q, k, v, o, lse, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, scale, mask_kind,
                         chunk_tokens, workspace, workspace_bytes, stream=None, check=True) -> int:
    """Forward on raw Q/K: per-head RMS norm into the workspace, then attention (see include/vdit_attn.h)."""
    st = lib().vdit_attn_fwd_qknorm(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), _addr(q_norm_weight),
                                    _addr(k_norm_weight), float(eps), B, H, Sq, Skv, D, float(scale), mask_kind,
                                    chunk_tokens, _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_qknorm")
    return st


FP8_PARTS = ("q", "k", "vt", "mu_img", "q_scale", "k_scale", "v_scale", "v_amax", "mu")


def vdit_fp8_layout(B, H, Sq, Skv, D):
    """Returns (status, {part: byte offset}, total bytes) of the 8-bit path's workspace."""
    off = (ctypes.c_size_t * (len(FP8_PARTS) + 1))()
    st = lib().vdit_fp8_layout(B, H, Sq, Skv, D, off)
    return int(st), dict(zip(FP8_PARTS, [int(x) for x in off[:-1]])), int(off[len(FP8_PARTS)])


def vdit_attn_fp8_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens):
    """Returns (status, workspace bytes) of the 8-bit path."""
    ws = ctypes.c_size_t(0)
    st = lib().vdit_attn_fp8_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens, ctypes.byref(ws))
    return int(st), int(ws.value)


def vdit_fp8_quantize(q, k, v, B, H, Sq, Skv, D, workspace, workspace_bytes, stream=None, check=True) -> int:
    st = lib().vdit_fp8_quantize(_addr(q), _addr(k), _addr(v), B, H, Sq, Skv, D, _addr(workspace),
                                 int(workspace_bytes), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_fp8_quantize")
    return st


def vdit_attn_fwd_fp8_quantized(o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, workspace,
                                workspace_bytes, stream=None, check=True) -> int:
    st = lib().vdit_attn_fwd_fp8_quantized(_addr(o), _addr(lse), B, H, Sq, Skv, D, float(scale), mask_kind,
                                           chunk_tokens, _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_fp8_quantized")
    return st


def vdit_attn_fwd_fp8(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, workspace,
                      workspace_bytes, stream=None, check=True) -> int:
    st = lib().vdit_attn_fwd_fp8(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), B, H, Sq, Skv, D,
                                 float(scale), mask_kind, chunk_tokens, _addr(workspace), int(workspace_bytes),
                                 _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_fp8")
    return st


def attention_fp8(q, k, v, scale=None, mask_kind=VDIT_MASK_FULL, chunk_tokens=0, workspace=None, stream=None):
    """Convenience wrapper over vdit_attn_fwd_fp8 for CUDA bf16 [B, S, H, 128] tensors.

    workspace: a CUDA uint8 tensor of at least vdit_attn_fp8_plan bytes, or None
    to allocate one with torch.  Returns (o, lse, workspace)."""
    import torch
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    st, need = vdit_attn_fp8_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens)
    if st != VDIT_OK:
        raise VditError(st, "vdit_attn_fp8_plan")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    vdit_attn_fwd_fp8(q, k, v, out, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, workspace,
                      workspace.numel(), stream)
    return out, lse, workspace


def vdit_vsmooth_group_plan(B, H, S, D, C):
    ws = ctypes.c_size_t(0)
    st = lib().vdit_vsmooth_group_plan(B, H, S, D, C, ctypes.byref(ws))
    return int(st), int(ws.value)


def vdit_vsmooth_group(v, centroids, labels, perm, B, H, S, D, C, iters, workspace, workspace_bytes, stream=None,
                       check=True) -> int:
    st = lib().vdit_vsmooth_group(_addr(v), _addr(centroids), _addr(labels), _addr(perm), B, H, S, D, C, iters,
                                  _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_vsmooth_group")
    return st


def vdit_permute_kv(k, v, perm, k_out, v_out, B, H, S, D, stream=None, check=True) -> int:
    st = lib().vdit_permute_kv(_addr(k), _addr(v), _addr(perm), _addr(k_out), _addr(v_out), B, H, S, D,
                               _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_permute_kv")
    return st


def vsmooth_group(v, centroids, iters=4, stream=None):
    """Group step on CUDA tensors: v bf16 [B, S, H, 128], centroids fp32 [B, H, C, 128] (updated in place).
    Returns (labels, perm), int32 [B, H, S]."""
    import torch
    B, S, H, D = v.shape
    C = centroids.shape[2]
    st, need = vdit_vsmooth_group_plan(B, H, S, D, C)
    if st != VDIT_OK:
        raise VditError(st, "vdit_vsmooth_group_plan")
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=v.device)
    labels = torch.empty((B, H, S), dtype=torch.int32, device=v.device)
    perm = torch.empty((B, H, S), dtype=torch.int32, device=v.device)
    vdit_vsmooth_group(v, centroids, labels, perm, B, H, S, D, C, iters, ws, ws.numel(), stream)
    return labels, perm


def permute_kv(k, v, perm, stream=None):
    """K and V gathered per head by perm (CUDA bf16 [B, S, H, 128], perm int32 [B, H, S])."""
    import torch
    B, S, H, D = k.shape
    k_out, v_out = torch.empty_like(k), torch.empty_like(v)
    vdit_permute_kv(k, v, perm, k_out, v_out, B, H, S, D, stream)
    return k_out, v_out


NOALLOC_SCRATCH_BYTES = 64 << 20  # VDIT_NOALLOC_SCRATCH_BYTES in include/vdit_attn.h


def vdit_attn_fwd_qknorm_noalloc(q, k, v, o, lse, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, scale,
                                 mask_kind, chunk_tokens, stream=None, check=True) -> int:
    """vdit_attn_fwd_qknorm without a workspace argument: the library's fixed device scratch holds the
    normalised Q and K, so nothing is allocated (see include/vdit_attn.h)."""
    st = lib().vdit_attn_fwd_qknorm_noalloc(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                            _addr(q_norm_weight), _addr(k_norm_weight), float(eps), B, H, Sq, Skv,
                                            D, float(scale), mask_kind, chunk_tokens, _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_fwd_qknorm_noalloc")
    return st


def vdit_attn_merge(o_acc, lse_acc, o_part, lse_part, B, H, S, D, stream=None, check=True) -> int:
    """Fold (o_part, lse_part) into (o_acc, lse_acc) in place (see include/vdit_attn.h)."""
    st = lib().vdit_attn_merge(_addr(o_acc), _addr(lse_acc), _addr(o_part), _addr(lse_part), B, H, S, D,
                               _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_merge")
    return st


def vdit_attn_merge_f32(o_acc, lse_acc, o_part, lse_part, o_out, B, H, S, D, stream=None, check=True) -> int:
    """Fold (o_part, lse_part) into an fp32 running (o_acc, lse_acc); o_out (bf16, optional) also receives the
    merged O rounded to bf16 (see include/vdit_attn.h)."""
    st = lib().vdit_attn_merge_f32(_addr(o_acc), _addr(lse_acc), _addr(o_part), _addr(lse_part), _addr(o_out),
                                   B, H, S, D, _stream(stream))
    if check and st != VDIT_OK:
        raise VditError(st, "vdit_attn_merge_f32")
    return st


def vdit_testing_attn_fwd(q, k, v, o, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, fault,
                          wait_timeout_ns, stream=None) -> int:
    """Test-only forward with an injected fault (see include/vdit_attn_testing.h); returns the status."""
    return int(lib().vdit_testing_attn_fwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), B, H, Sq, Skv, D,
                                           float(scale), mask_kind, chunk_tokens, int(fault),
                                           int(wait_timeout_ns), _stream(stream)))


def vdit_testing_cross_cta_spans(q, k, v, o, lse, B, H, Sq, Skv, D, scale, spans, max_ctas, stream=None):
    """Test-only cross-attention call recording each CTA's (smid, start ns, end ns) into spans
    (see include/vdit_attn_testing.h); returns (status, CTAs launched)."""
    grid = ctypes.c_int(0)
    st = lib().vdit_testing_cross_cta_spans(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), B, H, Sq, Skv, D,
                                            float(scale), _addr(spans), int(max_ctas), ctypes.byref(grid),
                                            _stream(stream))
    return int(st), int(grid.value)


def vdit_get_device_status(stream=None):
    """Returns (status, raw error word); synchronises the stream."""
    word = ctypes.c_uint32(0)
    st = lib().vdit_get_device_status(_stream(stream), ctypes.byref(word))
    return int(st), int(word.value)


def attention(q, k, v, scale=None, mask_kind=VDIT_MASK_FULL, chunk_tokens=0, out=None, lse=None,
              return_lse=True, stream=None):
    """Convenience wrapper over vdit_attn_fwd for CUDA bf16 tensors in [B, S, H, D].

    Output buffers are allocated with torch when not given (torch only serves
    as the device-memory allocator here).  Returns (o, lse) or o.
    """
    import torch
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    for t in (q, k, v, out):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("q, k, v, out must be contiguous CUDA bf16 tensors")
    vdit_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, mask_kind, chunk_tokens, stream)
    return (out, lse) if return_lse else out


def attention_block_sparse(q, k, v, block_mask, scale=None, out=None, lse=None, stream=None):
    """Convenience wrapper over vdit_attn_fwd_block_sparse (CUDA bf16 [B, S, H, D] tensors,
    block_mask a CUDA uint8 tensor [B, H, ceil(Sq/128), ceil(Skv/128)]).  Returns (o, lse)."""
    import torch
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    nqb, nkb = -(-Sq // SPARSE_BLOCK), -(-Skv // SPARSE_BLOCK)
    if block_mask.dtype != torch.uint8 or tuple(block_mask.shape) != (B, H, nqb, nkb) or not block_mask.is_cuda \
            or not block_mask.is_contiguous():
        raise ValueError(f"block_mask must be a contiguous CUDA uint8 tensor [B, H, {nqb}, {nkb}]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    vdit_attn_fwd_block_sparse(q, k, v, out, lse, block_mask, B, H, Sq, Skv, D, scale, stream)
    return out, lse


def attention_qknorm(q, k, v, q_norm_weight=None, k_norm_weight=None, eps=1e-6, scale=None,
                     mask_kind=VDIT_MASK_FULL, chunk_tokens=0, workspace=None, stream=None):
    """Convenience wrapper over vdit_attn_fwd_qknorm (raw CUDA bf16 q, k; fp32 [H, D] weights or None).

    workspace: a CUDA uint8 tensor of at least vdit_attn_qknorm_plan bytes, or
    None to allocate one with torch.  Returns (o, lse)."""
    import torch
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    st, need = vdit_attn_qknorm_plan(B, H, Sq, Skv, D, mask_kind, chunk_tokens)
    if st != VDIT_OK:
        raise VditError(st, "vdit_attn_qknorm_plan")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    vdit_attn_fwd_qknorm(q, k, v, out, lse, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, scale,
                         mask_kind, chunk_tokens, workspace, workspace.numel(), stream)
    return out, lse


def qk_rms_norm(q, k, q_norm_weight=None, k_norm_weight=None, eps=1e-6, inplace=False, stream=None):
    """Convenience wrapper over vdit_qk_rms_norm for CUDA bf16 [B, S, H, 128] q and k. Returns (q_n, k_n)."""
    import torch
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    q_out, k_out = (q, k) if inplace else (torch.empty_like(q), torch.empty_like(k))
    vdit_qk_rms_norm(q, k, q_out, k_out, q_norm_weight, k_norm_weight, eps, B, H, Sq, Skv, D, stream)
    return q_out, k_out
