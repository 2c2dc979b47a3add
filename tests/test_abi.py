"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/vdit_attn.h, and rejects bad arguments on the host before
touching the device."""
import os
import re

import pytest

from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200.build import build

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build()
    return vb.lib()


def declared_functions():
    names = set()
    for f in sorted(os.listdir(INCLUDE)):
        if f.endswith(".h"):
            text = re.sub(r"/\*.*?\*/", "", open(os.path.join(INCLUDE, f)).read(), flags=re.S)
            names.update(re.findall(r"\b(vdit_\w+)\s*\(", text))
    return sorted(names)


def test_header_and_binding_agree():
    assert declared_functions() == sorted(vb.EXPORTS)


def test_library_exports_every_declared_symbol():
    h = vb.lib()
    for name in declared_functions():
        assert hasattr(h, name), name


def test_abi_version_and_status_strings():
    assert vb.vdit_abi_version() == 1
    assert vb.vdit_status_string(vb.VDIT_OK) == "VDIT_OK"
    assert vb.vdit_status_string(vb.VDIT_ERR_TIMEOUT) == "VDIT_ERR_TIMEOUT"
    assert vb.vdit_status_string(999) == "VDIT_ERR_UNKNOWN"


def test_plan_reports_grid_and_zero_workspace():
    ws, grid = vb.vdit_attn_plan(1, 40, 75600, 75600, 128, vb.VDIT_MASK_FULL, 0)
    assert ws == 0 and grid == 296 * 40
    ws, grid = vb.vdit_attn_plan(2, 3, 300, 300, 128, vb.VDIT_MASK_BLOCK_CAUSAL, 100)
    assert grid == 2 * 3 * 2
    # cross attention: one 128-row query tile per CTA
    ws, grid = vb.vdit_attn_plan(1, 40, 75600, 512, 128, vb.VDIT_MASK_CROSS, 0)
    assert ws == 0 and grid == 591 * 40
    assert vb.vdit_attn_plan(1, 1, 0, 5, 128, 0, 0) == (0, 0)


@pytest.mark.parametrize("args,status", [
    ((1, 1, 16, 16, 64, 0, 0), vb.VDIT_ERR_UNSUPPORTED),
    ((1, 1, 16, 0, 128, 0, 0), vb.VDIT_ERR_INVALID_ARG),
    ((1, 1, 16, 16, 128, 4, 0), vb.VDIT_ERR_INVALID_ARG),
    ((1, 1, 16, 262145, 128, 3, 0), vb.VDIT_ERR_INVALID_ARG),
    ((1, 1, 16, 16, 128, 1, 0), vb.VDIT_ERR_INVALID_ARG),
    ((1, 1, 16, 32, 128, 1, 8), vb.VDIT_ERR_INVALID_ARG),
    ((-1, 1, 16, 16, 128, 0, 0), vb.VDIT_ERR_INVALID_ARG),
    ((1, 70000, 16, 16, 128, 0, 0), vb.VDIT_ERR_INVALID_ARG),
])
def test_plan_rejects_bad_shapes(args, status):
    with pytest.raises(vb.VditError) as e:
        vb.vdit_attn_plan(*args)
    assert e.value.status == status


A = 1 << 20  # a fake, 16-byte aligned "device" address: never dereferenced


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), vb.VDIT_ERR_INVALID_ARG),
    (dict(o=None), vb.VDIT_ERR_INVALID_ARG),
    (dict(q=A + 2), vb.VDIT_ERR_MISALIGNED),
    (dict(lse=A * 9 + 4), vb.VDIT_ERR_MISALIGNED),
    (dict(scale=0.0), vb.VDIT_ERR_INVALID_ARG),
    (dict(scale=float("nan")), vb.VDIT_ERR_INVALID_ARG),
    (dict(scale=-1.0), vb.VDIT_ERR_INVALID_ARG),
    (dict(D=96), vb.VDIT_ERR_UNSUPPORTED),
    (dict(o=A), vb.VDIT_ERR_INVALID_ARG),  # output aliases q
    (dict(mask_kind=1, chunk_tokens=0), vb.VDIT_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_arguments_before_any_launch(kw, status):
    args = dict(q=A, k=A * 3, v=A * 5, o=A * 7, lse=A * 9, B=1, H=2, Sq=64, Skv=64, D=128,
                scale=0.1, mask_kind=0, chunk_tokens=0)
    args.update(kw)
    st = vb.vdit_attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                          args["Sq"], args["Skv"], args["D"], args["scale"], args["mask_kind"],
                          args["chunk_tokens"], stream=0, check=False)
    assert st == status


def test_testing_entry_point_rejects_bad_fault_or_limit():
    args = (A, A * 3, A * 5, A * 7, A * 9, 1, 2, 64, 64, 128, 0.1, 0, 0)
    assert vb.vdit_testing_attn_fwd(*args, 7, 10 ** 8, stream=0) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_testing_attn_fwd(*args, vb.VDIT_TESTING_WITHHOLD_KV, 10, stream=0) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_testing_attn_fwd(*args, vb.VDIT_TESTING_WITHHOLD_KV, 10 ** 11, stream=0) == vb.VDIT_ERR_INVALID_ARG


def test_block_sparse_needs_its_entry_point_and_a_mask():
    assert vb.vdit_attn_plan(1, 2, 300, 262144, 128, vb.VDIT_MASK_BLOCK_SPARSE, 0)[1] == 4
    args = (A, A * 3, A * 5, A * 7, A * 9)
    # the plain forward does not take the block-sparse mask kind
    assert vb.vdit_attn_fwd(*args, 1, 2, 64, 64, 128, 0.1, vb.VDIT_MASK_BLOCK_SPARSE, 0, stream=0,
                            check=False) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_fwd_block_sparse(*args, None, 1, 2, 64, 64, 128, 0.1, stream=0,
                                         check=False) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_fwd_block_sparse(*args, A * 11, 1, 2, 64, 300000, 128, 0.1, stream=0,
                                         check=False) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_fwd_block_sparse(*args, A * 11, 1, 2, 64, 64, 96, 0.1, stream=0,
                                         check=False) == vb.VDIT_ERR_UNSUPPORTED


def test_qknorm_entry_point_argument_checks():
    args = (A, A * 3, A * 5, A * 7, A * 9)
    ok_shape = (1, 2, 64, 64, 128, 0.1)
    ws = A * 64
    st, need = vb.vdit_attn_qknorm_plan(1, 2, 64, 64, 128, 0, 0)
    assert st == vb.VDIT_OK and need == 64 * 2 * 128 * 2 * 2   # normalised Q and K, Q rounded up to 256 B
    assert vb.vdit_attn_qknorm_plan(1, 2, 64, 64, 128, vb.VDIT_MASK_BLOCK_SPARSE, 0)[0] == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_qknorm_plan(1, 2, 64, 64, 64, 0, 0)[0] == vb.VDIT_ERR_UNSUPPORTED

    def call(*extra, eps=1e-6, qw=None, mask=0, workspace=ws, nbytes=need):
        return vb.vdit_attn_fwd_qknorm(*args, qw, None, eps, *ok_shape, mask, 0, workspace, nbytes, stream=0,
                                       check=False)
    assert call(eps=0.0) == vb.VDIT_ERR_INVALID_ARG                     # eps must be > 0
    assert call(eps=float("nan")) == vb.VDIT_ERR_INVALID_ARG
    assert call(mask=vb.VDIT_MASK_BLOCK_SPARSE) == vb.VDIT_ERR_INVALID_ARG
    assert call(qw=A * 11 + 4) == vb.VDIT_ERR_MISALIGNED
    assert call(workspace=None) == vb.VDIT_ERR_WORKSPACE
    assert call(nbytes=need - 1) == vb.VDIT_ERR_WORKSPACE
    assert call(workspace=ws + 16) == vb.VDIT_ERR_MISALIGNED            # 256-byte alignment
    assert call(workspace=A) == vb.VDIT_ERR_INVALID_ARG                 # overlaps q


def test_qk_rms_norm_argument_checks():
    def call(q=A, k=A * 3, qo=A * 5, ko=A * 7, eps=1e-6, D=128, Sq=64, Skv=64, qw=None):
        return vb.vdit_qk_rms_norm(q, k, qo, ko, qw, None, eps, 1, 2, Sq, Skv, D, stream=0, check=False)
    assert call(eps=-1.0) == vb.VDIT_ERR_INVALID_ARG
    assert call(D=64) == vb.VDIT_ERR_UNSUPPORTED
    assert call(qo=A * 5 + 8) == vb.VDIT_ERR_MISALIGNED
    assert call(qw=A * 9 + 4) == vb.VDIT_ERR_MISALIGNED
    assert call(qo=A + 256) == vb.VDIT_ERR_INVALID_ARG                  # partial overlap with its input
    assert call(ko=A * 5) == vb.VDIT_ERR_INVALID_ARG                    # the two outputs overlap
    assert call(k=None, Skv=64) == vb.VDIT_ERR_INVALID_ARG
    assert call(Sq=0, Skv=0) == vb.VDIT_OK                              # nothing to do, nothing launched


def test_fp8_entry_point_argument_checks():
    st, parts, total = vb.vdit_fp8_layout(1, 2, 300, 333, 128)
    assert st == vb.VDIT_OK and total > 0
    assert list(parts.values()) == sorted(parts.values())                       # parts in order
    assert all(o % 256 == 0 for o in parts.values())                            # each 256-byte aligned
    assert parts["k"] - parts["q"] >= 300 * 2 * 128                             # Q codes: one byte per element
    st, need = vb.vdit_attn_fp8_plan(1, 2, 300, 333, 128, 0, 0)
    assert st == vb.VDIT_OK and need == total
    assert vb.vdit_attn_fp8_plan(1, 2, 300, 333, 128, vb.VDIT_MASK_BLOCK_SPARSE, 0)[0] == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_fp8_plan(1, 2, 300, 333, 64, 0, 0)[0] == vb.VDIT_ERR_UNSUPPORTED
    ws = A * 64
    q, k, v, o, lse = A, A * 3, A * 5, A * 7, A * 9
    assert vb.vdit_fp8_quantize(q, k, v, 1, 2, 300, 333, 128, None, 0, stream=0, check=False) == vb.VDIT_ERR_WORKSPACE
    assert vb.vdit_fp8_quantize(q, k, v, 1, 2, 300, 333, 128, ws, total - 1, stream=0,
                                check=False) == vb.VDIT_ERR_WORKSPACE
    assert vb.vdit_fp8_quantize(q, k, v, 1, 2, 300, 333, 128, ws + 128, total, stream=0,
                                check=False) == vb.VDIT_ERR_MISALIGNED
    assert vb.vdit_fp8_quantize(q, k, v + 8, 1, 2, 300, 333, 128, ws, total, stream=0,
                                check=False) == vb.VDIT_ERR_MISALIGNED
    assert vb.vdit_fp8_quantize(q, k, v, 1, 2, 300, 333, 128, q, total, stream=0,
                                check=False) == vb.VDIT_ERR_INVALID_ARG           # workspace over q
    assert vb.vdit_attn_fwd_fp8(q, k, v, o, lse, 1, 2, 300, 333, 128, 0.1, vb.VDIT_MASK_BLOCK_CAUSAL, 100, ws,
                                total, stream=0, check=False) == vb.VDIT_ERR_INVALID_ARG   # needs Sq == Skv
    assert vb.vdit_attn_fwd_fp8(q, k, v, o, lse, 1, 2, 300, 333, 128, -1.0, 0, 0, ws, total, stream=0,
                                check=False) == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_attn_fwd_fp8_quantized(o, lse, 1, 2, 300, 333, 128, 0.1, 0, 0, ws, total - 256, stream=0,
                                          check=False) == vb.VDIT_ERR_WORKSPACE


def test_group_entry_point_argument_checks():
    st, need = vb.vdit_vsmooth_group_plan(1, 2, 1000, 128, 64)
    assert st == vb.VDIT_OK and need >= 2 * 64 * 128 * 4 + 2 * 64 * 4
    for C in (0, 65):
        assert vb.vdit_vsmooth_group_plan(1, 2, 1000, 128, C)[0] == vb.VDIT_ERR_INVALID_ARG
    assert vb.vdit_vsmooth_group_plan(1, 2, 1000, 64, 8)[0] == vb.VDIT_ERR_UNSUPPORTED
    v, cent, labels, perm, ws = A, A * 3, A * 5, A * 7, A * 64

    def group(**kw):
        a = dict(v=v, centroids=cent, labels=labels, perm=perm, iters=2, workspace=ws, nbytes=need)
        a.update(kw)
        return vb.vdit_vsmooth_group(a["v"], a["centroids"], a["labels"], a["perm"], 1, 2, 1000, 128, 64,
                                     a["iters"], a["workspace"], a["nbytes"], stream=0, check=False)
    assert group(workspace=None) == vb.VDIT_ERR_WORKSPACE
    assert group(nbytes=need - 4) == vb.VDIT_ERR_WORKSPACE
    assert group(labels=labels + 2) == vb.VDIT_ERR_MISALIGNED
    assert group(iters=-1) == vb.VDIT_ERR_INVALID_ARG
    assert group(perm=labels) == vb.VDIT_ERR_INVALID_ARG                         # labels and perm overlap
    assert group(workspace=v) == vb.VDIT_ERR_INVALID_ARG                         # workspace over v
    k, kout, vout = A * 9, A * 11, A * 13
    assert vb.vdit_permute_kv(k, v, perm, kout, vout, 1, 2, 1000, 64, stream=0,
                              check=False) == vb.VDIT_ERR_UNSUPPORTED
    assert vb.vdit_permute_kv(k, v, perm, kout, kout, 1, 2, 1000, 128, stream=0,
                              check=False) == vb.VDIT_ERR_INVALID_ARG             # both outputs in one buffer
    assert vb.vdit_permute_kv(k, v, perm, k, vout, 1, 2, 1000, 128, stream=0,
                              check=False) == vb.VDIT_ERR_INVALID_ARG             # in place is not allowed
    assert vb.vdit_permute_kv(k, v, perm, kout + 4, vout, 1, 2, 1000, 128, stream=0,
                              check=False) == vb.VDIT_ERR_MISALIGNED


def test_empty_call_is_a_no_op():
    for B, H, Sq in [(0, 2, 64), (1, 0, 64), (1, 2, 0)]:
        assert vb.vdit_attn_fwd(None, None, None, None, None, B, H, Sq, 64, 128, 0.1, 0, 0,
                                stream=0, check=False) == vb.VDIT_OK


def test_cta_span_entry_checks_its_buffer_on_the_host():
    ok_args = dict(q=1 << 20, k=2 << 20, v=3 << 20, o=4 << 20, lse=None, B=1, H=2, Sq=300, Skv=77, D=128, scale=0.1)
    a = ok_args
    st, grid = vb.vdit_testing_cross_cta_spans(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Sq"],
                                               a["Skv"], a["D"], a["scale"], None, 16)
    assert st == vb.VDIT_ERR_INVALID_ARG and grid == 0
    st, _ = vb.vdit_testing_cross_cta_spans(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Sq"],
                                            a["Skv"], a["D"], a["scale"], (5 << 20) + 4, 16)
    assert st == vb.VDIT_ERR_MISALIGNED
    st, _ = vb.vdit_testing_cross_cta_spans(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Sq"],
                                            a["Skv"], a["D"], a["scale"], 5 << 20, 0)
    assert st == vb.VDIT_ERR_INVALID_ARG
