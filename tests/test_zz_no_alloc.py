"""The entry point that allocates nothing: vdit_attn_fwd_qknorm_noalloc.

Some callers of this library cannot call cudaMalloc: a plugin running inside
an application that owns every byte of the GPU through its own memory pool
(a raw allocation would go around the pool and may fail once the pool holds
the rest of the device), or a latency-critical loop in which cudaMalloc and
cudaFree can synchronise the device.  For them the Q/K-norm + attention call
has a variant that keeps its normalised Q and K in a fixed scratch array
built into the library instead of in a workspace the caller allocates.

This test calls that variant through the C ABI several times in a row, with
different shapes, masks and data (the scratch still holds the previous call's
contents when the next one runs), and requires each result to equal, bit for
bit, that of the workspace entry point vdit_attn_fwd_qknorm on the same
inputs: both run the same deterministic kernels on the same data, so any
difference (a call reading what an earlier one left in the scratch, say)
is a fault.  The file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import math

import pytest
import torch

from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def _with_workspace(q, k, v, qw, kw, mask, chunk):
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    st, need = vb.vdit_attn_qknorm_plan(B, H, Sq, Skv, D, mask, chunk)
    assert st == vb.VDIT_OK
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    o, lse = torch.empty_like(q), torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    vb.vdit_attn_fwd_qknorm(q, k, v, o, lse, qw, kw, 1e-6, B, H, Sq, Skv, D, 1 / math.sqrt(D), mask, chunk,
                            ws, need)
    return o, lse


def _no_alloc(q, k, v, qw, kw, mask, chunk):
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    o, lse = torch.empty_like(q), torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    st = vb.vdit_attn_fwd_qknorm_noalloc(q, k, v, o, lse, qw, kw, 1e-6, B, H, Sq, Skv, D, 1 / math.sqrt(D), mask,
                                         chunk, check=False)
    assert st == vb.VDIT_OK, vb.vdit_status_string(st)
    return o, lse


def test_no_alloc_entry_equals_the_workspace_entry_on_calls_in_a_row():
    dev = torch.device("cuda:0")
    cases = [  # (B, H, Sq, Skv, mask, chunk, seed)
        (1, 4, 1000, 1000, vb.VDIT_MASK_FULL, 0, 81),
        (2, 3, 777, 777, vb.VDIT_MASK_BLOCK_CAUSAL, 300, 82),
        (1, 2, 640, 77, vb.VDIT_MASK_CROSS, 0, 83),
        (1, 4, 1000, 1000, vb.VDIT_MASK_FULL, 0, 84),  # the first shape again, on other data
    ]
    for B, H, Sq, Skv, mask, chunk, seed in cases:
        q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, Sq, Skv, 128, seed=seed))
        g = torch.Generator().manual_seed(seed)
        qw = (torch.rand(H, 128, generator=g) + 0.5).to(dev)
        kw = (torch.rand(H, 128, generator=g) + 0.5).to(dev)
        o_n, l_n = _no_alloc(q, k, v, qw, kw, mask, chunk)
        o_w, l_w = _with_workspace(q, k, v, qw, kw, mask, chunk)
        torch.cuda.synchronize()
        assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
        assert torch.equal(o_n, o_w), (B, H, Sq, Skv, mask)
        assert torch.equal(l_n, l_w), (B, H, Sq, Skv, mask)


def test_no_alloc_entry_checks_arguments_like_the_workspace_entry():
    # an empty shape still has its eps and weight alignment checked, as the
    # workspace entry point does; nothing is launched either way
    for eps, qw, want in ((0.0, None, vb.VDIT_ERR_INVALID_ARG), (float("nan"), None, vb.VDIT_ERR_INVALID_ARG),
                          (1e-6, (1 << 20) + 4, vb.VDIT_ERR_MISALIGNED), (1e-6, None, vb.VDIT_OK)):
        for fn in ("noalloc", "ws"):
            if fn == "noalloc":
                st = vb.vdit_attn_fwd_qknorm_noalloc(None, None, None, None, None, qw, None, eps, 1, 2, 0, 16, 128,
                                                     0.1, 0, 0, check=False)
            else:
                st = vb.vdit_attn_fwd_qknorm(None, None, None, None, None, qw, None, eps, 1, 2, 0, 16, 128, 0.1, 0,
                                             0, None, 0, check=False)
            assert st == want, (fn, eps, qw, vb.vdit_status_string(st))


def test_no_alloc_entry_rejects_shapes_beyond_its_scratch():
    # 2 * 4096 rows * 32 heads * 256 B = 64 MiB of normalised Q and K fits; one more token does not
    B, H, S = 1, 32, 4096
    assert vb.vdit_attn_qknorm_plan(B, H, S, S, 128, 0, 0)[1] == vb.NOALLOC_SCRATCH_BYTES
    st = vb.vdit_attn_fwd_qknorm_noalloc(1 << 20, 3 << 20, 5 << 20, 7 << 20, None, None, None, 1e-6,
                                         B, H, S + 1, S + 1, 128, 0.1, 0, 0, check=False)
    assert st == vb.VDIT_ERR_WORKSPACE
