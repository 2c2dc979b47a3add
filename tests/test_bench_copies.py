"""The end-to-end leg's head-group copies, on the CPU.

bench.copy_heads moves heads [h0, h0 + hg) between a tensor holding every
head and a compact one holding only those heads, as one pitched copy
(cudaMemcpy2DAsync).  Here a stand-in runtime performs the pitched copy row
by row in host memory, so the pointer, pitch, width and row arithmetic is
checked against plain slicing for every tensor kind the bench moves.
"""
import ctypes
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


class _HostRuntime:
    """cudaMemcpy2DAsync semantics on host pointers."""

    def __init__(self):
        self.calls = []

    def cudaMemcpy2DAsync(self, dst, dpitch, src, spitch, width, height, kind, stream):
        assert width <= dpitch and width <= spitch
        for r in range(height):
            ctypes.memmove(dst + r * dpitch, src + r * spitch, width)
        self.calls.append((dpitch, spitch, width, height, kind))
        return 0


class _Stream:
    cuda_stream = 0


@pytest.mark.parametrize("shape,axis,dtype", [
    ((2, 37, 8, 16), 2, torch.bfloat16),    # BSHD activations
    ((1, 300, 40, 128), 2, torch.bfloat16),
    ((2, 8, 37), 1, torch.float32),         # LSE [B, H, S]
    ((2, 8, 5, 7), 1, torch.uint8),         # block mask [B, H, n_qb, n_kvb]
])
@pytest.mark.parametrize("groups", [1, 2, 4, 8])
def test_copy_heads_round_trip(shape, axis, dtype, groups):
    import bench
    H = shape[axis]
    if H % groups:
        pytest.skip("groups must divide H")
    hg = H // groups
    g = torch.Generator().manual_seed(0)
    full = (torch.randn(shape, generator=g) * 100).to(dtype)
    back = torch.zeros_like(full)
    rt = _HostRuntime()
    for gi in range(groups):
        gshape = tuple(hg if a == axis else n for a, n in enumerate(shape))
        part = torch.zeros(gshape, dtype=dtype)
        bench.copy_heads(rt, part, full, axis, gi * hg, hg, True, _Stream())
        idx = [slice(None)] * len(shape)
        idx[axis] = slice(gi * hg, (gi + 1) * hg)
        assert torch.equal(part, full[tuple(idx)].contiguous())
        bench.copy_heads(rt, part, back, axis, gi * hg, hg, False, _Stream())
    assert torch.equal(back, full)
    # one pitched copy per tensor and direction
    assert len(rt.calls) == 2 * groups
    assert {c[4] for c in rt.calls} == {1, 2}


def test_head_axes_cover_every_input():
    import bench
    from video_diffusion_transformer_attention_b200 import workloads as wl
    for name in wl.WORKLOADS:
        w = wl.WORKLOADS[name]
        keys = {"q", "k", "v"} | ({"k_text", "v_text"} if w.text_tokens else set())
        if w.calls[0].mask_kind == wl.MASK_BLOCK_SPARSE:
            keys |= {"block_mask"}
        assert keys <= set(bench.HEAD_AXIS), name
