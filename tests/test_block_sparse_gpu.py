"""Block-sparse attention on the GPU against the fp64 oracle's block-sparse mode."""
import math

import numpy as np
import pytest
import torch

from oracle import MASK_BLOCK_SPARSE as ORACLE_SPARSE
from oracle import attention as oracle_attention
from tests.helpers import check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def run_sparse(q, k, v, mask, scale):
    dev = torch.device("cuda:0")
    o, lse = vb.attention_block_sparse(q.to(dev), k.to(dev), v.to(dev), mask.to(dev), scale)
    st, word = vb.vdit_get_device_status()
    assert st == vb.VDIT_OK, f"device status {vb.vdit_status_string(st)} word={word:#x}"
    return o, lse


def check_all_rows(q, k, v, mask, scale, label):
    o, lse = run_sparse(q, k, v, mask, scale)
    o_g = o.float().cpu().numpy().astype(np.float64)
    l_g = lse.cpu().numpy().astype(np.float64)
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, ORACLE_SPARSE,
                                block_mask=mask.numpy())
    B, Sq, H, D = q.shape
    empty = np.isneginf(l_r)
    # rows without any allowed key: exactly zero output and LSE = -inf
    for b in range(B):
        for h in range(H):
            rows = empty[b, h]
            assert np.all(o_g[b, rows, h] == 0.0)
            assert np.all(np.isneginf(l_g[b, h, rows]))
    og, orr, lg, lr, groups, n = [], [], [], [], [], 0
    for b in range(B):
        for h in range(H):
            rows = ~empty[b, h]
            if rows.sum() == 0:
                continue
            og.append(o_g[b, rows, h]); orr.append(o_r[b, rows, h])
            lg.append(l_g[b, h, rows]); lr.append(l_r[b, h, rows])
            groups.append(np.arange(n, n + rows.sum())); n += rows.sum()
    res = check_parity(np.concatenate(og), np.concatenate(orr), np.concatenate(lg), np.concatenate(lr),
                       groups, label)
    assert res["ok"], res
    return empty


@pytest.mark.parametrize("B,H,Sq,Skv,density", [
    (1, 2, 1024, 1024, 0.5),
    (1, 2, 1024, 1024, 0.1),
    (2, 3, 300, 333, 0.4),
    (1, 1, 2000, 1500, 0.25),
    (1, 2, 129, 700, 0.3),
])
def test_block_sparse_matches_oracle(B, H, Sq, Skv, density):
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=41 + Sq + Skv, recipe="rms_qk")
    mask = wl.draw_block_mask(B, H, Sq, Skv, density, seed=Sq * 7 + Skv, keep_diagonal=False)
    check_all_rows(q, k, v, mask, 1 / math.sqrt(128), f"sparse {B}x{H}x{Sq}x{Skv} d{density}")


def test_empty_blocks_and_empty_ctas():
    B, H, Sq, Skv = 1, 2, 1024, 900
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=50, recipe="rms_qk")
    mask = wl.draw_block_mask(B, H, Sq, Skv, 0.5, seed=51, keep_diagonal=False)
    mask[0, 0, 1, :] = 0          # one query block with no keys, its partner block has some
    mask[0, 1, 4:6, :] = 0        # both query blocks of one CTA have no keys: nothing to visit
    mask[0, 1, 0, :] = 0
    mask[0, 1, 0, 6] = 1          # a single allowed block, the ragged last one
    empty = check_all_rows(q, k, v, mask, 1 / math.sqrt(128), "empty blocks")
    assert empty[0, 1, 512:768].all() and empty[0, 0, 128:256].all()


def test_unequal_key_lists():
    # The MMA issuer derives each stream entry's owner from the two list
    # lengths: entries alternate while both lists last, then the longer one's
    # rest follows.  Cover a long tail on either tile, equal lengths (no
    # tail), one entry against many, and one empty list.
    B, H, Sq, Skv = 1, 2, 1024, 1500
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=54, recipe="rms_qk")
    nkb = -(-Skv // 128)
    mask = torch.zeros((B, H, Sq // 128, nkb), dtype=torch.uint8)
    mask[0, 0, 0, :] = 1          # CTA 0: tile 0 has every key block, tile 1 one
    mask[0, 0, 1, 5] = 1
    mask[0, 0, 2, 3] = 1          # CTA 1: tile 0 one block, tile 1 every other block
    mask[0, 0, 3, ::2] = 1
    mask[0, 0, 4, 1:9] = 1        # CTA 2: equal lengths, different blocks
    mask[0, 0, 5, 3:11] = 1
    mask[0, 0, 6, :4] = 1         # CTA 3: tile 1 has no key block
    mask[0, 1, 0, 10:] = 1        # head 1: tails of two and ten entries
    mask[0, 1, 1, :] = 1
    mask[0, 1, 2, :] = 1
    mask[0, 1, 3, 7:9] = 1
    mask[0, 1, 4:8, :] = torch.rand((4, nkb), generator=torch.Generator().manual_seed(55)).lt(0.6).to(torch.uint8)
    empty = check_all_rows(q, k, v, mask, 1 / math.sqrt(128), "unequal key lists")
    assert empty[0, 0, 896:1024].all() and not empty[0, 0, :896].any()


def test_all_ones_mask_equals_the_full_path_bitwise():
    dev = torch.device("cuda:0")
    B, H, Sq, Skv = 1, 2, 1000, 777
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, Sq, Skv, 128, seed=52, recipe="rms_qk"))
    ones = torch.ones((B, H, 8, 7), dtype=torch.uint8, device=dev)
    o1, l1 = vb.attention_block_sparse(q, k, v, ones)
    o2, l2 = vb.attention(q, k, v, None, vb.VDIT_MASK_CROSS)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_block_causal_pattern_equals_the_block_causal_path_bitwise():
    dev = torch.device("cuda:0")
    B, H, S, c = 1, 2, 1300, 256
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, S, S, 128, seed=53, recipe="rms_qk"))
    nb = -(-S // 128)
    blk = torch.arange(nb) * 128 // c
    pattern = (blk[None, :] <= blk[:, None]).to(torch.uint8)
    mask = pattern.expand(B, H, nb, nb).contiguous().to(dev)
    o1, l1 = vb.attention_block_sparse(q, k, v, mask)
    o2, l2 = vb.attention(q, k, v, None, vb.VDIT_MASK_BLOCK_CAUSAL, c)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_full_size_sparse_workload_sampled():
    name = "wan21_14b_720p_sparse25"
    call = wl.WORKLOADS[name].calls[0]
    inp = wl.workload_inputs(name)
    o, lse = run_sparse(inp["q"], inp["k"], inp["v"], inp["block_mask"], call.scale)
    o_g = o.float().cpu().numpy().astype(np.float64)
    l_g = lse.cpu().numpy().astype(np.float64)
    rows = wl.sample_rows(call.B, call.H, call.Sq, 10, seed=105)
    o_r, l_r = oracle_attention(wl.bf16_bits(inp["q"]), wl.bf16_bits(inp["k"]), wl.bf16_bits(inp["v"]),
                                call.scale, ORACLE_SPARSE, rows=rows, block_mask=inp["block_mask"].numpy())
    o_s = o_g[rows[:, 0], rows[:, 2], rows[:, 1]]
    l_s = l_g[rows[:, 0], rows[:, 1], rows[:, 2]]
    groups = [np.nonzero(rows[:, 1] == h)[0] for h in range(call.H)]
    res = check_parity(o_s, o_r, l_s, l_r, groups, name)
    assert res["ok"], res
