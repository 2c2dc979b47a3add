"""V-Smooth Group on the GPU: k-means assignment and update, the stable cluster
sort, the joint K/V gather, and what grouping buys the 8-bit attention.

Centroid sums use float atomics, whose order varies, so the GPU's centroids
are checked as what they must be (the mean of the tokens assigned to them, on
data whose assignment has no near-ties), its labels as valid nearest
centroids of its own centroids, and its permutation exactly, as the stable
sort of its own labels.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as exact_attention
from oracle import fp8_oracle as f8
from oracle import vsmooth_group as vg
from tests.helpers import check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def _clustered_v(B, S, H, C, seed, spread=1.0, noise=0.3):
    """V from C value clusters per head, in random token order; returns (v bf16, labels)."""
    g = np.random.default_rng(seed)
    v = np.zeros((B, S, H, 128))
    truth = np.zeros((B, H, S), np.int64)
    for b in range(B):
        for h in range(H):
            centers = g.normal(0, spread, (C, 128))
            lab = g.integers(0, C, S)
            v[b, :, h] = centers[lab] + g.normal(0, noise, (S, 128))
            truth[b, h] = lab
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16), truth


def _seed_centroids(v, truth, C):
    """One token of every true cluster as the starting centroid (fp32 [B, H, C, 128])."""
    B, S, H, _ = v.shape
    vf = v.float().numpy()
    c = np.zeros((B, H, C, 128), np.float32)
    for b in range(B):
        for h in range(H):
            for k in range(C):
                idx = np.flatnonzero(truth[b, h] == k)
                # a cluster without tokens gets a far-away seed that no token picks
                c[b, h, k] = vf[b, idx[0], h] if len(idx) else 1000.0 + k
    return torch.tensor(c)


@pytest.mark.parametrize("B,H,S,C,iters", [(1, 2, 1000, 8, 3), (2, 1, 2500, 16, 1), (1, 3, 300, 64, 2)])
def test_group_recovers_clusters_means_and_a_stable_sort(B, H, S, C, iters):
    dev = torch.device("cuda:0")
    v, truth = _clustered_v(B, S, H, C, seed=S + C, spread=2.0, noise=0.2)
    cent = _seed_centroids(v, truth, C).to(dev)
    labels, perm = vb.vsmooth_group(v.to(dev), cent, iters=iters)
    torch.cuda.synchronize()
    lab = labels.cpu().numpy()
    pm = perm.cpu().numpy()
    cg = cent.cpu().numpy().astype(np.float64)
    vf = v.float().numpy().astype(np.float64)
    for b in range(B):
        for h in range(H):
            present = np.unique(truth[b, h])
            assert np.array_equal(lab[b, h], truth[b, h])                      # no near-ties in this data
            for k in present:                                                  # centroid = mean of its tokens
                want = vf[b, truth[b, h] == k, h].mean(axis=0)
                assert np.allclose(cg[b, h, k], want, rtol=1e-5, atol=1e-5)
            assert np.array_equal(pm[b, h], vg.group_permutation(lab[b, h]))   # exact stable sort


@pytest.mark.parametrize("C,iters", [(8, 0), (32, 2)])
def test_group_labels_are_nearest_centroids_on_unstructured_data(C, iters):
    dev = torch.device("cuda:0")
    B, H, S = 1, 2, 777
    _, _, v = wl.draw_qkv(B, H, S, S, 128, seed=97, recipe="rms_qk_vout")
    vf = v.float().numpy().astype(np.float64)
    init = torch.tensor(np.stack([vf[0, np.linspace(0, S - 1, C).astype(int), h] for h in range(H)])[None],
                        dtype=torch.float32)
    cent = init.clone().to(dev)
    labels, perm = vb.vsmooth_group(v.to(dev), cent, iters=iters)
    torch.cuda.synchronize()
    lab = labels.cpu().numpy()
    cg = cent.cpu().numpy().astype(np.float64)
    if iters == 0:
        assert torch.equal(cent.cpu(), init)                                  # no update without iterations
    for h in range(H):
        d = vg.distances(vf[0, :, h], cg[0, h])
        chosen = d[np.arange(S), lab[0, h]]
        scale = (vf[0, :, h] ** 2).sum(axis=1) + (cg[0, h] ** 2).sum(axis=1).max()
        assert np.all(chosen <= d.min(axis=1) + 1e-5 * scale)
        assert np.array_equal(perm.cpu().numpy()[0, h], vg.group_permutation(lab[0, h]))


def test_permute_kv_is_the_per_head_gather():
    dev = torch.device("cuda:0")
    B, H, S = 2, 3, 301
    q, k, v = wl.draw_qkv(B, H, S, S, 128, seed=98)
    perm = np.stack([np.stack([np.random.default_rng(b * 10 + h).permutation(S) for h in range(H)])
                     for b in range(B)]).astype(np.int32)
    ko, vo = vb.permute_kv(k.to(dev), v.to(dev), torch.tensor(perm).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(wl.bf16_bits(ko.cpu()), vg.permute_tokens(wl.bf16_bits(k), perm))
    assert np.array_equal(wl.bf16_bits(vo.cpu()), vg.permute_tokens(wl.bf16_bits(v), perm))


def _v_reconstruction_error(q, k, v):
    """Relative RMS error of V rebuilt from the GPU's V-Smooth codes, scales and block means."""
    dev = torch.device("cuda:0")
    B, S, H, D = v.shape
    st, parts, total = vb.vdit_fp8_layout(B, H, S, S, D)
    ws = torch.empty(total, dtype=torch.uint8, device=dev)
    vb.vdit_fp8_quantize(q, k, v, B, H, S, S, D, ws, total)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    nkb = -(-S // 128)
    vt = np.frombuffer(w[parts["vt"]:parts["vt"] + B * H * nkb * 128 * 128].tobytes(), np.uint8)
    vt = vt.reshape(B, H, nkb, 128, 128).transpose(0, 1, 2, 4, 3).reshape(B, H, nkb * 128, 128)[:, :, :S]
    sc = np.frombuffer(w[parts["v_scale"]:parts["v_scale"] + B * H * 512].tobytes(), np.float32).reshape(B, H, 1, 128)
    mu = np.frombuffer(w[parts["mu"]:parts["mu"] + B * H * nkb * 512].tobytes(), np.float32).reshape(B, H, nkb, 128)
    rec = f8.e4m3_values(vt) * sc + np.repeat(mu, 128, axis=2)[:, :, :S]
    ref = v.float().cpu().numpy().transpose(0, 2, 1, 3).astype(np.float64)
    return np.sqrt(((rec - ref) ** 2).mean()) / np.sqrt((ref ** 2).mean())


def test_grouping_shrinks_the_v_quantisation_error_and_keeps_attention_parity():
    dev = torch.device("cuda:0")
    B, H, S, C = 1, 2, 2048, 16
    v, truth = _clustered_v(B, S, H, C, seed=99, spread=1.0, noise=0.15)
    q, k, _ = wl.draw_qkv(B, H, S, S, 128, seed=99, recipe="rms_qk")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    cent = _seed_centroids(v.cpu(), truth, C).to(dev)
    _, perm = vb.vsmooth_group(v, cent, iters=2)
    kp, vp = vb.permute_kv(k, v, perm)
    e_plain = _v_reconstruction_error(q, k, v)
    e_grp = _v_reconstruction_error(q, kp, vp)
    assert e_grp < 0.5 * e_plain, (e_grp, e_plain)

    scale = 1 / math.sqrt(128)
    o_x, _ = exact_attention(wl.bf16_bits(q.cpu()), wl.bf16_bits(k.cpu()), wl.bf16_bits(v.cpu()), scale)

    def rel(o):
        return np.sqrt(((o - o_x) ** 2).mean()) / np.sqrt((o_x ** 2).mean())

    o_plain, _, _ = vb.attention_fp8(q, k, v, scale)
    o_grp, lse_grp, _ = vb.attention_fp8(q, kp, vp, scale)
    torch.cuda.synchronize()
    assert rel(o_grp.float().cpu().numpy().astype(np.float64)) <= \
        1.05 * rel(o_plain.float().cpu().numpy().astype(np.float64))
    # the grouped call is the 8-bit attention of the permuted K/V
    o_r, l_r = f8.attention_fp8(wl.bf16_bits(q.cpu()), wl.bf16_bits(kp.cpu()), wl.bf16_bits(vp.cpu()), scale)
    og = np.concatenate([o_grp.float().cpu().numpy()[0, :, h] for h in range(H)]).astype(np.float64)
    orr = np.concatenate([o_r[0, :, h] for h in range(H)])
    lg = lse_grp.cpu().numpy().reshape(-1).astype(np.float64)
    res = check_parity(og, orr, lg, l_r.reshape(-1), [np.arange(i * S, (i + 1) * S) for i in range(H)], "grouped",
                       excess_bar=None)
    assert res["ok"], res
