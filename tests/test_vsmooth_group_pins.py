"""Pins of the V-Smooth Group oracle (oracle/vsmooth_group.py)."""
import math

import numpy as np
import torch

from oracle import attention
from oracle import vsmooth_group as vg
from tests.helpers import to_bf16_bits


def test_well_separated_clusters_are_recovered_with_their_means():
    g = np.random.default_rng(1)
    centers = np.array([[8.0] * 4, [-8.0] * 4, [8.0, -8.0] * 2, [-8.0, 8.0] * 2])
    truth = g.integers(0, 4, 400)
    x = centers[truth] + g.normal(0, 0.1, (400, 4))
    init = np.stack([x[np.flatnonzero(truth == k)[0]] for k in range(4)])   # one seed token per cluster
    lab = vg.assign(x, init)
    c = vg.update(x, lab, init)
    assert np.array_equal(lab, truth)
    for k in range(4):
        assert np.allclose(c[k], x[truth == k].mean(axis=0), rtol=0, atol=1e-12)
    assert np.array_equal(vg.assign(x, c), truth)


def test_ties_go_to_the_lowest_index_and_empty_clusters_stay():
    x = np.array([[0.0, 0.0], [2.0, 0.0]])
    c = np.array([[1.0, 1.0], [1.0, -1.0], [50.0, 50.0]])   # both tokens equidistant from 0 and 1
    lab = vg.assign(x, c)
    assert lab.tolist() == [0, 0]
    new = vg.update(x, lab, c)
    assert np.allclose(new[0], [1.0, 0.0]) and np.array_equal(new[1], c[1]) and np.array_equal(new[2], c[2])


def test_the_permutation_is_a_stable_sort_by_cluster():
    assert vg.group_permutation([2, 0, 1, 0, 2, 1]).tolist() == [1, 3, 2, 5, 0, 4]


def test_joint_key_value_permutation_leaves_full_attention_unchanged():
    g = torch.Generator().manual_seed(2)
    q, k, v = (torch.randn(1, n, 2, 128, generator=g).to(torch.bfloat16) for n in (50, 300, 300))
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    perm = np.stack([np.random.default_rng(h).permutation(300) for h in range(2)])[None]
    kp = vg.permute_tokens(bits(k), perm)
    vp = vg.permute_tokens(bits(v), perm)
    o1, l1 = attention(bits(q), bits(k), bits(v), 1 / math.sqrt(128))
    o2, l2 = attention(bits(q), kp, vp, 1 / math.sqrt(128))
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(l1, l2, rtol=0, atol=1e-12)
    # and the gather is the per-head permutation it claims
    assert np.array_equal(kp[0, :, 1], bits(k)[0, perm[0, 1], 1])


def test_grouping_lets_the_block_mean_remove_more_of_the_energy():
    # V from 8 well-spread value clusters in random token order: block means of
    # the raw order remove little, after grouping they remove most of it
    g = np.random.default_rng(3)
    S, D, C = 2048, 128, 8
    centers = g.normal(0, 1, (C, D))
    truth = g.integers(0, C, S)
    v = centers[truth] + g.normal(0, 0.3, (S, D))
    vb = to_bf16_bits(v)[:, None, None, :].transpose(1, 0, 2, 3)          # [1, S, 1, D]
    init = np.stack([v[np.flatnonzero(truth == k)[0]] for k in range(C)])[None, None]
    labels, cent, perm = vg.kmeans(vb, init, iters=3)
    vf = (vb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[0, :, 0, :]
    before = vg.block_energy_removed(vf)
    after = vg.block_energy_removed(vf[perm[0, 0]])
    assert after > 0.5 and after > 3 * before, (before, after)
    assert np.array_equal(labels[0, 0], truth)
