"""Pins of the oracle's IBCS stages (mean key, per-block k-means, block score).

The AB-Attention news page, section «Три приёма AB-Attention» (IBCS), fixes: 128-token
query blocks, clusters with a centroid and a weight equal to the share of the block's
queries, and a block score equal to the weighted attention of the centroids to the
block's averaged keys. These tests pin the oracle to hand-worked examples, closed forms
and special cases that reduce to library routines.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from block_sparse_attention_ab_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def _points_tensor(points, d):
    """One head, one block: point values on coordinate 0, zero elsewhere, zero padding."""
    q = np.zeros((1, 1, 128, d), dtype=np.float32)
    q[0, 0, : len(points), 0] = points
    return _bf16(q)


def test_kmeans_hand_worked(orc):
    g = json.load(open(os.path.join(GOLD, "kmeans_hand.json")))
    d = g["d"]
    for case in g["cases"]:
        pts = case["points"]
        q = _points_tensor(pts, d)
        cent, wts, assign, gap, inert = orc.kmeans(q, len(pts), case["C"], case["T"])
        np.testing.assert_array_equal(cent[0, 0, 0, :, 0], case["centroids"], err_msg=case["name"])
        assert np.all(cent[0, 0, 0, :, 1:] == 0.0)
        np.testing.assert_array_equal(wts[0, 0, 0], case["weights"], err_msg=case["name"])
        np.testing.assert_array_equal(assign[0, 0, : len(pts)], case["assign"], err_msg=case["name"])
        assert np.all(assign[0, 0, len(pts):] == 255)


def _tiny_inputs():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(w)
    return w, q, k, v


def test_kmeans_invariants(orc):
    w, q, k, v = _tiny_inputs()
    C, T = 8, 5
    cent, wts, assign, gap, inert = orc.kmeans(q, w.N, C, T)
    # Shares of the block's queries sum to one (counts are integers).
    np.testing.assert_allclose(wts.sum(-1), 1.0, rtol=0, atol=1e-15)
    assert np.all(wts * 128 == np.round(wts * 128))
    # Centroid = mean of its members under the final assignment (non-empty clusters).
    qf = q.float().numpy().astype(np.float64)
    for h in range(w.H):
        for qb in range(w.n_blocks):
            rows = qf[0, h, qb * 128:(qb + 1) * 128]
            lab = assign[0, h, qb * 128:(qb + 1) * 128]
            for c in range(C):
                m = lab == c
                if m.any():
                    np.testing.assert_allclose(cent[0, h, qb, c], rows[m].mean(0), rtol=1e-12,
                                               atol=1e-12)
                # Final assignment is the nearest centroid of the previous update;
                # after convergence it is a fixed point, checked below with T large.
    # Inertia never increases from one Lloyd iteration to the next.
    assert np.all(np.diff(inert, axis=-1) <= 1e-9 * inert[..., :-1])


def test_kmeans_converged_fixed_point(orc):
    """With many iterations Lloyd's algorithm reaches a fixed point: every query is at
    its nearest centroid (brute-force distances with numpy)."""
    w, q, k, v = _tiny_inputs()
    cent, wts, assign, gap, _ = orc.kmeans(q, w.N, 8, 60)
    qf = q.float().numpy().astype(np.float64)
    for h in range(w.H):
        for qb in range(w.n_blocks):
            rows = qf[0, h, qb * 128:(qb + 1) * 128]
            dist = ((rows[:, None, :] - cent[0, h, qb][None, :, :]) ** 2).sum(-1)
            lab = assign[0, h, qb * 128:(qb + 1) * 128]
            best = dist.min(1)
            np.testing.assert_allclose(dist[np.arange(128), lab], best, rtol=1e-12, atol=0)


def test_kmeans_one_cluster_is_block_mean(orc):
    w, q, k, v = _tiny_inputs()
    cent, wts, assign, gap, _ = orc.kmeans(q, w.N, 1, 3)
    qf = q.float().numpy().astype(np.float64)
    means = qf[0].reshape(w.H, w.n_blocks, 128, w.d).mean(2)
    np.testing.assert_allclose(cent[0, :, :, 0], means, rtol=1e-13, atol=1e-13)
    assert np.all(wts == 1.0)


def test_kmeans_ragged_block(orc):
    """The last block of a ragged sequence clusters only its valid queries."""
    rng = np.random.default_rng(5)
    N = 128 + 37
    q = np.zeros((1, 1, 256, 64), dtype=np.float32)
    q[0, 0, :N] = rng.standard_normal((N, 64))
    q[0, 0, N:] = 1e3  # padding content must not matter
    qt = _bf16(q)
    cent, wts, assign, _, _ = orc.kmeans(qt, N, 8, 5)
    q2 = q.copy()
    q2[0, 0, N:] = 0.0
    cent2, wts2, assign2, _, _ = orc.kmeans(_bf16(q2), N, 8, 5)
    np.testing.assert_array_equal(cent, cent2)
    np.testing.assert_array_equal(wts, wts2)
    assert np.all(wts[0, 0, 1] * 37 == np.round(wts[0, 0, 1] * 37))
    np.testing.assert_allclose(wts[0, 0, 1].sum(), 1.0, atol=1e-15)
    assert np.all(assign[0, 0, N:] == 255)


def test_mean_key_matches_numpy(orc):
    rng = np.random.default_rng(1)
    N = 3 * 128 + 16  # last block holds 16 valid keys
    k = np.zeros((2, 3, 512, 64), dtype=np.float32)
    k[:, :, :N] = rng.standard_normal((2, 3, N, 64))
    k[:, :, N:] = 7.0  # padding must be ignored
    kt = _bf16(k)
    kbar = orc.mean_key(kt, N)
    kv = kt.float().numpy().astype(np.float64)
    for j in range(4):
        t1 = min(N, (j + 1) * 128)
        np.testing.assert_allclose(kbar[:, :, j], kv[:, :, j * 128:t1].mean(2), rtol=1e-13,
                                   atol=1e-14)


def test_score_hand_worked(orc):
    g = json.load(open(os.path.join(GOLD, "score_hand.json")))
    d = g["d"]
    for case in g["cases"]:
        C = len(case["centroid_e0"])
        nkb = len(case["kbar_e0"])
        cent = np.zeros((1, 1, 1, C, d))
        cent[0, 0, 0, :, 0] = case["centroid_e0"]
        kbar = np.zeros((1, 1, nkb, d))
        kbar[0, 0, :, 0] = case["kbar_e0"]
        wts = np.asarray(case["weights"], dtype=np.float64).reshape(1, 1, 1, C)
        s = orc.score(cent, wts, kbar)
        np.testing.assert_allclose(s[0, 0, 0], case["scores"], rtol=1e-14, atol=1e-15,
                                   err_msg=case["name"])


def test_score_invariants_and_mean_pool(orc):
    w, q, k, v = _tiny_inputs()
    s = orc.ibcs_scores(q, k, w.N, 8, 5)
    # A convex combination of softmax rows: sums to one per query block.
    np.testing.assert_allclose(s.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert np.all(s > 0)
    # One cluster: the mean-pooled block score softmax_j(qbar . kbar_j / sqrt(d)),
    # computed here with numpy means and scipy's softmax.
    s1 = orc.ibcs_scores(q, k, w.N, 1, 5)
    qf = q.float().numpy().astype(np.float64)[0]
    kf = k.float().numpy().astype(np.float64)[0]
    qbar = qf.reshape(w.H, w.n_blocks, 128, w.d).mean(2)
    kbar = kf.reshape(w.H, w.n_blocks, 128, w.d).mean(2)
    logits = np.einsum("hqd,hkd->hqk", qbar, kbar) / math.sqrt(w.d)
    np.testing.assert_allclose(s1[0], scipy.special.softmax(logits, axis=-1), rtol=1e-12,
                               atol=1e-15)


def test_score_identical_key_blocks_are_uniform(orc):
    rng = np.random.default_rng(2)
    d, nb = 64, 5
    blk = rng.standard_normal((128, d)).astype(np.float32)
    k = np.tile(blk, (nb, 1)).reshape(1, 1, nb * 128, d)
    q = rng.standard_normal((1, 1, nb * 128, d)).astype(np.float32)
    s = orc.ibcs_scores(_bf16(q), _bf16(k), nb * 128, 8, 5)
    np.testing.assert_allclose(s, 1.0 / nb, rtol=1e-13)
