"""Pins of the oracle's block-sparse attention.

The AB-Attention news page, section «Три приёма AB-Attention» (SIP): each kept block
counts with weight 1/p in both the attention numerator and the softmax normaliser,
which gives unbiased estimates of both and keeps the computation ordinary softmax
attention with shifted logits. Section «Где ломаются прежние разреженные схемы»: top-k
drops a block from the numerator and from the normaliser. These tests check the oracle
against torch's scaled_dot_product_attention in fp64 (a library routine) in the cases
that reduce to it, and check unbiasedness by Monte Carlo.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_sparse_attention_ab_b200 import synth


def _tiny():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(w)
    return w, q, k, v


def _ragged(N=3 * 128 + 50, H=2, d=64, seed=0):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    q = torch.zeros(1, H, N_pad, d)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    q[:, :, :N] = torch.randn(1, H, N, d, generator=g) * 1.5
    k[:, :, :N] = torch.randn(1, H, N, d, generator=g) * 1.5
    v[:, :, :N] = torch.randn(1, H, N, d, generator=g)
    return N, q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def _sdpa(q, k, v, N, key_mask=None):
    """fp64 SDPA over the valid tokens; key_mask [B,H,N_pad,N_pad] boolean (True = keep)."""
    qf, kf, vf = (t.double()[:, :, :N] for t in (q, k, v))
    mask = None if key_mask is None else key_mask[:, :, :N, :N]
    return F.scaled_dot_product_attention(qf, kf, vf, attn_mask=mask)


def _all_blocks(B, H, nb):
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, H, nb, 1))
    cnt = np.full((B, H, nb), nb, dtype=np.int32)
    return idx, cnt


def _flat(out, B, H, nb, d):
    return out.reshape(B, H, nb * 128, d)


@pytest.mark.parametrize("case", ["tiny", "ragged"])
def test_all_blocks_equals_dense_sdpa(orc, case):
    if case == "tiny":
        w, q, k, v = _tiny()
        N = w.N
    else:
        N, q, k, v = _ragged()
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    idx, cnt = _all_blocks(B, H, nb)
    ones = np.ones((B, H, nb, nb), dtype=np.float32)
    out, lse, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, ones)
    out = _flat(out, B, H, nb, d)
    ref = _sdpa(q, k, v, N).numpy()
    np.testing.assert_allclose(out[:, :, :N], ref, rtol=1e-12, atol=1e-12)
    assert np.all(out[:, :, N:] == 0)
    # lse = logsumexp of the scaled logits over the valid keys
    logits = torch.einsum("bhid,bhjd->bhij", q.double()[:, :, :N], k.double()[:, :, :N]) / math.sqrt(d)
    ref_lse = torch.logsumexp(logits, -1).numpy()
    np.testing.assert_allclose(lse.reshape(B, H, N_pad)[:, :, :N], ref_lse, rtol=1e-12, atol=1e-12)
    # the separately coded dense oracle agrees too
    dense, dense_lse = orc.dense_attn(q, k, v, N)
    np.testing.assert_allclose(dense[:, :, :N], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dense_lse[:, :, :N], ref_lse, rtol=1e-12, atol=1e-12)


def test_topk_equals_sdpa_restricted_to_kept_blocks(orc):
    N, q, k, v = _ragged(N=5 * 128 + 9, seed=3)
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    rng = np.random.default_rng(4)
    s = rng.random((B, H, nb, nb)).astype(np.float32)
    idx, cnt, wts = orc.topk(s, 3)
    out, lse, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, None)
    out = _flat(out, B, H, nb, d)
    mask = torch.zeros(B, H, N_pad, N_pad, dtype=torch.bool)
    for b, h, qb in np.ndindex(B, H, nb):
        for j in idx[b, h, qb, : cnt[b, h, qb]]:
            mask[b, h, qb * 128:(qb + 1) * 128, j * 128:(j + 1) * 128] = True
    ref = _sdpa(q, k, v, N, mask).numpy()
    np.testing.assert_allclose(out[:, :, :N], ref, rtol=1e-12, atol=1e-12)


def test_integer_weight_equals_duplicated_keys(orc):
    """Weight w_j = m (integer) must equal dense attention in which block j's keys and
    values appear m times ("a block with probability 25% counts as four")."""
    N, q, k, v = _ragged(N=4 * 128, H=1, seed=8)
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    sel = [0, 2, 3]
    mult = [1, 4, 2]
    idx = np.full((B, H, nb, nb), -1, dtype=np.int32)
    wts = np.zeros((B, H, nb, nb), dtype=np.float32)
    cnt = np.full((B, H, nb), len(sel), dtype=np.int32)
    idx[..., : len(sel)] = sel
    wts[..., : len(sel)] = mult
    out, lse, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, wts)
    out = _flat(out, B, H, nb, d)
    kk = torch.cat([k[:, :, j * 128:(j + 1) * 128].repeat(1, 1, m, 1) for j, m in zip(sel, mult)], 2)
    vv = torch.cat([v[:, :, j * 128:(j + 1) * 128].repeat(1, 1, m, 1) for j, m in zip(sel, mult)], 2)
    ref = F.scaled_dot_product_attention(q.double(), kk.double(), vv.double()).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    logits = torch.einsum("bhid,bhjd->bhij", q.double(), kk.double()) / math.sqrt(d)
    np.testing.assert_allclose(lse.reshape(B, H, N_pad), torch.logsumexp(logits, -1).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_empty_selection_and_padding_rows(orc):
    N, q, k, v = _ragged(N=2 * 128 + 5, H=1, seed=2)
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    idx = np.zeros((B, H, nb, nb), dtype=np.int32)
    cnt = np.zeros((B, H, nb), dtype=np.int32)
    cnt[0, 0, 1] = 1  # only query block 1 attends (to key block 0)
    out, lse, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, None)
    assert np.all(out[0] == 0) and np.all(lse[0] == -np.inf)
    assert np.all(out[2, 5:] == 0) and np.all(lse[2, 5:] == 0)
    assert np.all(out[2, :5] == 0) and np.all(lse[2, :5] == -np.inf)
    assert np.abs(out[1]).sum() > 0


def test_ht_estimator_unbiased_monte_carlo(orc):
    """Over seeds 0..9999 of SIP at the tiny workload, the mean Horvitz-Thompson estimate
    of the numerator and of the denominator matches the full-attention values: per
    element |mean - full| <= 5 sigma_hat / sqrt(n), with at most 0.1% above 4 sigma.

    The numerator and denominator are linear in the per-block sums, so the oracle's
    attention is evaluated once per key block (unweighted, one block selected) and each
    draw's estimate is sum over kept blocks of w_j times that block's sums; a direct
    check that the oracle's weighted call equals that combination runs on a few seeds."""
    w_, q, k, v = _tiny()
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    N = w_.N
    s = orc.ibcs_scores(q, k, N, 8, 5).astype(np.float32)
    K = w_.budget_blocks(w_.budgets[0])
    # per-block unshifted numerator / denominator, blocks one at a time
    num_b = np.zeros((nb, B, H, nb, 128, d))
    den_b = np.zeros((nb, B, H, nb, 128))
    for j in range(nb):
        idx = np.full((B, H, nb, nb), j, dtype=np.int32)
        cnt = np.ones((B, H, nb), dtype=np.int32)
        _, _, num, den = orc.attn_rows(q, k, v, N, idx, cnt, None, want_num_den=True)
        num_b[j] = num.reshape(B, H, nb, 128, d)
        den_b[j] = den.reshape(B, H, nb, 128)
    full_num = num_b.sum(0)
    full_den = den_b.sum(0)
    # the all-blocks oracle call gives the same totals
    idx_all, cnt_all = _all_blocks(B, H, nb)
    _, _, num_all, den_all = orc.attn_rows(q, k, v, N, idx_all, cnt_all, None, want_num_den=True)
    np.testing.assert_allclose(num_all.reshape(full_num.shape), full_num, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(den_all.reshape(full_den.shape), full_den, rtol=1e-12)

    n = 10_000
    acc_n = np.zeros_like(full_num)
    acc_n2 = np.zeros_like(full_num)
    acc_d = np.zeros_like(full_den)
    acc_d2 = np.zeros_like(full_den)
    for seed in range(n):
        idx, cnt, wts, p, bad = orc.sip(s, K, seed, with_p=False)
        weight = np.zeros((B, H, nb, nb))
        for r in np.ndindex(B, H, nb):
            c = cnt[r]
            weight[r][idx[r][:c]] = wts[r][:c]
        est_n = np.einsum("bhqj,jbhqid->bhqid", weight, num_b)
        est_d = np.einsum("bhqj,jbhqi->bhqi", weight, den_b)
        acc_n += est_n
        acc_n2 += est_n**2
        acc_d += est_d
        acc_d2 += est_d**2
        if seed < 3:
            _, _, num_s, den_s = orc.attn_rows(q, k, v, N, idx, cnt, wts, want_num_den=True)
            np.testing.assert_allclose(num_s.reshape(est_n.shape), est_n, rtol=1e-6, atol=1e-9)
            np.testing.assert_allclose(den_s.reshape(est_d.shape), est_d, rtol=1e-6)
    for acc, acc2, full in ((acc_n, acc_n2, full_num), (acc_d, acc_d2, full_den)):
        mean = acc / n
        var = np.maximum(acc2 / n - mean**2, 0.0)
        se = np.sqrt(var / n)
        dev = np.abs(mean - full)
        tight = se > 1e-12 * np.abs(full).max()
        assert np.all(dev[~tight] <= 1e-9 * np.abs(full).max())
        z = dev[tight] / se[tight]
        assert z.max() <= 5.0, z.max()
        assert np.mean(z > 4.0) <= 1e-3
