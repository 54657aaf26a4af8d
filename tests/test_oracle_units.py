"""Pins of the oracle at key-unit granularity (AB-Attention page, section «Три приёма
AB-Attention», third technique: key/value selection units of 4 tokens gathered into
full tensor-core tiles). Every check compares the oracle with an independent
computation: a reshape-mean, a scipy softmax, or fp64 SDPA over an explicit key mask."""

import numpy as np
import pytest
import torch
from scipy.special import softmax

U = 4


def _qkv(seed=0, B=1, H=2, N=300, d=64, scale=1.5):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    x = [torch.zeros(B, H, N_pad, d, dtype=torch.bfloat16) for _ in range(3)]
    for t, s in zip(x, (scale, scale, 1.0)):
        t[:, :, :N] = (torch.randn(B, H, N, d, generator=g) * s).to(torch.bfloat16)
    return x[0], x[1], x[2], N


def _sdpa_masked(q, k, v, N, keep):
    """fp64 attention of every row over the keys where keep[b, h, qb, t] is True."""
    B, H, N_pad, d = q.shape
    qf, kf, vf = (t.double() for t in (q, k, v))
    logits = torch.einsum("bhid,bhjd->bhij", qf, kf) / np.sqrt(d)
    m = keep.repeat_interleave(128, dim=2)  # [B, H, N_pad (rows), N_pad (keys)]
    logits = logits.masked_fill(~m, float("-inf"))
    p = torch.softmax(logits, dim=-1)
    out = torch.einsum("bhij,bhjd->bhid", torch.nan_to_num(p), vf)
    out[:, :, N:] = 0
    return out.numpy()


def test_unit_mean_key_is_the_mean_of_each_4_token_unit(orc):
    q, k, v, N = _qkv(1, N=299)  # last unit has 3 valid tokens, units past it are empty
    kb = orc.mean_key(k, N, unit=U)
    B, H, N_pad, d = k.shape
    kf = k.double().clone()
    valid = (torch.arange(N_pad) < N).double().view(1, 1, N_pad, 1)
    sums = (kf * valid).view(B, H, N_pad // U, U, d).sum(3)
    counts = valid.view(1, 1, N_pad // U, U, 1).sum(3)
    ref = torch.where(counts > 0, sums / counts.clamp(min=1), torch.zeros_like(sums))
    np.testing.assert_allclose(kb, ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(kb[:, :, -(N_pad // U - (N + U - 1) // U):] == 0)


def test_unit_scores_mean_pooled_case_is_a_softmax_over_existing_units(orc):
    q, k, v, N = _qkv(2, N=301)
    B, H, N_pad, d = k.shape
    n_valid = (N + U - 1) // U
    s = orc.ibcs_scores(q, k, N, C=1, T=1, unit=U)
    kb = orc.mean_key(k, N, unit=U)
    for h in range(H):
        for qb in range(N_pad // 128):
            rows = q[0, h, qb * 128:(qb + 1) * 128].double().numpy()
            nv = min(128, N - qb * 128)
            qm = rows[:nv].mean(0)
            ref = softmax(kb[0, h, :n_valid] @ qm / np.sqrt(d))
            np.testing.assert_allclose(s[0, h, qb, :n_valid], ref, rtol=1e-10, atol=1e-15)
            assert np.all(s[0, h, qb, n_valid:] == 0)


def test_unit_scores_rows_sum_to_one(orc):
    q, k, v, N = _qkv(3, N=383)
    s = orc.ibcs_scores(q, k, N, C=8, T=5, unit=U)
    np.testing.assert_allclose(s.sum(-1), 1.0, rtol=1e-12)


def test_unit_attention_with_every_unit_is_dense_attention(orc):
    q, k, v, N = _qkv(4, N=290)
    B, H, N_pad, d = q.shape
    nku = N_pad // U
    nqb = N_pad // 128
    idx = np.tile(np.arange(nku, dtype=np.int32), (B, H, nqb, 1))
    cnt = np.full((B, H, nqb), nku, dtype=np.int32)
    out, _, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, unit=U)
    keep = torch.zeros(B, H, nqb, N_pad, dtype=torch.bool)
    keep[..., :N] = True
    ref = _sdpa_masked(q, k, v, N, keep).reshape(B * H * nqb, 128, d)
    np.testing.assert_allclose(out, ref, atol=1e-12)


@pytest.mark.parametrize("weighted", [False, True])
def test_unit_attention_on_a_random_selection_matches_masked_sdpa(orc, weighted):
    q, k, v, N = _qkv(5, N=333)
    B, H, N_pad, d = q.shape
    nku, nqb = N_pad // U, N_pad // 128
    rng = np.random.default_rng(5)
    idx = np.full((B, H, nqb, nku), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    w = np.zeros((B, H, nqb, nku), dtype=np.float32)
    keep = torch.zeros(B, H, nqb, N_pad, dtype=torch.bool)
    dup = {}
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                sel = np.sort(rng.choice((N + U - 1) // U, size=37, replace=False))
                idx[b, h, qb, :37] = sel
                cnt[b, h, qb] = 37
                w[b, h, qb, :37] = 1.0
                if weighted:  # one unit counts twice (weight 2 = its keys duplicated)
                    w[b, h, qb, 5] = 2.0
                    dup[(b, h, qb)] = sel[5]
                for j in sel:
                    keep[b, h, qb, j * U:min(N, j * U + U)] = True
    out, _, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, w if weighted else None, unit=U)
    if not weighted:
        ref = _sdpa_masked(q, k, v, N, keep).reshape(B * H * nqb, 128, d)
        np.testing.assert_allclose(out, ref, atol=1e-12)
        return
    # weight 2 on a unit = the same softmax with that unit's keys present twice
    for (b, h, qb), j in dup.items():
        toks = torch.nonzero(keep[b, h, qb]).flatten().tolist()
        toks += list(range(j * U, min(N, j * U + U)))
        qf = q[b, h, qb * 128:(qb + 1) * 128].double()
        kf, vf = k[b, h, toks].double(), v[b, h, toks].double()
        p = torch.softmax(qf @ kf.T / np.sqrt(d), dim=-1)
        ref = (p @ vf).numpy()
        nv = min(128, N - qb * 128)
        r = (b * H + h) * nqb + qb
        np.testing.assert_allclose(out[r, :nv], ref[:nv], atol=1e-12)
