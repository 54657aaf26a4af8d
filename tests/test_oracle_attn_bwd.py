"""Pins of the oracle's attention backward (gradients with respect to Q, K and V).

The AB-Attention news page, section «Три приёма AB-Attention» (SIP): the kept blocks
enter ordinary softmax attention with the logit shifted by ln(1/p) = ln w. The gradient
of that function with respect to Q, K and V is fixed by the forward alone, so the
oracle's hand-written backward is checked against torch autograd in fp64 of the same
function written densely (a log-weight bias on kept blocks, -inf elsewhere), and against
two closed forms: the softmax is invariant to a shift of a row's logits, so the key
gradients of a head sum to zero, and each row's probabilities sum to one, so the value
gradients of a head sum to the sum of the upstream gradient rows. The value gradient is
also tied to the separately written forward oracle: O is linear in V, so an exact change
of one value changes the loss by exactly that change times its gradient.
"""

import math

import numpy as np
import pytest
import torch


def _inputs(N, H, d, seed, B=1, scale=1.5):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    out = []
    for s in (scale, scale, 1.0, 1.0):
        t = torch.zeros(B, H, N_pad, d)
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g) * s
        out.append(t.to(torch.bfloat16))
    return out  # q, k, v, dO


def _plan(B, H, nb, budget, seed, weighted=True, empty_row=None):
    """A random plan: `budget` distinct ascending blocks per row, weights in [1, 6)."""
    rng = np.random.default_rng(seed)
    idx = np.full((B, H, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nb), dtype=np.int32)
    w = np.zeros((B, H, nb, nb), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for qb in range(nb):
                if empty_row == (b, h, qb):
                    continue
                k = min(budget, nb)
                sel = np.sort(rng.choice(nb, size=k, replace=False))
                idx[b, h, qb, :k] = sel
                cnt[b, h, qb] = k
                w[b, h, qb, :k] = rng.uniform(1.0, 6.0, size=k).astype(np.float32) if weighted else 1.0
    return idx, cnt, (w if weighted else None)


def _autograd(q, k, v, do, N, idx, cnt, w):
    """fp64 autograd of the dense masked attention with ln w on the kept blocks."""
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    bias = torch.full((B, H, N_pad, N_pad), -math.inf, dtype=torch.float64)
    row_ok = torch.zeros((B, H, N_pad), dtype=torch.bool)
    for b in range(B):
        for h in range(H):
            for qb in range(nb):
                for c in range(int(cnt[b, h, qb])):
                    j = int(idx[b, h, qb, c])
                    lw = 0.0 if w is None else math.log(float(w[b, h, qb, c]))
                    bias[b, h, qb * 128:(qb + 1) * 128, j * 128:(j + 1) * 128] = lw
    bias[:, :, :, N:] = -math.inf
    row_ok[:, :, :N] = torch.isfinite(bias[:, :, :N]).any(-1)
    bias[~row_ok] = 0.0  # rows left out of the loss: any finite logits
    qf, kf, vf = (t.double().requires_grad_(True) for t in (q, k, v))
    logits = torch.einsum("bhid,bhjd->bhij", qf, kf) / math.sqrt(d) + bias
    out = torch.softmax(logits, -1) @ vf
    g = do.double() * row_ok[..., None]
    (out * g).sum().backward()
    return qf.grad.numpy(), kf.grad.numpy(), vf.grad.numpy(), row_ok.numpy()


CASES = [
    # N, H, d, budget, weighted, empty row
    (3 * 128 + 50, 2, 64, 2, True, None),
    (4 * 128, 1, 128, 3, False, None),
    (5 * 128 + 1, 2, 64, 3, True, (0, 1, 2)),
    (2 * 128 + 127, 1, 128, 3, True, None),
]


@pytest.mark.parametrize("case", CASES)
def test_bwd_matches_autograd(orc, case):
    N, H, d, budget, weighted, empty = case
    q, k, v, do = _inputs(N, H, d, seed=N + d)
    nb = q.shape[2] // 128
    idx, cnt, w = _plan(1, H, nb, budget, seed=7 * N, weighted=weighted, empty_row=empty)
    dq, dk, dv = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    rq, rk, rv, row_ok = _autograd(q, k, v, do, N, idx, cnt, w)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)
    # padding rows / keys and an empty row carry no gradient
    assert np.all(dq[:, :, N:] == 0) and np.all(dk[:, :, N:] == 0) and np.all(dv[:, :, N:] == 0)
    if empty is not None:
        b, h, qb = empty
        assert np.all(dq[b, h, qb * 128:(qb + 1) * 128] == 0)


@pytest.mark.parametrize("weighted", [True, False])
def test_bwd_closed_forms(orc, weighted):
    N, H, d = 3 * 128 + 77, 2, 64
    q, k, v, do = _inputs(N, H, d, seed=11)
    nb = q.shape[2] // 128
    idx, cnt, w = _plan(1, H, nb, 2, seed=3, weighted=weighted, empty_row=(0, 0, 1))
    dq, dk, dv = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    # shift invariance of each row's softmax: sum over keys of dK is zero per head
    sdk = dk.sum(axis=2)
    assert np.abs(sdk).max() < 1e-10 * max(1.0, np.abs(dk).max())
    # probabilities sum to one: sum over keys of dV = sum over rows with a non-empty
    # selection of dO
    g = do.double().numpy().copy()
    g[:, :, N:] = 0
    g[0, 0, 128:256] = 0
    np.testing.assert_allclose(dv.sum(axis=2), g.sum(axis=2), rtol=1e-11, atol=1e-11)


def test_bwd_weight_is_block_multiplicity(orc):
    """A block kept with w = 2 has the gradients of two identical copies of it, and a
    block kept with w = 1 those of one copy: the weight is a multiplicity (the
    Horvitz-Thompson reading), checked against autograd of the duplicated keys."""
    N, H, d = 3 * 128, 1, 64
    q, k, v, do = _inputs(N, H, d, seed=5)
    nb = 3
    idx = np.full((1, 1, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((1, 1, nb), dtype=np.int32)
    w = np.zeros((1, 1, nb, nb), dtype=np.float32)
    for qb in range(nb):
        idx[0, 0, qb, :2] = [0, 2]
        cnt[0, 0, qb] = 2
        w[0, 0, qb, :2] = [2.0, 1.0]
    dq, dk, dv = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    # dense reference over keys [block 0, block 0, block 2]
    qf, kf, vf = (t.double().requires_grad_(True) for t in (q, k, v))
    kk = torch.cat([kf[:, :, 0:128], kf[:, :, 0:128], kf[:, :, 256:384]], 2)
    vv = torch.cat([vf[:, :, 0:128], vf[:, :, 0:128], vf[:, :, 256:384]], 2)
    att = torch.softmax(torch.einsum("bhid,bhjd->bhij", qf, kk) / math.sqrt(d), -1) @ vv
    (att * do.double()).sum().backward()
    np.testing.assert_allclose(dq, qf.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kf.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vf.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_bwd_dv_is_the_forward_oracles_derivative(orc):
    """O is linear in V, so doubling one value v of V (exact in bf16) changes the loss
    L = sum_i dO_i . O_i by exactly v * dL/dv. The separately written forward oracle
    gives both losses; the backward oracle's dV must equal their difference over v."""
    N, H, d = 3 * 128 + 40, 1, 64
    q, k, v, do = _inputs(N, H, d, seed=21)
    nb = q.shape[2] // 128
    idx, cnt, w = _plan(1, H, nb, 2, seed=9, weighted=True)
    _, _, dv = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    g = do.double().numpy()[0, 0]

    def loss(vv):
        out, _, _, _ = orc.attn_rows(q, k, vv, N, idx, cnt, w)
        o = out.reshape(nb * 128, d)
        return float((o[:N] * g[:N]).sum())

    base = loss(v)
    checked = 0
    for t, e in ((5, 3), (130, 17), (300, 63), (N - 1, 0)):
        val = float(v[0, 0, t, e].float())
        if val == 0.0:
            continue
        v2 = v.clone()
        v2[0, 0, t, e] = torch.tensor(2.0 * val).to(torch.bfloat16)
        assert float(v2[0, 0, t, e].float()) == 2.0 * val
        fd = (loss(v2) - base) / val
        assert abs(fd - dv[0, 0, t, e]) <= 1e-9 * max(1.0, abs(dv[0, 0, t, e]))
        checked += 1
    assert checked >= 3
