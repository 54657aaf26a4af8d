"""Pins of the oracle's SIP and top-k selection and of its Philox4x32-10 generator.

The AB-Attention news page, section «Три приёма AB-Attention» (SIP), fixes: inclusion
probability proportional to the score, the most important blocks always taken, every
other block with a nonzero chance, and each kept block weighted by the inverse
probability ("a block with probability 25% counts as four"). The section «Где
ломаются прежние разреженные схемы» describes top-k selection.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _row(scores):
    return np.asarray(scores, dtype=np.float32).reshape(1, 1, 1, -1)


def test_sip_hand_worked(orc):
    g = json.load(open(os.path.join(GOLD, "sip_hand.json")))
    for case in g["cases"]:
        s = _row(case["scores"])
        for seed in range(64):
            idx, cnt, w, p, bad = orc.sip(s, case["K"], seed)
            assert bad.sum() == 0
            np.testing.assert_array_equal(p[0, 0, 0], case["p"], err_msg=case["name"])
            kept = idx[0, 0, 0, : cnt[0, 0, 0]]
            assert np.all(np.diff(kept) > 0)
            for j in case["saturated"]:
                assert j in kept, (case["name"], seed)
            for c, j in enumerate(kept):
                assert w[0, 0, 0, c] == np.float32(case["w"][j])
            assert np.all(idx[0, 0, 0, cnt[0, 0, 0]:] == -1)


def exact_water_fill(scores, K):
    """Independent exact rational water-filling (textbook form): sort the fixed-point
    scores u_j = floor(s_j 2^50) descending and take the smallest m such that, with the
    top m blocks saturated and c = (K - m) / (sum of the others), the largest remaining
    block has c u <= 1. Returns (top-m set, exact probabilities min(1, c u_j))."""
    u = [int(Fraction(float(x)) * 2**50) for x in scores]  # floor of the exact value
    n = len(u)
    positive = [j for j in range(n) if u[j] > 0]
    if len(positive) <= K:
        return set(positive), [Fraction(1) if u[j] > 0 else Fraction(0) for j in range(n)]
    order = sorted(range(n), key=lambda j: (-u[j], j))
    for m in range(K):
        rest = sum(u[order[i]] for i in range(m, n))
        c = Fraction(K - m, rest)
        if c * u[order[m]] <= 1:
            S = set(order[:m])
            return S, [Fraction(1) if j in S else min(Fraction(1), c * u[j]) for j in range(n)]
    raise AssertionError("no water level found")


def test_sip_matches_exact_rational_water_filling(orc):
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(2, 40))
        K = int(rng.integers(1, n + 1))
        kind = trial % 3
        if kind == 0:
            s = rng.dirichlet(np.ones(n) * 0.3)
        elif kind == 1:
            s = rng.exponential(size=n)
            s = s / s.sum()
            s[rng.integers(0, n)] = 0.0
        else:
            s = np.exp(rng.standard_normal(n) * 4)
            s = s / s.sum()
        s = s.astype(np.float32)
        S, p_exact = exact_water_fill(s, K)
        idx, cnt, w, p, bad = orc.sip(_row(s), K, trial)
        assert bad.sum() == 0
        got = p[0, 0, 0]
        assert set(np.nonzero(got == 1.0)[0]) >= S
        for j in range(n):
            if j in S:
                assert got[j] == 1.0
            else:
                # two roundings to double before the divide: within 2 ulp of exact
                assert abs(Fraction(float(got[j])) - p_exact[j]) <= 2 * np.spacing(float(p_exact[j])) + 0, (trial, j)
        feasible = np.count_nonzero(s) > K
        if feasible:
            assert abs(got.sum() - K) <= 1e-9 * K
        # monotone in the score
        order = np.argsort(-s, kind="stable")
        assert np.all(np.diff(got[order]) <= 1e-15)


def test_sip_probabilities_are_valid_and_sum_to_budget(orc):
    rng = np.random.default_rng(11)
    s = rng.dirichlet(np.ones(256) * 0.5, size=(2, 3, 5)).astype(np.float32)
    idx, cnt, w, p, bad = orc.sip(s, 26, 123)
    assert bad.sum() == 0
    assert np.all(p > 0) and np.all(p <= 1)
    np.testing.assert_allclose(p.sum(-1), 26, rtol=1e-9)
    # every kept block carries w = fl32(1/p)
    for r in np.ndindex(2, 3, 5):
        kept = idx[r][: cnt[r]]
        np.testing.assert_array_equal(w[r][: cnt[r]], (1.0 / p[r][kept]).astype(np.float32))


def test_sip_inclusion_frequency(orc):
    """Empirical inclusion frequency over 10^4 seeds is within 5 binomial sigma of p_j,
    and saturated blocks are kept in every draw."""
    rng = np.random.default_rng(3)
    s = rng.dirichlet(np.ones(16) * 0.4, size=(1, 1, 2)).astype(np.float32)
    K = 5
    hits = np.zeros((2, 16))
    n = 10_000
    p0 = None
    for seed in range(n):
        idx, cnt, w, p, bad = orc.sip(s, K, seed)
        if p0 is None:
            p0 = p[0, 0]
        for r in range(2):
            hits[r, idx[0, 0, r, : cnt[0, 0, r]]] += 1
    freq = hits / n
    sigma = np.sqrt(p0 * (1 - p0) / n)
    assert np.all(np.abs(freq - p0) <= 5 * sigma + 1e-12)
    assert np.all(freq[p0 == 1.0] == 1.0)


def test_sip_rejects_bad_scores(orc):
    for bad_val in (np.nan, np.inf, -0.5, 3.0):
        s = _row([0.5, bad_val, 0.25])
        idx, cnt, w, p, bad = orc.sip(s, 2, 0)
        assert bad[0, 0, 0] == 1 and cnt[0, 0, 0] == 0
        assert np.all(idx == -1)


def test_sip_rejects_rows_whose_exact_sum_overflows(orc):
    # 8192 scores of 2.0: U = 8192 * 2^51 = 2^64 does not fit in 64 bits, so the row is
    # invalid (the integers of the water-filling would wrap); one score less fits.
    s = np.full((1, 1, 2, 8192), 2.0, dtype=np.float32)
    s[0, 0, 1, 0] = 1.75
    idx, cnt, w, p, bad = orc.sip(s, 100, 0)
    assert bad[0, 0, 0] == 1 and cnt[0, 0, 0] == 0 and np.all(idx[0, 0, 0] == -1)
    assert bad[0, 0, 1] == 0 and cnt[0, 0, 1] > 0
    # nearly equal scores: p ~ K / n for each block and sum p = K
    assert abs(p[0, 0, 1].sum() - 100) <= 1e-9 * 100
    np.testing.assert_allclose(p[0, 0, 1, 1:], 100 / 8192, rtol=1e-3)


def test_topk_reference_cases(orc):
    s = _row([0.1, 0.3, 0.3, 0.05, 0.25])
    idx, cnt, w = orc.topk(s, 2)
    assert cnt[0, 0, 0] == 2
    np.testing.assert_array_equal(idx[0, 0, 0, :2], [1, 2])
    idx, cnt, w = orc.topk(s, 3)
    np.testing.assert_array_equal(idx[0, 0, 0, :3], [1, 2, 4])
    # ties go to the lower index
    s = _row([0.2, 0.2, 0.2, 0.2])
    idx, cnt, w = orc.topk(s, 2)
    np.testing.assert_array_equal(idx[0, 0, 0, :2], [0, 1])
    # budget >= blocks selects everything
    idx, cnt, w = orc.topk(s, 9)
    assert cnt[0, 0, 0] == 4
    np.testing.assert_array_equal(idx[0, 0, 0], [0, 1, 2, 3])
    assert np.all(w[0, 0, 0] == 1.0)


def test_topk_matches_numpy_argsort(orc):
    rng = np.random.default_rng(9)
    s = rng.random((2, 2, 4, 100)).astype(np.float32)
    s[..., 10] = s[..., 11]  # a tie
    idx, cnt, w = orc.topk(s, 17)
    for r in np.ndindex(2, 2, 4):
        order = np.lexsort((np.arange(100), -s[r]))
        np.testing.assert_array_equal(idx[r][:17], np.sort(order[:17]))


_TRITON_PHILOX = r"""
import json, os, sys
os.environ["TRITON_INTERPRET"] = "1"
import numpy as np
import torch
import triton
import triton.language as tl


@triton.jit
def _philox_kernel(out_ptr, c0_ptr, c1_ptr, c2_ptr, c3_ptr, seed, n: tl.constexpr):
    offs = tl.arange(0, n)
    c0 = tl.load(c0_ptr + offs)
    c1 = tl.load(c1_ptr + offs)
    c2 = tl.load(c2_ptr + offs)
    c3 = tl.load(c3_ptr + offs)
    a, b, c, d = tl.philox(seed, c0, c1, c2, c3)
    tl.store(out_ptr + offs * 4 + 0, a)
    tl.store(out_ptr + offs * 4 + 1, b)
    tl.store(out_ptr + offs * 4 + 2, c)
    tl.store(out_ptr + offs * 4 + 3, d)


req = json.loads(sys.stdin.read())
res = []
for item in req:
    ctr = np.asarray(item["ctr"], dtype=np.uint64).astype(np.uint32)  # [4, n]
    n = ctr.shape[1]
    cs = [torch.from_numpy(ctr[i].view(np.int32).copy()) for i in range(4)]
    out = torch.zeros(4 * n, dtype=torch.int32)
    seed = item["seed"]
    _philox_kernel[(1,)](out, *cs, seed if seed < 2**63 else seed - 2**64, n=n)
    res.append(out.numpy().view(np.uint32).reshape(n, 4).tolist())
print(json.dumps(res))
"""


def test_philox_matches_independent_implementation(orc):
    """The oracle's Philox4x32-10 against Triton's tl.philox run in Triton's CPU
    interpreter, in a subprocess: an independent implementation of the same published
    generator (Salmon et al., SC'11). Key = (lo32 seed, hi32 seed), 4-word counter."""
    import json
    import subprocess
    import sys

    rng = np.random.default_rng(0)
    n = 16
    req = []
    for seed in (0, 1, 0x123456789ABCDEF0, 2**64 - 1):
        ctr = rng.integers(0, 2**32, size=(4, n), dtype=np.uint64)
        ctr[:, 0] = 0
        ctr[:, 1] = [5, 3, 2, 1]  # (kb, qb, h, b)-style small counters
        req.append({"seed": seed, "ctr": ctr.tolist()})
    env = dict(os.environ, TRITON_INTERPRET="1")
    out = subprocess.run([sys.executable, "-c", _TRITON_PHILOX], input=json.dumps(req),
                         capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    for item, ref in zip(req, res):
        seed = item["seed"]
        key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32)
        ctr = np.asarray(item["ctr"], dtype=np.uint64).astype(np.uint32)
        for i in range(n):
            np.testing.assert_array_equal(orc.philox4x32_10(ctr[:, i], key),
                                          np.asarray(ref[i], dtype=np.uint32))
