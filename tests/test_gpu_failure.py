"""Failure detection without a GPU fault: an in-kernel wait on an mbarrier that nothing
completes must give up after its limit, report AB_FLAG_TIMEOUT through the device flag
and return, leaving the CUDA context usable for the next call (the bounded wait every
pipeline role of the library uses). The attention kernel itself is run with its waits
limited to 1 us, so that its own unwind path (drains, softmax loops run out, tensor
memory freed) runs and the next call on the same context still gives the right result."""

import time

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    ab.lib()


def test_wait_that_nothing_completes_times_out_and_reports():
    t0 = time.perf_counter()
    bits, done = ab.selftest_bounded_wait(20000, complete=False)  # 20 ms limit
    elapsed = time.perf_counter() - t0
    assert bits & ab.FLAG_TIMEOUT
    assert done == 2
    assert elapsed < 5.0


def test_completed_wait_reports_nothing():
    bits, done = ab.selftest_bounded_wait(20000, complete=True)
    assert bits == 0
    assert done == 1


def test_context_stays_usable_after_a_timeout(orc):
    ab.selftest_bounded_wait(5000, complete=False)
    # a normal attention call afterwards still matches the oracle
    g = torch.Generator().manual_seed(0)
    N, d = 300, 64
    q, k, v = (torch.zeros(1, 1, 384, d, dtype=torch.bfloat16) for _ in range(3))
    for t in (q, k, v):
        t[:, :, :N] = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    idx = torch.tensor([[[[0, 1, 2], [0, 2, -1], [1, -1, -1]]]], dtype=torch.int32)
    cnt = torch.tensor([[[3, 2, 1]]], dtype=torch.int32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ab.attn_topk_fwd(q.cuda(), k.cuda(), v.cuda(), N, idx.cuda(), cnt.cuda(), dev_flag=flag,
                           out_dtype=torch.float32)
    assert ab.check_flag(flag) == 0
    ref, _, _, _ = orc.attn_rows(q, k, v, N, idx.numpy(), cnt.numpy())
    np.testing.assert_allclose(out.cpu().numpy().reshape(3, 128, d), ref, atol=1e-2)


def test_selftest_argument_checks():
    L = ab.lib()
    assert L.ab_selftest_bounded_wait(0, 0, None, None, None) == 1
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.ab_selftest_bounded_wait(0, 0, ab._ptr(flag), ab._ptr(flag), None) == 5


def _attn_with_limit(q, k, v, N, idx, cnt, w, unit, limit_ns):
    """ab_selftest_attn_wait_limit through the C ABI: the attention call with every wait
    inside the kernel limited to limit_ns; returns (flag bits, out)."""
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    code = ab.lib().ab_selftest_attn_wait_limit(
        ab._ptr(q), ab._ptr(k), ab._ptr(v), ab.make_shape(q, N), unit, ab._ptr(idx), ab._ptr(cnt),
        ab._ptr(w), ab._ptr(out), ab.AB_F32, None, ab._ptr(flag), int(limit_ns), ab._stream())
    assert code == 0, ab.STATUS.get(code, code)
    return ab.check_flag(flag), out


@pytest.mark.parametrize("unit", [128, 4])
def test_attention_wait_limit_runs_out(orc, unit):
    # the attention kernel's own waits (TMA tiles, MMAs, the item ring) given 1 us: with
    # more items than CTAs each CTA's item scheduler waits for its TMA warp to start the
    # next item, which takes far longer, so that wait gives up; the flag reports it,
    # every CTA unwinds and returns, and the next call on the same context matches the
    # oracle
    g = torch.Generator().manual_seed(11)
    N, H, d = 2000, 12, 128
    N_pad = (N + 127) // 128 * 128
    q, k, v = (torch.zeros(1, H, N_pad, d, dtype=torch.bfloat16) for _ in range(3))
    for t in (q, k, v):
        t[:, :, :N] = torch.randn(1, H, N, d, generator=g).to(torch.bfloat16)
    nkb = N_pad // unit
    n_valid = -(-N // unit)
    nqb = N_pad // 128
    rng = np.random.default_rng(unit)
    idx = np.full((1, H, nqb, nkb), -1, dtype=np.int32)
    cnt = np.zeros((1, H, nqb), dtype=np.int32)
    w = np.zeros((1, H, nqb, nkb), dtype=np.float32)
    for h in range(H):
        for qb in range(nqb):
            c = int(rng.integers(min(n_valid, 200) // 2, min(n_valid, 200) + 1))
            idx[0, h, qb, :c] = np.sort(rng.choice(n_valid, c, replace=False))
            cnt[0, h, qb] = c
            w[0, h, qb, :c] = rng.uniform(1.0, 3.0, c)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    # a generous limit: nothing gives up and the result is right
    bits, good = _attn_with_limit(qc, kc, vc, N, ic, cc, wc, unit, 1_000_000_000)
    assert bits == 0
    t0 = time.perf_counter()
    bits, _ = _attn_with_limit(qc, kc, vc, N, ic, cc, wc, unit, 1000)
    assert time.perf_counter() - t0 < 10.0
    assert bits & ab.FLAG_TIMEOUT and not bits & ~(ab.FLAG_TIMEOUT | ab.FLAG_BAD_INDEX)
    # the context is usable: the normal call gives the result it gave before
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    again = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, dev_flag=flag, out_dtype=torch.float32, unit=unit)
    assert ab.check_flag(flag) == 0
    assert torch.equal(again, good)
    rows = np.arange(0, H * nqb, 7, dtype=np.int64)
    ref, _, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, w, rows=rows, unit=unit)
    got = good.cpu().numpy().reshape(H * nqb, 128, d)[rows]
    assert np.abs(got - ref).max() <= 1e-2


def test_attention_wait_limit_argument_checks():
    L = ab.lib()
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    s = ab.Shape(1, 1, 128, 128, 64, ab.AB_BF16)
    p = ab._ptr(z)
    assert L.ab_selftest_attn_wait_limit(p, p, p, s, 128, p, p, p, p, ab.AB_F32, None, None, 1000, None) == 1
    assert L.ab_selftest_attn_wait_limit(p, p, p, s, 128, p, p, p, p, ab.AB_F32, None, p, 0, None) == 5


def test_backward_wait_limit_runs_out(orc):
    # the attention backward's own waits (TMA tiles, MMAs, the compute warps' handovers)
    # given 1 ns: a wait not satisfied at its first poll gives up at the next tick of the
    # GPU's global timer; the flag reports it, every CTA lets its copies and MMAs land,
    # frees its tensor memory and returns, and the next call on the same context gives
    # the result it gave before, which matches the oracle's gradient
    g = torch.Generator().manual_seed(5)
    N, H, d = 2000, 4, 128
    N_pad = (N + 127) // 128 * 128
    nb = N_pad // 128
    q, k, v, do = (torch.zeros(1, H, N_pad, d, dtype=torch.bfloat16) for _ in range(4))
    for t in (q, k, v, do):
        t[:, :, :N] = torch.randn(1, H, N, d, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(3)
    idx = np.full((1, H, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((1, H, nb), dtype=np.int32)
    w = np.zeros((1, H, nb, nb), dtype=np.float32)
    for h in range(H):
        for qb in range(nb):
            c = int(rng.integers(3, 9))
            idx[0, h, qb, :c] = np.sort(rng.choice(nb, c, replace=False))
            cnt[0, h, qb] = c
            w[0, h, qb, :c] = rng.uniform(1.0, 3.0, c)
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, do))
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    out, lse = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, want_lse=True)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    good = ab.attn_bwd(qc, kc, vc, N, ic, cc, wc, out, lse, gc, dev_flag=flag,
                       wait_limit_ns=1_000_000_000)
    assert ab.check_flag(flag) == 0
    t0 = time.perf_counter()
    flag.zero_()
    ab.attn_bwd(qc, kc, vc, N, ic, cc, wc, out, lse, gc, dev_flag=flag, wait_limit_ns=1)
    bits = ab.check_flag(flag)
    assert time.perf_counter() - t0 < 10.0
    assert bits & ab.FLAG_TIMEOUT and not bits & ~ab.FLAG_TIMEOUT
    flag.zero_()
    again = ab.attn_bwd(qc, kc, vc, N, ic, cc, wc, out, lse, gc, dev_flag=flag)
    assert ab.check_flag(flag) == 0
    for a, b in zip(again, good):
        assert torch.equal(a, b)
    ref = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    for got, r in zip(good, ref):
        got = got.double().cpu().numpy()
        assert np.linalg.norm(got - r) <= 1e-2 * np.linalg.norm(r)
