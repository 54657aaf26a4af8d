"""GPU parity of the attention kernel's dynamic item scheduling against the oracle.

The kernel runs one persistent CTA per SM; each CTA starts with item blockIdx.x and
claims further (b, h, query block) items from a global counter, writes the output of
empty items itself and hands the others to its roles through a ring in shared memory.
Small problems give every CTA a single item, so these tests use more items than SMs
(up to several per CTA), with many empty items, ragged counts and unit plans, and check
every row against the oracle with the bounds of tests/test_gpu_parity.py. A run of more
launches than there are claim slots checks that every reuse of a slot starts clean, and
two calls forced onto one slot while both run check that the sharing is flagged.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab

pytestmark = pytest.mark.gpu

ATOL_MAX = 1e-2
RTOL_FRO = 5e-3
LSE_ATOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


def _inputs(N, H, d=128, B=1, seed=0):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    x = [torch.zeros(B, H, N_pad, d) for _ in range(3)]
    for t in x:
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g)
    return [t.to(torch.bfloat16) for t in x]


def _half_ulp_bf16(x):
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def _plan(B, H, nqb, nkb, n_valid, max_cnt, p_empty, seed):
    """Random sorted selections of 0..max_cnt entries per row (a share p_empty empty),
    entries below n_valid, weights in [1, 4)."""
    rng = np.random.default_rng(seed)
    idx = np.full((B, H, nqb, nkb), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    w = np.zeros((B, H, nqb, nkb), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                c = 0 if rng.random() < p_empty else int(rng.integers(1, max_cnt + 1))
                sel = np.sort(rng.choice(n_valid, size=c, replace=False))
                idx[b, h, qb, :c] = sel
                cnt[b, h, qb] = c
                w[b, h, qb, :c] = rng.uniform(1.0, 4.0, c)
    return idx, cnt, w


def _check(orc, q, k, v, N, idx, cnt, w, out, lse, unit):
    B, H, N_pad, d = q.shape
    nqb = N_pad // 128
    rows = np.arange(B * H * nqb, dtype=np.int64)
    ref, ref_lse, _, _ = orc.attn_rows(q, k, v, N, idx, cnt, w, rows=rows, unit=unit)
    og = out.float().cpu().numpy().reshape(B * H * nqb, 128, d)
    lg = lse.cpu().numpy().reshape(B * H * nqb, 128)
    diff = np.abs(og - ref)
    if out.dtype == torch.float32:
        assert diff.max() <= ATOL_MAX, diff.max()
    else:
        assert (diff - _half_ulp_bf16(ref)).max() <= ATOL_MAX
    assert np.linalg.norm(og - ref) / np.linalg.norm(ref) <= RTOL_FRO
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lg))
    assert np.all(lg[~fin] == ref_lse[~fin])
    assert np.abs(lg[fin] - ref_lse[fin]).max(initial=0) <= LSE_ATOL


@pytest.mark.parametrize("weighted", [True, False])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_many_items_per_cta_blocks(orc, weighted, out_dtype):
    # 16 heads x 40 query blocks = 640 items (about 4 per CTA), a third of them empty,
    # 1..3 key blocks each, ragged sequence end
    N, H = 5100, 16
    q, k, v = _inputs(N, H, seed=21)
    B, _, N_pad, d = q.shape
    nqb = nkb = N_pad // 128
    idx, cnt, w = _plan(B, H, nqb, nkb, nkb, 3, 0.35, seed=5)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    if weighted:
        out, lse = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, want_lse=True, dev_flag=flag,
                               out_dtype=out_dtype)
    else:
        out, lse = ab.attn_topk_fwd(qc, kc, vc, N, ic, cc, want_lse=True, dev_flag=flag,
                                    out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    _check(orc, q, k, v, N, idx, cnt, w if weighted else None, out, lse, unit=128)


def test_many_items_per_cta_units(orc):
    # 4-token units: 12 heads x 24 query blocks = 288 items, a quarter empty, 1..70 units
    # (up to 3 tiles of 32 units) each
    N, H, U = 3070, 12, 4
    q, k, v = _inputs(N, H, seed=22)
    B, _, N_pad, d = q.shape
    nqb, nku = N_pad // 128, N_pad // U
    idx, cnt, w = _plan(B, H, nqb, nku, (N + U - 1) // U, 70, 0.25, seed=6)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, want_lse=True, dev_flag=flag,
                           out_dtype=torch.float32, unit=U)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    _check(orc, q, k, v, N, idx, cnt, w, out, lse, unit=U)


def test_all_items_empty_but_one(orc):
    # every CTA but one finds only empty items: outputs 0, lse -inf (0 on padding rows)
    N, H = 4000, 12
    q, k, v = _inputs(N, H, seed=23)
    B, _, N_pad, d = q.shape
    nqb = nkb = N_pad // 128
    idx = np.full((B, H, nqb, nkb), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    idx[0, H - 1, nqb - 1, :2] = [0, nkb - 1]
    cnt[0, H - 1, nqb - 1] = 2
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    ic, cc = (torch.from_numpy(a).cuda() for a in (idx, cnt))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = ab.attn_topk_fwd(qc, kc, vc, N, ic, cc, want_lse=True, dev_flag=flag,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    _check(orc, q, k, v, N, idx, cnt, None, out, lse, unit=128)


def test_counter_slots_wrap(orc):
    # more launches than counter slots (4096): every slot is reused, so a counter left
    # non-zero by an earlier launch would skip items (stale output) in a later one
    N, H = 2000, 16
    q, k, v = _inputs(N, H, seed=24)
    B, _, N_pad, d = q.shape
    nqb = nkb = N_pad // 128
    idx, cnt, w = _plan(B, H, nqb, nkb, nkb, 2, 0.2, seed=7)
    qc, kc, vc = (t.cuda() for t in (q, k, v))
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, H, N_pad, d, dtype=torch.float32, device="cuda")
    first, lse = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, want_lse=True, dev_flag=flag,
                             out_dtype=torch.float32)
    for _ in range(4096 + 7):
        out.fill_(float("nan"))
        ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, dev_flag=flag, out=out, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    assert torch.equal(out, first)
    _check(orc, q, k, v, N, idx, cnt, w, first, lse, unit=128)


def test_calls_sharing_a_claim_slot_are_flagged_or_correct(orc):
    # Two calls forced onto the same claim slot, on two streams, so that they run at the
    # same time: a call that finds the other's tag raises AB_FLAG_SCHED_COLLISION; a call
    # that raises nothing must have written exactly what it writes alone.
    lib = ab.lib()
    runs = []
    for seed, (N, H, max_cnt) in enumerate([(32768, 16, 64), (4000, 6, 8)]):
        q, k, v = _inputs(N, H, seed=40 + seed)
        B, _, N_pad, d = q.shape
        nqb = N_pad // 128
        idx, cnt, w = _plan(B, H, nqb, nqb, nqb, max_cnt, 0.1, seed=50 + seed)
        t = [x.cuda() for x in (q, k, v)] + [torch.from_numpy(a).cuda() for a in (idx, cnt, w)]
        alone = ab.attn_fwd(*t[:3], N, *t[3:], out_dtype=torch.float32)
        runs.append((N, t, alone))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    flags = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in runs]
    outs = [torch.full_like(r[2], float("nan")) for r in runs]
    for (N, t, _), s, f, o in zip(runs, streams, flags, outs):
        with torch.cuda.stream(s):
            assert lib.ab_selftest_force_counter_slot(77) == 0
            ab.attn_fwd(*t[:3], N, *t[3:], dev_flag=f, out=o, out_dtype=torch.float32)
    torch.cuda.synchronize()
    seen = []
    for (N, t, alone), f, o in zip(runs, flags, outs):
        bits = ab.check_flag(f)
        assert bits & ~ab.FLAG_SCHED_COLLISION == 0
        if not bits & ab.FLAG_SCHED_COLLISION:
            assert torch.equal(o, alone)
        seen.append(bool(bits))
    print("collision flagged per call:", seen)
    # a slot forced once is used once: the next call is clean again
    N, t, alone = runs[1]
    f = torch.zeros(1, dtype=torch.int32, device="cuda")
    again = ab.attn_fwd(*t[:3], N, *t[3:], dev_flag=f, out_dtype=torch.float32)
    assert ab.check_flag(f) == 0 and torch.equal(again, alone)
    assert lib.ab_selftest_force_counter_slot(4096) == 5  # AB_ERR_RANGE
