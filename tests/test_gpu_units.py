"""GPU parity of the 4-token key-unit path (AB-Attention page, section «Три приёма
AB-Attention», third technique) against the oracle at unit granularity.

Same bounds as the block path (tests/test_gpu_parity.py): unit mean keys 1e-6 relative;
unit scores within 1e-4 relative of the oracle fed the GPU's own centroids, weights and
mean keys, exactly 0 for units past the sequence end; SIP and top-k plans over units
bit-exact; attention given the same plan max-abs <= 1e-2 and relative Frobenius <= 5e-3
(fp32 output; a bf16 output adds half a bf16 ulp), lse within 1e-3. Sizes cover several
query blocks, a ragged sequence end inside a unit (N mod 4 != 0), partial 32-unit tiles,
empty rows, unit indices past the sequence end, and every unit kept (dense attention).
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import synth

pytestmark = pytest.mark.gpu

U = 4
ATOL_MAX = 1e-2
RTOL_FRO = 5e-3
LSE_ATOL = 1e-3
SCORE_RTOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


def _inputs(N, H=2, d=128, B=1, seed=0, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    x = [torch.zeros(B, H, N_pad, d) for _ in range(3)]
    for t, s in zip(x, (scale, scale, 1.0)):
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g) * s
    return [t.to(torch.bfloat16) for t in x]


def _half_ulp_bf16(x):
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def _compare(orc, q, k, v, N, idx, cnt, w, out, lse, rows=None):
    B, H, N_pad, d = q.shape
    nqb = N_pad // 128
    if rows is None:
        rows = np.arange(B * H * nqb, dtype=np.int64)
    ref, ref_lse, _, _ = orc.attn_rows(q, k, v, N, idx.cpu().numpy(), cnt.cpu().numpy(),
                                       None if w is None else w.cpu().numpy(), rows=rows, unit=U)
    og = out.float().cpu().numpy().reshape(B * H * nqb, 128, d)[rows]
    lg = lse.cpu().numpy().reshape(B * H * nqb, 128)[rows]
    diff = np.abs(og - ref)
    if out.dtype == torch.float32:
        assert diff.max() <= ATOL_MAX, diff.max()
    else:
        assert (diff - _half_ulp_bf16(ref)).max() <= ATOL_MAX
    denom = np.linalg.norm(ref)
    if denom > 0:
        assert np.linalg.norm(og - ref) / denom <= RTOL_FRO
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lg))
    assert np.all(lg[~fin] == ref_lse[~fin])
    assert np.abs(lg[fin] - ref_lse[fin]).max(initial=0) <= LSE_ATOL


@pytest.mark.parametrize("N,d", [(681, 128), (1021, 64), (1024, 128)])
def test_unit_scores(orc, N, d):
    q, k, v = _inputs(N, d=d, seed=N)
    qc, kc = q.cuda(), k.cuda()
    s, kbar, cent, cw, _ = ab.score(qc, kc, N, 8, 5, intermediates=True, unit=U)
    torch.cuda.synchronize()
    B, H, N_pad, _ = q.shape
    n_valid = (N + U - 1) // U
    kb_ref = orc.mean_key(k, N, unit=U)
    np.testing.assert_allclose(kbar.cpu().numpy(), kb_ref, rtol=1e-5, atol=1e-6)
    sg = s.cpu().numpy()
    assert sg.shape == (B, H, N_pad // 128, N_pad // U)
    assert np.all(sg[..., n_valid:] == 0)
    ref = orc.score(cent.cpu().numpy().astype(np.float64), cw.cpu().numpy().astype(np.float64),
                    kbar.cpu().numpy().astype(np.float64), n_valid=n_valid)
    assert np.all(np.abs(sg - ref) <= SCORE_RTOL * np.abs(ref) + 1e-30)
    np.testing.assert_allclose(sg.sum(-1), 1.0, rtol=2e-5)


@pytest.mark.parametrize("N,d,budget", [(681, 128, 37), (1021, 64, 64), (1024, 128, 1),
                                        (897, 128, 96)])
@pytest.mark.parametrize("mode", ["sip", "topk"])
def test_unit_plan_and_attention(orc, N, d, budget, mode):
    q, k, v = _inputs(N, d=d, seed=N + budget)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    s = ab.score(qc, kc, N, unit=U)
    if mode == "sip":
        idx, cnt, w = ab.select(s, budget, "sip", 7)
        idx_r, cnt_r, w_r, _, _ = orc.sip(s.cpu().numpy(), budget, 7, with_p=False)
    else:
        idx, cnt, w = ab.select(s, budget, "topk")
        idx_r, cnt_r, w_r = orc.topk(s.cpu().numpy(), budget)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
    for out_dtype in (torch.float32, torch.bfloat16):
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        if mode == "sip":
            out, lse = ab.attn_fwd(qc, kc, vc, N, idx, cnt, w, want_lse=True, dev_flag=flag,
                                   out_dtype=out_dtype, unit=U)
        else:
            out, lse = ab.attn_topk_fwd(qc, kc, vc, N, idx, cnt, want_lse=True, dev_flag=flag,
                                        out_dtype=out_dtype, unit=U)
        torch.cuda.synchronize()
        assert ab.check_flag(flag) == 0
        _compare(orc, q, k, v, N, idx, cnt, w if mode == "sip" else None, out, lse)


def test_unit_attention_on_hand_made_plans(orc):
    """Arbitrary unit lists: empty rows, a single unit, the unit that holds the ragged
    sequence end, units entirely past it (alone: no valid key, so O = 0 and lse = -inf),
    full and partial 32-unit tiles, and every unit kept, with HT weights."""
    N, d = 681, 128
    q, k, v = _inputs(N, d=d, seed=3)
    B, H, N_pad, _ = q.shape
    nqb, nku = N_pad // 128, N_pad // U
    last = (N - 1) // U   # holds tokens 680 only
    rng = np.random.default_rng(11)
    idx = np.full((B, H, nqb, nku), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    w = np.zeros((B, H, nqb, nku), dtype=np.float32)
    plans = [[], [5], [last], [last, nku - 1], [nku - 2, nku - 1], list(range(32)),
             list(range(nku)),
             sorted(rng.choice(last + 1, 45, replace=False).tolist())]
    for h in range(H):
        for qb in range(nqb):
            sel = plans[(h * nqb + qb) % len(plans)]
            idx[0, h, qb, :len(sel)] = sel
            cnt[0, h, qb] = len(sel)
            w[0, h, qb, :len(sel)] = rng.uniform(1.0, 4.0, len(sel)).astype(np.float32)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    ic, cc, wc = (torch.from_numpy(a).cuda() for a in (idx, cnt, w))
    for weighted in (True, False):
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        if weighted:
            out, lse = ab.attn_fwd(qc, kc, vc, N, ic, cc, wc, want_lse=True, dev_flag=flag,
                                   out_dtype=torch.float32, unit=U)
        else:
            out, lse = ab.attn_topk_fwd(qc, kc, vc, N, ic, cc, want_lse=True, dev_flag=flag,
                                        out_dtype=torch.float32, unit=U)
        torch.cuda.synchronize()
        assert ab.check_flag(flag) == 0
        _compare(orc, q, k, v, N, ic, cc, wc if weighted else None, out, lse)


def test_unit_attention_flags_bad_indices(orc):
    N, d = 512, 64
    q, k, v = _inputs(N, d=d, seed=4)
    B, H, N_pad, _ = q.shape
    nqb, nku = N_pad // 128, N_pad // U
    idx = torch.zeros(B, H, nqb, nku, dtype=torch.int32)
    idx[..., :3] = torch.tensor([1, nku + 5, 2], dtype=torch.int32)
    cnt = torch.full((B, H, nqb), 3, dtype=torch.int32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    ab.attn_topk_fwd(q.cuda(), k.cuda(), v.cuda(), N, idx.cuda(), cnt.cuda(), dev_flag=flag, unit=U)
    assert ab.check_flag(flag) & 2  # AB_FLAG_BAD_INDEX


def test_unit_path_at_wan13b_size(orc):
    """The Wan2.1-1.3B-shaped workload with 4-token units at the same tile budget as the
    bench (26 tiles of 32 units): plans bit-exact on sampled rows, attention on sampled
    query blocks."""
    w = synth.WORKLOADS["wan13b"]
    q, k, v = synth.make_qkv(w, heads=[0, 1])
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    K = w.budget_blocks(w.budgets[0]) * 32
    s = ab.score(qc, kc, w.N, w.n_clusters, w.iters, unit=U)
    idx, cnt, wt = ab.select(s, K, "sip", w.sip_seed)
    torch.cuda.synchronize()
    s_np = s.cpu().numpy()
    rows = np.random.default_rng(0).choice(s_np.shape[2], 6, replace=False)
    sub = np.zeros_like(s_np)
    sub[:, :, rows] = s_np[:, :, rows]
    idx_r, cnt_r, w_r, _, _ = orc.sip(sub, K, w.sip_seed, with_p=False)
    np.testing.assert_array_equal(cnt.cpu().numpy()[:, :, rows], cnt_r[:, :, rows])
    np.testing.assert_array_equal(idx.cpu().numpy()[:, :, rows], idx_r[:, :, rows])
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = ab.attn_fwd(qc, kc, vc, w.N, idx, cnt, wt, want_lse=True, dev_flag=flag,
                           out_dtype=torch.float32, unit=U)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    nqb = w.N_pad // 128
    sample = np.array([0 * nqb + 3, 0 * nqb + nqb - 1, 1 * nqb + 100, 1 * nqb + 7], dtype=np.int64)
    _compare(orc, q, k, v, w.N, idx, cnt, wt, out, lse, rows=sample)


def test_unit_path_at_hunyuan720_size(orc):
    """Two heads of the HunyuanVideo-720p-shaped workload (N = 118800 tokens, 29728 4-token
    units per head, 29700 of them holding a valid token) at the bench's tile budget (93
    tiles = 2976 units): unit scores on sampled rows against the oracle fed the GPU's own
    centroids, weights and mean keys, the SIP and top-k plans bit-exact on sampled rows,
    attention on sampled query blocks."""
    w = synth.WORKLOADS["hunyuan720"]
    q, k, v = synth.make_qkv(w, heads=[0, 1])
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    nqb, nku = w.N_pad // 128, w.N_pad // U
    nvu = -(-w.N // U)
    assert nku == 29728 and nvu == 29700
    K = w.budget_blocks(w.budgets[0]) * 32
    s, kbar, cent, cw, _ = ab.score(qc, kc, w.N, w.n_clusters, w.iters, unit=U, intermediates=True)
    torch.cuda.synchronize()
    s_np = s.cpu().numpy()
    assert np.all(s_np[..., nvu:] == 0)
    np.testing.assert_allclose(s_np.sum(-1), 1.0, rtol=2e-5)
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(nqb, 5, replace=False))
    ref = orc.score(cent.cpu().numpy().astype(np.float64)[:, :, rows],
                    cw.cpu().numpy().astype(np.float64)[:, :, rows],
                    kbar.cpu().numpy().astype(np.float64), n_valid=nvu)
    got = s_np[:, :, rows]
    assert np.all(np.abs(got - ref) <= SCORE_RTOL * np.abs(ref) + 1e-30)
    sub = np.zeros_like(s_np)
    sub[:, :, rows] = s_np[:, :, rows]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for mode in ("topk", "sip"):
        idx, cnt, wt = ab.select(s, K, mode, w.sip_seed, dev_flag=flag)
        torch.cuda.synchronize()
        if mode == "sip":
            idx_r, cnt_r, w_r, _, _ = orc.sip(sub, K, w.sip_seed, with_p=False)
            np.testing.assert_array_equal(wt.cpu().numpy()[:, :, rows].view(np.uint32),
                                          w_r[:, :, rows].view(np.uint32))
        else:
            idx_r, cnt_r, _ = orc.topk(sub, K)
        np.testing.assert_array_equal(cnt.cpu().numpy()[:, :, rows], cnt_r[:, :, rows])
        np.testing.assert_array_equal(idx.cpu().numpy()[:, :, rows], idx_r[:, :, rows])
    assert ab.check_flag(flag) == 0
    out, lse = ab.attn_fwd(qc, kc, vc, w.N, idx, cnt, wt, want_lse=True, dev_flag=flag,
                           out_dtype=torch.float32, unit=U)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    sample = np.array([rows[0], nqb - 1, nqb + rows[2], nqb + rows[4]], dtype=np.int64)
    _compare(orc, q, k, v, w.N, idx, cnt, wt, out, lse, rows=sample)


@pytest.mark.parametrize("nku", [29728, 65536])
def test_selection_rows_of_many_units(orc, nku):
    """Selection rows of 4-token units up to the 65536-unit limit (the 262144-token shape):
    top-k (scores staged in shared memory up to 40960 entries, read from global memory
    beyond) and SIP (a 64 KB saturation map) bit-exact against the oracle, with ties."""
    rng = np.random.default_rng(nku)
    s = rng.random((1, 1, 3, nku), dtype=np.float32) ** 8
    s[0, 0, 1, 100:2000] = s[0, 0, 1, 99]  # a long run of equal scores
    s /= s.sum(-1, keepdims=True)
    K = 2976 if nku < 65536 else 6560
    sc = torch.from_numpy(s).cuda()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, cnt, _ = ab.select(sc, K, "topk", dev_flag=flag)
    idx_r, cnt_r, _ = orc.topk(s, K)
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    idx, cnt, wt, p = ab.select(sc, K, "sip", 5, want_p=True, dev_flag=flag)
    idx_r, cnt_r, w_r, p_r, _ = orc.sip(s, K, 5)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    np.testing.assert_array_equal(wt.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
    np.testing.assert_array_equal(p.cpu().numpy().view(np.uint64), p_r.view(np.uint64))
