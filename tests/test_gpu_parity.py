"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same
seeded inputs, element by element, at sizes that span several tiles and a ragged tail.

Tolerances (from the method's acceptance criteria):
  * SIP and top-k plans: bit-exact (idx, cnt, w, p) when fed the same fp32 scores;
  * k-means assignments: equal except in blocks where the oracle met a near tie, i.e.
    a relative gap (d2 - d1) / d2 < 1e-5 between best and second-best distances;
  * mean keys: 1e-6 relative; block scores: |s - s_ref| <= 1e-4 |s_ref| + 1e-30 with
    s_ref computed by the oracle from the GPU's own centroids, weights and mean keys;
  * attention given the same plan: max |O - O_ref| <= 1e-2 and
    ||O - O_ref||_F / ||O_ref||_F <= 5e-3 against the fp64 oracle on the same bf16
    inputs; lse within 1e-3. These bounds apply as stated to the kernel's fp32 output
    (out_dtype=float32). A bf16 output adds its own rounding, up to half a bf16 ulp of
    |O_ref| (0.0078 at |O| in [2, 4)), so its max-abs bound is 1e-2 + ulp_bf16(O_ref)/2;
    the Frobenius bound is unchanged.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import synth

pytestmark = pytest.mark.gpu

ATOL_MAX = 1e-2
RTOL_FRO = 5e-3
LSE_ATOL = 1e-3
SCORE_RTOL = 1e-4
TIE_GAP = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


def _inputs(N, H=2, d=128, B=1, seed=0, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    q = torch.zeros(B, H, N_pad, d)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    q[:, :, :N] = torch.randn(B, H, N, d, generator=g) * scale
    k[:, :, :N] = torch.randn(B, H, N, d, generator=g) * scale
    v[:, :, :N] = torch.randn(B, H, N, d, generator=g)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def _cuda(*ts):
    return [t.cuda() for t in ts]


def _flag():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _rows_all(B, H, nb):
    return np.arange(B * H * nb, dtype=np.int64)


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def _compare_attn(orc, q, k, v, N, idx, cnt, w, out_gpu, lse_gpu, rows=None):
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    if rows is None:
        rows = _rows_all(B, H, nb)
    ref, ref_lse, _, _ = orc.attn_rows(q, k, v, N, idx.cpu().numpy(), cnt.cpu().numpy(),
                                       None if w is None else w.cpu().numpy(), rows=rows)
    og = out_gpu.float().cpu().numpy().reshape(B * H * nb, 128, d)[rows]
    lg = lse_gpu.cpu().numpy().reshape(B * H * nb, 128)[rows]
    diff = np.abs(og - ref)
    if out_gpu.dtype == torch.float32:
        assert diff.max() <= ATOL_MAX, diff.max()
    else:
        excess = diff - half_ulp_bf16(ref)
        assert excess.max() <= ATOL_MAX, (diff.max(), excess.max())
    denom = np.linalg.norm(ref)
    if denom > 0:
        assert np.linalg.norm(og - ref) / denom <= RTOL_FRO
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lg))
    assert np.all(lg[~fin] == ref_lse[~fin])
    assert np.abs(lg[fin] - ref_lse[fin]).max(initial=0) <= LSE_ATOL
    return diff.max(), np.linalg.norm(og - ref) / max(denom, 1e-30)


# ------------------------------------------------------------------ selection --------

def _random_scores(B, H, nqb, nkb, seed, kind="dirichlet"):
    rng = np.random.default_rng(seed)
    if kind == "dirichlet":
        s = rng.dirichlet(np.ones(nkb) * 0.3, size=(B, H, nqb))
    else:
        s = np.exp(rng.standard_normal((B, H, nqb, nkb)) * 3)
        s = s / s.sum(-1, keepdims=True)
    return s.astype(np.float32)


@pytest.mark.parametrize("nkb,budget", [(8, 3), (300, 30), (2048, 205), (929, 93), (64, 64),
                                        (64, 100), (37, 1)])
def test_sip_bit_exact(orc, nkb, budget):
    s = _random_scores(1, 3, 5, nkb, seed=nkb + budget)
    s[0, 0, 0, : nkb // 2] = 0.0  # rows with zero scores
    for seed in (0, 12345, 2**63 + 7):
        idx_r, cnt_r, w_r, p_r, bad = orc.sip(s, budget, seed)
        flag = _flag()
        idx, cnt, w, p = ab.select(torch.from_numpy(s).cuda(), budget, "sip", seed, want_p=True,
                                   dev_flag=flag)
        torch.cuda.synchronize()
        assert ab.check_flag(flag) == 0
        np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
        np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
        np.testing.assert_array_equal(p.cpu().numpy().view(np.uint64), p_r.view(np.uint64))


def _boundary_row(orc, s, K, seed, h, qb, j0):
    """Move score j0 of row (h, qb) until its SIP probability times 2^53 lands on its own
    Philox draw R53 (the oracle's p and Philox), so that keeping j0 is decided by the last
    bits of p_j0."""
    key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32)
    x = orc.philox4x32_10(np.array([j0, qb, h, 0], dtype=np.uint32), key)
    target = ((((int(x[0]) << 32) | int(x[1])) >> 11) / 2.0**53)
    for _ in range(40):
        p = orc.sip(s.reshape(1, 1, 1, -1), K, seed)[3][0, 0, 0, j0]
        if not 0.0 < p < 1.0 or p == target:
            break
        v = np.float32(s[j0] * (target / p))
        if v == s[j0]:
            break
        s[j0] = v
    return s


@pytest.mark.parametrize("nkb,budget", [(200, 20), (9000, 900)])
def test_sip_draws_at_the_boundary(orc, nkb, budget):
    """Rows whose draw for one entry falls within a few float steps of p 2^53, on both
    sides: the kernel's fast fp32 pre-decision must hand these to the exact test, so the
    plan still equals the oracle's bit for bit (rows of up to 8192 entries and longer)."""
    seed = 11
    rng = np.random.default_rng(nkb)
    H, nqb = 2, 7  # row r = (h, qb): step -3 .. +3 float steps away from the boundary
    s = (rng.random((1, H, nqb, nkb)) * 0.01).astype(np.float32)
    for h in range(H):
        j0 = int(rng.integers(nkb))
        base = _boundary_row(orc, s[0, h, 0].copy(), budget, seed, h, 0, j0)
        for qb in range(nqb):
            row = _boundary_row(orc, base.copy(), budget, seed, h, qb, j0)
            v = row[j0]
            step = qb - 3
            for _ in range(abs(step)):
                v = np.nextafter(v, np.float32(np.inf) if step > 0 else np.float32(0))
            row[j0] = v
            s[0, h, qb] = row
    idx_r, cnt_r, w_r, p_r, bad = orc.sip(s, budget, seed)
    assert not bad.any()
    for want_p in (False, True):
        flag = _flag()
        res = ab.select(torch.from_numpy(s).cuda(), budget, "sip", seed, want_p=want_p,
                        dev_flag=flag)
        idx, cnt, w = res[:3]
        torch.cuda.synchronize()
        assert ab.check_flag(flag) == 0
        np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
        np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
        if want_p:
            np.testing.assert_array_equal(res[3].cpu().numpy().view(np.uint64), p_r.view(np.uint64))


@pytest.mark.parametrize("nkb,budget", [(8, 3), (300, 30), (2048, 614), (929, 93), (5, 9)])
def test_topk_bit_exact(orc, nkb, budget):
    s = _random_scores(2, 2, 3, nkb, seed=7 * nkb, kind="lognormal")
    s[0, 0, 0, :] = 0.125  # all ties
    s[0, 1, 1, 3:nkb:3] = s[0, 1, 1, 1]  # partial ties
    idx_r, cnt_r, w_r = orc.topk(s, budget)
    idx, cnt, w = ab.select(torch.from_numpy(s).cuda(), budget, "topk")
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    np.testing.assert_array_equal(w.cpu().numpy(), w_r)


def test_select_flags_bad_scores(orc):
    s = _random_scores(1, 1, 4, 16, seed=3)
    s[0, 0, 1, 5] = np.nan
    s[0, 0, 2, 0] = -1.0
    for mode in ("sip", "topk"):
        flag = _flag()
        idx, cnt, w = ab.select(torch.from_numpy(s).cuda(), 4, mode, 0, dev_flag=flag)
        assert ab.check_flag(flag) & ab.FLAG_BAD_SCORE
        c = cnt.cpu().numpy()[0, 0]
        assert c[1] == 0 and c[2] == 0 and c[0] > 0 and c[3] > 0
        assert np.all(idx.cpu().numpy()[0, 0, 1] == -1)


def test_sip_rejects_rows_whose_exact_sum_overflows(orc):
    # U = 8192 * 2^51 = 2^64 in row 0 (rejected on both sides); row 1 sums just below
    s = np.full((1, 1, 2, 8192), 2.0, dtype=np.float32)
    s[0, 0, 1, 0] = 1.75
    flag = _flag()
    idx, cnt, w, p = ab.select(torch.from_numpy(s).cuda(), 100, "sip", 0, want_p=True, dev_flag=flag)
    assert ab.check_flag(flag) & ab.FLAG_BAD_SCORE
    idx_r, cnt_r, w_r, p_r, bad_r = orc.sip(s, 100, 0)
    assert bad_r[0, 0, 0] == 1
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_r)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
    np.testing.assert_array_equal(p.cpu().numpy()[0, 0, 1].view(np.uint64), p_r[0, 0, 1].view(np.uint64))


# -------------------------------------------------------------------- scoring --------

@pytest.mark.parametrize("N,d,H,C", [(1024, 64, 2, 8), (3 * 128 + 77, 128, 3, 8),
                                     (9 * 128 + 16, 128, 2, 8), (640, 128, 1, 1),
                                     (200, 64, 1, 3)])
def test_score_parity(orc, N, d, H, C):
    q, k, _ = _inputs(N, H=H, d=d, seed=N + d)
    T = 5
    s_gpu, kbar, cent, cw, assign = ab.score(*_cuda(q, k), N, C, T, intermediates=True)
    torch.cuda.synchronize()
    kbar_ref = orc.mean_key(k, N)
    np.testing.assert_allclose(kbar.cpu().numpy(), kbar_ref, rtol=1e-6, atol=1e-7)
    cent_r, wts_r, assign_r, gap, _ = orc.kmeans(q, N, C, T)
    a_gpu = assign.cpu().numpy()
    B, H_, N_pad, _ = q.shape
    nb = N_pad // 128
    mism = (a_gpu != assign_r).reshape(B, H_, nb, 128).any(-1)
    near_tie = gap < TIE_GAP
    assert not np.any(mism & ~near_tie), "assignment mismatch outside a near tie"
    ok = ~mism
    np.testing.assert_array_equal(cw.cpu().numpy()[ok], wts_r[ok].astype(np.float32))
    np.testing.assert_allclose(cent.cpu().numpy()[ok], cent_r[ok], rtol=1e-5, atol=1e-5)
    assert np.all(a_gpu[..., N:] == 255)
    # scores from the GPU's own intermediates
    s_ref = orc.score(cent.cpu().numpy().astype(np.float64), cw.cpu().numpy().astype(np.float64),
                      kbar.cpu().numpy().astype(np.float64))
    sg = s_gpu.cpu().numpy()
    assert np.all(np.abs(sg - s_ref) <= SCORE_RTOL * np.abs(s_ref) + 1e-30)
    np.testing.assert_allclose(sg.sum(-1), 1.0, rtol=1e-5)


@pytest.mark.parametrize("T", [1, 2, 30])
def test_kmeans_rounds_past_convergence(orc, T):
    """k-means stops once a round reproduces the previous round's assignments; with T = 30
    most blocks converge long before the last round, and the GPU's outputs must still be
    those of all T rounds (the oracle runs every round). T = 1 and 2 leave no room for an
    early stop."""
    N, d, H, C = 5 * 128 + 77, 128, 2, 8
    q, k, _ = _inputs(N, H=H, d=d, seed=T + 11)
    _, _, cent, cw, assign = ab.score(*_cuda(q, k), N, C, T, intermediates=True)
    torch.cuda.synchronize()
    cent_r, wts_r, assign_r, gap, inertia = orc.kmeans(q, N, C, T)
    if T == 30:  # the early stop is exercised: most blocks settle by round 15
        assert np.mean(inertia[..., -1] == inertia[..., 14]) > 0.5
    B, H_, N_pad, _ = q.shape
    nb = N_pad // 128
    mism = (assign.cpu().numpy() != assign_r).reshape(B, H_, nb, 128).any(-1)
    assert not np.any(mism & ~(gap < TIE_GAP)), "assignment mismatch outside a near tie"
    ok = ~mism
    np.testing.assert_array_equal(cw.cpu().numpy()[ok], wts_r[ok].astype(np.float32))
    np.testing.assert_allclose(cent.cpu().numpy()[ok], cent_r[ok], rtol=1e-5, atol=1e-5)


def test_score_tiny_workload_end_to_end(orc):
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(w)
    s_gpu = ab.score(*_cuda(q, k), w.N, w.n_clusters, w.iters).cpu().numpy()
    s_ref = orc.ibcs_scores(q, k, w.N, w.n_clusters, w.iters)
    _, _, _, gap, _ = orc.kmeans(q, w.N, w.n_clusters, w.iters)
    ok = (gap >= TIE_GAP)[..., None]
    assert np.all((np.abs(s_gpu - s_ref) <= SCORE_RTOL * s_ref + 1e-30) | ~ok)


# ------------------------------------------------------------------ attention --------

OUT_DTYPES = [torch.bfloat16, torch.float32]


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
@pytest.mark.parametrize("N,d,H,budget", [
    (1024, 64, 2, 3),            # tiny shape, d = 64
    (5 * 128 + 41, 128, 2, 3),   # ragged tail, d = 128
    (9 * 128, 128, 3, 9),        # all blocks (dense)
    (7 * 128 + 1, 128, 1, 1),    # a last block with one valid key
    (12 * 128 + 100, 64, 2, 5),
])
def test_attn_sip_parity(orc, N, d, H, budget, out_dtype):
    q, k, v = _inputs(N, H=H, d=d, seed=N * 3 + d, scale=1.5)
    qc, kc, vc = _cuda(q, k, v)
    s = ab.score(qc, kc, N)
    flag = _flag()
    idx, cnt, w = ab.select(s, budget, "sip", seed=11)
    out, lse = ab.attn_fwd(qc, kc, vc, N, idx, cnt, w, want_lse=True, dev_flag=flag,
                           out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ab.check_flag(flag) == 0
    _compare_attn(orc, q, k, v, N, idx, cnt, w, out, lse)
    assert torch.all(out[:, :, N:] == 0)


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
@pytest.mark.parametrize("N,d,budget", [(1024, 64, 3), (6 * 128 + 5, 128, 4)])
def test_attn_topk_parity(orc, N, d, budget, out_dtype):
    q, k, v = _inputs(N, H=2, d=d, seed=N + 17, scale=1.5)
    qc, kc, vc = _cuda(q, k, v)
    s = ab.score(qc, kc, N)
    idx, cnt, _ = ab.select(s, budget, "topk")
    out, lse = ab.attn_topk_fwd(qc, kc, vc, N, idx, cnt, want_lse=True, out_dtype=out_dtype)
    torch.cuda.synchronize()
    _compare_attn(orc, q, k, v, N, idx, cnt, None, out, lse)


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_attn_hand_plans(orc, out_dtype):
    """Hand-built plans: empty rows, repeated large weights (lazy rescale path), a
    late block with a much larger logit than the first one."""
    N, d, H = 6 * 128, 128, 2
    q, k, v = _inputs(N, H=H, d=d, seed=5)
    # block 5 of head 0 dominates: its logits exceed the running max of the earlier blocks
    # by more than the lazy-rescale threshold (20 in log2 units), forcing O rescales
    k[0, 0, 5 * 128:6 * 128] *= 12
    nb = 6
    idx = torch.full((1, H, nb, nb), -1, dtype=torch.int32)
    cnt = torch.zeros(1, H, nb, dtype=torch.int32)
    w = torch.zeros(1, H, nb, nb)
    for h in range(H):
        for qb in range(nb):
            sel = [(qb + t) % nb for t in range(qb % 4)]
            sel = sorted(set(sel + ([5] if qb % 2 else [])))
            cnt[0, h, qb] = len(sel)
            idx[0, h, qb, : len(sel)] = torch.tensor(sel, dtype=torch.int32)
            w[0, h, qb, : len(sel)] = torch.tensor([1.0 + 7.0 * ((j * 3 + qb) % 4) for j in sel])
    qc, kc, vc = _cuda(q, k, v)
    out, lse = ab.attn_fwd(qc, kc, vc, N, idx.cuda(), cnt.cuda(), w.cuda(), want_lse=True,
                           out_dtype=out_dtype)
    torch.cuda.synchronize()
    _compare_attn(orc, q, k, v, N, idx, cnt, w, out, lse)
    assert torch.all(out[0, :, 0:128] == 0)  # qb = 0 has an empty selection


def test_attn_flags_bad_plan(orc):
    N, d = 4 * 128, 64
    q, k, v = _inputs(N, H=1, d=d, seed=9)
    idx = torch.tensor([[[[0, 1, -1, -1], [7, 0, -1, -1], [0, -1, -1, -1], [0, 1, 2, 3]]]],
                       dtype=torch.int32)
    cnt = torch.tensor([[[2, 2, 1, 4]]], dtype=torch.int32)
    w = torch.tensor([[[[1, 1, 0, 0], [1, 1, 0, 0], [-2, 0, 0, 0], [1, 1, 1, 1]]]],
                     dtype=torch.float32)
    flag = _flag()
    out = ab.attn_fwd(*_cuda(q, k, v), N, idx.cuda(), cnt.cuda(), w.cuda(), dev_flag=flag)
    f = ab.check_flag(flag)
    assert f & ab.FLAG_BAD_INDEX and f & ab.FLAG_BAD_WEIGHT
    assert not f & ab.FLAG_TIMEOUT
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
@pytest.mark.parametrize("name", ["tiny"])
def test_workload_full_path(orc, name, out_dtype):
    """Score -> select -> attention on a named workload, every row against the oracle
    (plan fed from the GPU so the attention check is independent of k-means ties)."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w)
    qc, kc, vc = _cuda(q, k, v)
    K = w.budget_blocks(w.budgets[0])
    s = ab.score(qc, kc, w.N, w.n_clusters, w.iters)
    idx, cnt, wt = ab.select(s, K, "sip", w.sip_seed)
    out, lse = ab.attn_fwd(qc, kc, vc, w.N, idx, cnt, wt, want_lse=True, out_dtype=out_dtype)
    torch.cuda.synchronize()
    idx_r, cnt_r, w_r, _, _ = orc.sip(s.cpu().numpy(), K, w.sip_seed)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_r)
    np.testing.assert_array_equal(wt.cpu().numpy(), w_r)
    _compare_attn(orc, q, k, v, w.N, idx, cnt, wt, out, lse)
    ti, tc, _ = ab.select(s, K, "topk")
    out_t, lse_t = ab.attn_topk_fwd(qc, kc, vc, w.N, ti, tc, want_lse=True, out_dtype=out_dtype)
    torch.cuda.synchronize()
    _compare_attn(orc, q, k, v, w.N, ti, tc, None, out_t, lse_t)
