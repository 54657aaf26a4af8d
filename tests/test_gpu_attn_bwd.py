"""GPU parity of the attention backward (gradients with respect to Q, K and V) through
the C ABI, against the CPU oracle's fp64 gradient on the same bf16 inputs and plan.

Tolerance, from the kernel's arithmetic: S, dP and the three gradients accumulate in
fp32 on the tensor cores; the operands P (for dV) and dS (for dQ and dK) are rounded to
bf16 (unit roundoff u = 2^-8), and D_i = dO_i . O_i uses the forward's O (bf16 or fp32).
Each gradient element is a sum of many such products with independent rounding errors,
so its relative Frobenius error is about u / sqrt(3) = 2.3e-3; the bound is
||g - g_ref||_F <= 1e-2 ||g_ref||_F and, element-wise, |g - g_ref| <= 3e-2 max|g_ref|
per tensor. Rows that take no part (padding, an empty selection, a key block that no
query block kept) must be exactly 0, and two runs must agree bit for bit (every sum
runs in a fixed order).

At full workload sizes the oracle cannot run whole; there the dQ rows of sampled query
blocks are checked against the oracle run on a sub-problem that holds only the block's
queries and its kept key blocks (a query row's gradient depends on nothing else), and
the key and value gradients through two identities that hold at any size: a softmax
row is invariant to a shift of its logits, so the key gradients of a head sum to 0, and
its probabilities sum to 1, so the value gradients of a head sum to the sum of the
upstream gradient rows that have a non-empty selection.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import synth

pytestmark = pytest.mark.gpu

RTOL_FRO = 1e-2
RTOL_MAX = 3e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


def _inputs(N, H, d, seed, B=1, scale=1.5):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    out = []
    for s in (scale, scale, 1.0, 1.0):
        t = torch.zeros(B, H, N_pad, d)
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g) * s
        out.append(t.to(torch.bfloat16))
    return out  # q, k, v, dO


def _random_plan(B, H, nb, budget, seed, weighted=True, empty_row=None):
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
                idx[b, h, qb, :k] = np.sort(rng.choice(nb, size=k, replace=False))
                cnt[b, h, qb] = k
                w[b, h, qb, :k] = rng.uniform(1.0, 6.0, size=k) if weighted else 1.0
    return idx, cnt, (w if weighted else None)


def _gpu_grads(q, k, v, do, N, idx, cnt, w, out_dtype=torch.bfloat16, repeat=False):
    dev = "cuda"
    qg, kg, vg, gg = (t.to(dev) for t in (q, k, v, do))
    ig = torch.as_tensor(idx).to(dev)
    cg = torch.as_tensor(cnt).to(dev)
    wg = None if w is None else torch.as_tensor(w).to(dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    if wg is not None:
        out, lse = ab.attn_fwd(qg, kg, vg, N, ig, cg, wg, want_lse=True, dev_flag=flag, out_dtype=out_dtype)
    else:
        out, lse = ab.attn_topk_fwd(qg, kg, vg, N, ig, cg, want_lse=True, dev_flag=flag, out_dtype=out_dtype)
    grads = ab.attn_bwd(qg, kg, vg, N, ig, cg, wg, out, lse, gg, dev_flag=flag)
    if repeat:
        again = ab.attn_bwd(qg, kg, vg, N, ig, cg, wg, out, lse, gg, dev_flag=flag)
        for a, b_ in zip(grads, again):
            assert torch.equal(a, b_), "two runs of the backward differ"
    assert ab.check_flag(flag) == 0
    return [t.cpu().double().numpy() for t in grads]


def _close(got, ref, name):
    err = np.abs(got - ref)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = err.max() / max(np.abs(ref).max(), 1e-300)
    print(f"{name}: rel_fro={fro:.3e} max_err/max_ref={mx:.3e}")
    assert fro <= RTOL_FRO, (name, fro)
    assert mx <= RTOL_MAX, (name, mx)


def _check_zero_rows(dq, dk, dv, N, idx, cnt):
    B, H, N_pad, _ = dq.shape
    nb = N_pad // 128
    assert np.all(dq[:, :, N:] == 0) and np.all(dk[:, :, N:] == 0) and np.all(dv[:, :, N:] == 0)
    for b in range(B):
        for h in range(H):
            kept = set()
            for qb in range(nb):
                if cnt[b, h, qb] == 0:
                    assert np.all(dq[b, h, qb * 128:(qb + 1) * 128] == 0)
                kept.update(int(j) for j in idx[b, h, qb, :cnt[b, h, qb]])
            for kb in set(range(nb)) - kept:
                assert np.all(dk[b, h, kb * 128:(kb + 1) * 128] == 0)
                assert np.all(dv[b, h, kb * 128:(kb + 1) * 128] == 0)


CASES = [
    # N, H, d, budget, weighted, out dtype, empty row
    (3 * 128 + 50, 2, 64, 2, True, torch.bfloat16, None),
    (8 * 128 + 37, 2, 128, 3, True, torch.float32, (0, 1, 3)),
    (6 * 128, 1, 128, 6, False, torch.bfloat16, None),        # every block, top-k weights
    (5 * 128 + 1, 2, 128, 2, False, torch.float32, (0, 0, 4)),
    (9 * 128 + 100, 1, 64, 4, True, torch.float32, None),
]


@pytest.mark.parametrize("case", CASES)
def test_bwd_matches_oracle(orc, case):
    N, H, d, budget, weighted, odt, empty = case
    q, k, v, do = _inputs(N, H, d, seed=N + 3 * d)
    nb = q.shape[2] // 128
    idx, cnt, w = _random_plan(1, H, nb, budget, seed=N, weighted=weighted, empty_row=empty)
    dq, dk, dv = _gpu_grads(q, k, v, do, N, idx, cnt, w, out_dtype=odt, repeat=True)
    rq, rk, rv = orc.attn_bwd(q, k, v, do, N, idx, cnt, w)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(got, ref, name)
    _check_zero_rows(dq, dk, dv, N, idx, cnt)


@pytest.mark.parametrize("mode", ["sip", "topk"])
def test_bwd_on_the_method_plan(orc, mode):
    """The plan from ab_score + ab_select on positionally structured inputs (the tiny
    workload, 8 x 8 blocks, d = 64)."""
    wl = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_qkv(wl)
    g = torch.Generator().manual_seed(99)
    do = torch.zeros_like(q, dtype=torch.float32)
    do[:, :, :wl.N] = torch.randn(wl.B, wl.H, wl.N, wl.d, generator=g)
    do = do.to(torch.bfloat16)
    s = ab.score(q.cuda(), k.cuda(), wl.N)
    res = ab.select(s, budget=3, mode=mode, seed=5)
    idx, cnt, w = (t.cpu().numpy() for t in res[:3])
    dq, dk, dv = _gpu_grads(q, k, v, do, wl.N, idx, cnt, w if mode == "sip" else None)
    rq, rk, rv = orc.attn_bwd(q, k, v, do, wl.N, idx, cnt, w if mode == "sip" else None)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(got, ref, name)
    _check_zero_rows(dq, dk, dv, wl.N, idx, cnt)


def test_bwd_flags_a_duplicate_block():
    N, H, d = 4 * 128, 1, 64
    q, k, v, do = (t.cuda() for t in _inputs(N, H, d, seed=1))
    idx = torch.full((1, 1, 4, 4), -1, dtype=torch.int32)
    cnt = torch.full((1, 1, 4), 2, dtype=torch.int32)
    idx[..., :2] = torch.tensor([0, 2], dtype=torch.int32)
    w = torch.ones(1, 1, 4, 4)
    idx[0, 0, 1, :2] = torch.tensor([3, 3], dtype=torch.int32)  # block 3 twice in one row
    idx, cnt, w = idx.cuda(), cnt.cuda(), w.cuda()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = ab.attn_fwd(q, k, v, N, idx, cnt, w, want_lse=True)
    ab.attn_bwd(q, k, v, N, idx, cnt, w, out, lse, do, dev_flag=flag)
    assert ab.check_flag(flag) & 2  # AB_FLAG_BAD_INDEX


def _dq_sub_problem(orc, q, k, v, do, N, idx, cnt, w, b, h, qb):
    """The oracle's dQ rows of query block qb from a problem holding only that block's
    queries (block 0) and its kept key blocks (blocks 1..c, in plan order)."""
    N_pad, d = q.shape[2], q.shape[3]
    c = int(cnt[b, h, qb])
    sel = [int(j) for j in idx[b, h, qb, :c]]
    nb2 = c + 1
    Q2 = torch.zeros(1, 1, nb2 * 128, d, dtype=torch.bfloat16)
    K2, V2, G2 = torch.zeros_like(Q2), torch.zeros_like(Q2), torch.zeros_like(Q2)
    Q2[0, 0, :128] = q[b, h, qb * 128:(qb + 1) * 128]
    G2[0, 0, :128] = do[b, h, qb * 128:(qb + 1) * 128]
    for m, j in enumerate(sel):
        K2[0, 0, (m + 1) * 128:(m + 2) * 128] = k[b, h, j * 128:(j + 1) * 128]
        V2[0, 0, (m + 1) * 128:(m + 2) * 128] = v[b, h, j * 128:(j + 1) * 128]
    # only the sequence's last block is ragged; plan rows are ascending, so it comes last
    N2 = nb2 * 128 - ((N_pad - N) if sel and sel[-1] == N_pad // 128 - 1 else 0)
    idx2 = np.full((1, 1, nb2, nb2), -1, dtype=np.int32)
    cnt2 = np.zeros((1, 1, nb2), dtype=np.int32)
    idx2[0, 0, 0, :c] = np.arange(1, c + 1)
    cnt2[0, 0, 0] = c
    w2 = None
    if w is not None:
        w2 = np.zeros((1, 1, nb2, nb2), dtype=np.float32)
        w2[0, 0, 0, :c] = w[b, h, qb, :c]
    dq2, _, _ = orc.attn_bwd(Q2, K2, V2, G2, N2, idx2, cnt2, w2)
    return dq2[0, 0, :128]


@pytest.mark.parametrize("name", ["wan13b", "hunyuan720"])
def test_bwd_at_workload_size(orc, name):
    """The whole path (score, SIP, forward, backward) at a full workload size."""
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl)
    g = torch.Generator().manual_seed(7)
    do = torch.zeros(q.shape)
    do[:, :, :wl.N] = torch.randn(wl.B, wl.H, wl.N, wl.d, generator=g)
    do = do.to(torch.bfloat16)
    qg, kg, vg, gg = (t.cuda() for t in (q, k, v, do))
    K = wl.budget_blocks(wl.budgets[0])
    s = ab.score(qg, kg, wl.N)
    idx, cnt, w = ab.select(s, budget=K, mode="sip", seed=wl.sip_seed)[:3]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = ab.attn_fwd(qg, kg, vg, wl.N, idx, cnt, w, want_lse=True, dev_flag=flag)
    dq, dk, dv = ab.attn_bwd(qg, kg, vg, wl.N, idx, cnt, w, out, lse, gg, dev_flag=flag)
    assert ab.check_flag(flag) == 0
    # identities over each head
    sdk = dk.double().sum(2)
    print(f"{name}: |sum_t dK_t| / ||dK|| = {(sdk.norm() / dk.double().norm()).item():.3e}")
    assert sdk.norm() <= 1e-2 * dk.double().norm()
    rows_on = (cnt > 0).repeat_interleave(128, dim=2)[..., :wl.N_pad].clone()
    rows_on[:, :, wl.N:] = False
    sdo = (gg.double() * rows_on[..., None]).sum(2)
    sdv = dv.double().sum(2)
    rel = ((sdv - sdo).norm() / sdo.norm()).item()
    print(f"{name}: sum_t dV_t against sum_i dO_i: rel {rel:.3e}")
    assert rel <= 1e-2
    # dQ of sampled query blocks (first, middle, the ragged last) against the oracle
    idx_c, cnt_c = idx.cpu().numpy(), cnt.cpu().numpy()
    w_c = w.cpu().numpy()
    dq_c = dq[0].cpu().double().numpy()
    nb = wl.n_blocks
    for h, qb in ((0, 0), (wl.H // 2, nb // 2), (wl.H - 1, nb - 1)):
        ref = _dq_sub_problem(orc, q, k, v, do, wl.N, idx_c, cnt_c, w_c, 0, h, qb)
        _close(dq_c[h, qb * 128:(qb + 1) * 128], ref, f"{name} dq[h={h}, qb={qb}]")
