"""The selection-quality harness (quality.py): its dense reference against the oracle,
its metrics on hand-made cases (CPU), and one run of the whole harness on the GPU.

Mass recall and attention error are the quantities the AB-Attention page uses for its
claims (section «Три приёма AB-Attention»); the harness computes them against an exact
fp32 reference, so the reference is pinned to the fp64 oracle here first."""

import numpy as np
import pytest
import torch

import quality
from block_sparse_attention_ab_b200 import synth


def _small(seed=0, B=1, H=2, N=300, d=64):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    q = torch.zeros(B, H, N_pad, d, dtype=torch.bfloat16)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    q[:, :, :N] = (torch.randn(B, H, N, d, generator=g) * 1.5).to(torch.bfloat16)
    k[:, :, :N] = (torch.randn(B, H, N, d, generator=g) * 1.5).to(torch.bfloat16)
    v[:, :, :N] = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return q, k, v, N


def test_dense_reference_matches_oracle(orc):
    q, k, v, N = _small()
    o, mass = quality.dense_reference(q, k, v, N, rows_per_chunk=128)
    ref, _ = orc.dense_attn(q, k, v, N)
    np.testing.assert_allclose(o[:, :, :N].numpy(), ref[:, :, :N], atol=2e-5, rtol=1e-4)
    # every valid row's block masses sum to 1, padding keys get none
    np.testing.assert_allclose(mass[:, :, :N].sum(-1).numpy(), 1.0, atol=1e-5)
    assert torch.all(mass[:, :, N:] == 0)


def test_mass_recall_all_blocks_is_one_and_none_is_zero():
    q, k, v, N = _small(1)
    _, mass = quality.dense_reference(q, k, v, N)
    B, H, N_pad, nkb = mass.shape
    nqb = N_pad // 128
    idx = torch.arange(nkb, dtype=torch.int32).expand(B, H, nqb, nkb).contiguous()
    cnt = torch.full((B, H, nqb), nkb, dtype=torch.int32)
    assert quality.mass_recall(mass, idx, cnt, N) == pytest.approx(1.0, abs=1e-5)
    assert quality.mass_recall(mass, idx, torch.zeros_like(cnt), N) == 0.0


def test_mass_recall_counts_block_zero_once():
    # padding entries of idx point at block 0 and must not add or erase its mass
    mass = torch.zeros(1, 1, 128, 3)
    mass[..., 0] = 0.5
    mass[..., 2] = 0.5
    idx = torch.tensor([[[[2, 0, 0]]]], dtype=torch.int32)
    assert quality.mass_recall(mass, idx, torch.tensor([[[1]]], dtype=torch.int32), 128) == pytest.approx(0.5)
    idx = torch.tensor([[[[0, 0, 0]]]], dtype=torch.int32)
    assert quality.mass_recall(mass, idx, torch.tensor([[[1]]], dtype=torch.int32), 128) == pytest.approx(0.5)


def test_ideal_topk_has_the_largest_recall_among_topk_selections():
    q, k, v, N = _small(2, N=640)
    _, mass = quality.dense_reference(q, k, v, N)
    s = quality.ideal_scores(mass)
    B, H, nqb, nkb = s.shape
    K = 2
    best = torch.argsort(-s, dim=-1, stable=True)[..., :K].to(torch.int32).contiguous()
    cnt = torch.full((B, H, nqb), K, dtype=torch.int32)
    r_best = quality.mass_recall(mass, best, cnt, N)
    g = torch.Generator().manual_seed(3)
    for _ in range(20):
        rnd = torch.stack([torch.randperm(nkb, generator=g)[:K] for _ in range(B * H * nqb)])
        rnd = rnd.view(B, H, nqb, K).to(torch.int32).contiguous()
        assert quality.mass_recall(mass, rnd, cnt, N) <= r_best + 1e-6


def test_rel_error():
    a = torch.randn(1, 1, 256, 8)
    assert quality.rel_error(a, a, 200) == 0.0
    assert quality.rel_error(2 * a, a, 256) == pytest.approx(1.0, rel=1e-6)


@pytest.mark.gpu
def test_harness_on_tiny_workload():
    from block_sparse_attention_ab_b200 import build
    build.build()
    w = synth.WORKLOADS["tiny"]
    rows = quality.evaluate(w, 0, [0.25, 0.5, 1.0], seeds=4)
    methods = ("ibcs_sip", "ibcs_topk", "meanpool_topk", "ideal_topk")
    for r in rows:
        for m in methods:
            assert 0.0 <= r[m]["mass_recall"] <= 1.0 + 1e-5
            assert np.isfinite(r[m]["attn_error"])
        # no top-k selection keeps more true mass than the ideal one
        for m in ("ibcs_topk", "meanpool_topk"):
            assert r[m]["mass_recall"] <= r["ideal_topk"]["mass_recall"] + 1e-5
    # nested top-k sets: recall does not decrease with the budget
    for m in ("ibcs_topk", "meanpool_topk", "ideal_topk"):
        rec = [r[m]["mass_recall"] for r in rows]
        assert all(b >= a - 1e-6 for a, b in zip(rec, rec[1:]))
    # every block kept: all methods give the dense result up to bf16 rounding
    full = rows[-1]
    for m in methods:
        assert full[m]["mass_recall"] == pytest.approx(1.0, abs=1e-5)
        assert full[m]["attn_error"] < 1e-2
