"""Selection quality of AB-Attention on synthetic inputs.

The AB-Attention page (section «Три приёма AB-Attention») states its gains as relative
quality claims at a fixed block budget: IBCS scoring keeps more of the true attention
mass than scoring with one mean-pooled query per block, and SIP's importance-weighted
sampling gives a lower attention error than deterministic top-k. This harness measures
the same quantities on the seeded synthetic workloads, with no model or dataset:

  mass recall  = for each query row, the share of its exact softmax mass that lies in
                 the key blocks selected for its query block, averaged over valid rows;
  attn error   = ||O_sparse - O_dense||_F / ||O_dense||_F over valid rows, O_dense the
                 exact attention in fp32.

Methods, each at the same budget K (blocks per query block):
  ibcs_sip       IBCS scores (C = 8 clusters) -> SIP sampling -> HT-weighted attention
                 (averaged over --seeds draws);
  ibcs_topk      IBCS scores -> top-k -> plain attention over the kept blocks;
  meanpool_topk  scores from one mean-pooled query per block (C = 1) -> top-k;
  ideal_topk     the K blocks with the largest true attention mass of the query block
                 (the best any top-k selection can do on mass recall).
With --units, the same at the page's 4-token key units (third technique) for the same
number of tensor-core tiles (32 units per 128-key tile): unit4_ibcs_sip,
unit4_ibcs_topk, unit4_ideal_topk.

Everything but the dense reference runs through the library's kernels; the reference
(per-row block masses and O_dense) is plain fp32 PyTorch on the same device.

  python quality.py [--config wan13b] [--heads 2] [--budgets 0.05,0.1,0.2] [--seeds 4]
"""

from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402


def dense_reference(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, N: int,
                    rows_per_chunk: int = 1024, unit: int = 128):
    """Exact attention in fp32 for [B, H, N_pad, d] bf16 inputs on one device.

    Returns (O_dense fp32 [B, H, N_pad, d], mass fp32 [B, H, N_pad, N_pad / unit]) where
    mass[..., i, j] is the softmax probability mass of query row i on key unit j of
    `unit` tokens (keys t >= N excluded). Rows i >= N are zero in both."""
    B, H, N_pad, d = q.shape
    nkb = N_pad // unit
    o = torch.zeros(B, H, N_pad, d, device=q.device, dtype=torch.float32)
    mass = torch.zeros(B, H, N_pad, nkb, device=q.device, dtype=torch.float32)
    scale = 1.0 / d ** 0.5
    key_ok = torch.arange(N_pad, device=q.device) < N
    for b in range(B):
        for h in range(H):
            kf = k[b, h].float()
            vf = v[b, h].float()
            for r0 in range(0, N, rows_per_chunk):
                r1 = min(N, r0 + rows_per_chunk)
                logits = (q[b, h, r0:r1].float() @ kf.T) * scale
                logits.masked_fill_(~key_ok, float("-inf"))
                p = torch.softmax(logits, dim=-1)
                o[b, h, r0:r1] = p @ vf
                mass[b, h, r0:r1] = p.view(r1 - r0, nkb, unit).sum(-1)
    return o, mass


def mass_recall(mass: torch.Tensor, idx: torch.Tensor, cnt: torch.Tensor, N: int) -> float:
    """Mean over valid query rows of the true softmax mass on the selected key units
    (blocks of 128 or units of 4 tokens; query rows are grouped in blocks of 128).
    mass: [B, H, N_pad, n_ku]; idx: [B, H, n_qb, >= max cnt] (first cnt entries valid)."""
    B, H, N_pad, nkb = mass.shape
    nqb = N_pad // 128
    sel = torch.zeros(B, H, nqb, nkb, device=mass.device, dtype=torch.float32)
    pos = torch.arange(idx.shape[-1], device=mass.device)
    valid = pos.view(1, 1, 1, -1) < cnt.unsqueeze(-1)
    safe = torch.where(valid, idx.long(), torch.zeros_like(idx, dtype=torch.long))
    sel.scatter_add_(3, safe, valid.float())  # kept indices are distinct; padding adds 0
    per_row = (mass.view(B, H, nqb, 128, nkb) * sel.unsqueeze(3)).sum(-1).view(B, H, N_pad)
    return float(per_row[:, :, :N].mean())


def rel_error(o: torch.Tensor, o_ref: torch.Tensor, N: int) -> float:
    diff = (o[:, :, :N].float() - o_ref[:, :, :N])
    return float(diff.norm() / o_ref[:, :, :N].norm())


def ideal_scores(mass: torch.Tensor) -> torch.Tensor:
    """Per (query block, key block): the block's true mass averaged over the query
    block's rows; its top-k maximises the mean mass recall among top-k selections."""
    B, H, N_pad, nkb = mass.shape
    return mass.view(B, H, N_pad // 128, 128, nkb).mean(3).contiguous()


def evaluate(w, heads: int, budgets, seeds: int, device="cuda", units: bool = False):
    import block_sparse_attention_ab_b200 as ab
    from block_sparse_attention_ab_b200 import synth

    hs = list(range(min(heads, w.H))) if heads else None
    q, k, v = synth.make_qkv(w, heads=hs)
    qc, kc, vc = q.to(device), k.to(device), v.to(device)
    o_ref, mass = dense_reference(qc, kc, vc, w.N)
    s_ibcs = ab.score(qc, kc, w.N, w.n_clusters, w.iters)
    s_pool = ab.score(qc, kc, w.N, 1, 1)
    s_ideal = ideal_scores(mass)
    nkb = w.N_pad // 128
    if units:
        # the page's 4-token units at the same tile budget (32 units per 128-key tile)
        mass4 = dense_reference(qc, kc, vc, w.N, unit=4)[1]
        s_ibcs4 = ab.score(qc, kc, w.N, w.n_clusters, w.iters, unit=4)
        s_ideal4 = ideal_scores(mass4)
    rows = []
    for frac in budgets:
        K = max(1, int(frac * nkb + 0.5))
        res = {"budget_frac": frac, "budget_blocks": K}
        for name, s in (("ibcs_topk", s_ibcs), ("meanpool_topk", s_pool), ("ideal_topk", s_ideal)):
            idx, cnt, _ = ab.select(s, K, "topk")
            o = ab.attn_topk_fwd(qc, kc, vc, w.N, idx, cnt, out_dtype=torch.float32)
            res[name] = {"mass_recall": round(mass_recall(mass, idx, cnt, w.N), 5),
                         "attn_error": round(rel_error(o, o_ref, w.N), 5)}
        rec, err, kept = [], [], []
        for sd in range(seeds):
            idx, cnt, wt = ab.select(s_ibcs, K, "sip", w.sip_seed + sd)
            o = ab.attn_fwd(qc, kc, vc, w.N, idx, cnt, wt, out_dtype=torch.float32)
            rec.append(mass_recall(mass, idx, cnt, w.N))
            err.append(rel_error(o, o_ref, w.N))
            kept.append(float(cnt.float().mean()))
        res["ibcs_sip"] = {"mass_recall": round(float(np.mean(rec)), 5),
                           "attn_error": round(float(np.mean(err)), 5),
                           "mean_kept_blocks": round(float(np.mean(kept)), 2), "seeds": seeds}
        if units:
            K4 = 32 * K
            for name, s4 in (("unit4_ibcs_topk", s_ibcs4), ("unit4_ideal_topk", s_ideal4)):
                idx, cnt, _ = ab.select(s4, K4, "topk")
                o = ab.attn_topk_fwd(qc, kc, vc, w.N, idx, cnt, out_dtype=torch.float32, unit=4)
                res[name] = {"mass_recall": round(mass_recall(mass4, idx, cnt, w.N), 5),
                             "attn_error": round(rel_error(o, o_ref, w.N), 5)}
            rec, err = [], []
            for sd in range(seeds):
                idx, cnt, wt = ab.select(s_ibcs4, K4, "sip", w.sip_seed + sd)
                o = ab.attn_fwd(qc, kc, vc, w.N, idx, cnt, wt, out_dtype=torch.float32, unit=4)
                rec.append(mass_recall(mass4, idx, cnt, w.N))
                err.append(rel_error(o, o_ref, w.N))
            res["unit4_ibcs_sip"] = {"mass_recall": round(float(np.mean(rec)), 5),
                                     "attn_error": round(float(np.mean(err)), 5), "seeds": seeds}
        rows.append(res)
    return rows


def main():
    from block_sparse_attention_ab_b200 import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="wan13b")
    ap.add_argument("--heads", type=int, default=2, help="first H heads only (0 = all)")
    ap.add_argument("--budgets", default="0.05,0.1,0.2,0.3")
    ap.add_argument("--seeds", type=int, default=4)
    ap.add_argument("--units", action="store_true",
                    help="also the page's 4-token key units at the same tile budget")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.config]
    budgets = [float(x) for x in args.budgets.split(",")]
    rows = evaluate(w, args.heads, budgets, args.seeds, units=args.units)
    for r in rows:
        print(json.dumps({"workload": w.name, "heads": args.heads or w.H, **r}))


if __name__ == "__main__":
    main()
