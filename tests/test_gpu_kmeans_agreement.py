"""How closely the GPU's per-block k-means follows the oracle on the named workloads,
measured on whole heads and reported (printed, and written as JSON to $AB_REPORT_DIR
when that is set).

Per workload and sampled head, over every query block:
  * near-tie blocks: the oracle's smallest relative gap between the best and second-best
    squared distance, over all queries and iterations, is below 1e-5 (the reading of
    "distance gap < 1e-5" as relative);
  * blocks whose final assignments differ from the oracle's; every such block must be a
    near-tie block (asserted), and its GPU centroids must still be the means of its GPU
    members (asserted: the GPU state is a consistent k-means state, so the difference
    is a tie broken the other way, carried through the later iterations);
  * the end-to-end score error: GPU scores against the oracle's scores computed from the
    oracle's own k-means and mean keys (independent k-means on both sides), overall and on
    the rows of blocks without a near tie.
"""

import json
import os

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import synth

pytestmark = pytest.mark.gpu

TIE_GAP = 1e-5
SCORE_RTOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


_REPORT = {}


@pytest.mark.parametrize("name,heads", [("wan13b", [0, 7]), ("wan14b", [3, 29]),
                                        ("hunyuan720", [5]), ("long", [2])])
def test_kmeans_agreement_report(orc, name, heads):
    w = synth.WORKLOADS[name]
    q, k, _ = synth.make_qkv(w, heads=heads)
    qc, kc = q.cuda(), k.cuda()
    s, kbar, cent, cw, assign = ab.score(qc, kc, w.N, w.n_clusters, w.iters, intermediates=True)
    torch.cuda.synchronize()
    s_g = s.cpu().numpy().astype(np.float64)
    asg_g = assign.cpu().numpy()
    cent_g = cent.cpu().numpy().astype(np.float64)
    cw_g = cw.cpu().numpy()
    cent_r, wts_r, asg_r, gap_r, _ = orc.kmeans(q, w.N, w.n_clusters, w.iters)
    s_r = orc.score(cent_r, wts_r, orc.mean_key(k, w.N))
    H, nb = len(heads), w.n_blocks
    near = gap_r < TIE_GAP                               # [1, H, nb]
    blk_asg_g = asg_g.reshape(1, H, nb, 128)
    blk_asg_r = asg_r.reshape(1, H, nb, 128)
    differ = np.any(blk_asg_g != blk_asg_r, axis=-1)     # [1, H, nb]
    assert not np.any(differ & ~near), "assignments differ in a block without a near tie"
    qf = q.float().numpy().reshape(1, H, nb, 128, -1).astype(np.float64)
    for (b, h, j) in zip(*np.nonzero(differ)):
        nv = min(128, w.N - j * 128)
        for c in range(w.n_clusters):
            m = blk_asg_g[b, h, j, :nv] == c
            if m.any():
                np.testing.assert_allclose(cent_g[b, h, j, c], qf[b, h, j, :nv][m].mean(0),
                                           rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(cw_g[b, h, j].sum(), 1.0, rtol=1e-6)
    rel = np.abs(s_g - s_r) / np.maximum(np.abs(s_r), 1e-30)
    clean = ~near[..., None] & np.ones_like(rel, dtype=bool)
    rec = {"heads": heads, "blocks": int(H * nb),
           "near_tie_blocks": int(near.sum()), "near_tie_rate": float(near.mean()),
           "blocks_with_different_assignments": int(differ.sum()),
           "score_rel_err_max": float(rel.max()),
           "score_rel_err_max_without_near_ties": float(rel[clean].max(initial=0.0)),
           "score_rel_err_p99": float(np.quantile(rel, 0.99))}
    _REPORT[name] = rec
    print(name, json.dumps(rec))
    # scores of blocks without a near tie agree as the parity tests require
    assert rec["score_rel_err_max_without_near_ties"] <= SCORE_RTOL
    out_dir = os.environ.get("AB_REPORT_DIR")
    if out_dir:
        os.makedirs(out_dir, exist_ok=True)
        with open(os.path.join(out_dir, "kmeans_agreement.json"), "w") as f:
            json.dump(_REPORT, f, indent=1)
