"""The entry points under CUDA-graph capture and from several streams at once.

ab_score runs its mean-key pass on a library side stream forked from the caller's stream
(joined again before the block score) and falls back to in-order launches while the
caller's stream is being captured. These tests check that a captured and replayed path
equals the eager calls bit for bit, on new inputs copied into the captured buffers, and
that ab_score calls issued concurrently from two streams give the eager results.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


def _qkv(N, H=2, d=128, seed=0):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    t = torch.zeros(3, 1, H, N_pad, d)
    t[:, :, :, :N] = torch.randn(3, 1, H, N, d, generator=g)
    q, k, v = t.to(torch.bfloat16).cuda().unbind(0)
    return q.contiguous(), k.contiguous(), v.contiguous()


def _path(q, k, v, N, budget, seed, bufs):
    s = ab.score(q, k, N, workspace=bufs["ws"], out=bufs["s"])
    idx, cnt, w = ab.select(s, budget, "sip", seed, out=(bufs["idx"], bufs["cnt"], bufs["w"]))
    return ab.attn_fwd(q, k, v, N, idx, cnt, w, out=bufs["o"])


def _bufs(q, N):
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    dev = q.device
    shape = ab.make_shape(q, N)
    return {
        "ws": torch.empty(ab.score_workspace_bytes(shape), device=dev, dtype=torch.uint8),
        "s": torch.empty(B, H, nb, nb, device=dev),
        "idx": torch.empty(B, H, nb, nb, device=dev, dtype=torch.int32),
        "cnt": torch.empty(B, H, nb, device=dev, dtype=torch.int32),
        "w": torch.empty(B, H, nb, nb, device=dev),
        "o": torch.empty_like(q),
    }


def test_captured_path_equals_eager():
    N, budget, seed = 1636, 4, 3
    q, k, v = _qkv(N, seed=1)
    bufs = _bufs(q, N)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _path(q, k, v, N, budget, seed, bufs)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _path(q, k, v, N, budget, seed, bufs)
    for data_seed in (7, 8):
        q2, k2, v2 = _qkv(N, seed=data_seed)
        eager = _bufs(q2, N)
        _path(q2, k2, v2, N, budget, seed, eager)
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        for name in ("s", "idx", "cnt", "w", "o"):
            a, b = bufs[name].cpu(), eager[name].cpu()
            assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                               b.view(torch.int32) if b.dtype == torch.float32 else b), name


def test_scores_from_two_streams_at_once():
    N = 3000
    inputs = [_qkv(N, H=3, seed=s) for s in (11, 12)]
    ref = [ab.score(q, k, N) for q, k, _ in inputs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [None, None]
    for rep in range(3):
        for i, st in enumerate(streams):
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                q, k, _ = inputs[i]
                outs[i] = ab.score(q, k, N)
        for st in streams:
            torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        for i in range(2):
            np.testing.assert_array_equal(outs[i].cpu().numpy().view(np.uint32),
                                          ref[i].cpu().numpy().view(np.uint32))
