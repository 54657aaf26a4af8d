"""GPU: guard canaries around every output and workspace. Each buffer the library writes
is carved out of a larger allocation whose bytes are first set to a sentinel; after the
call the guard regions before and after it must still hold the sentinel, so a kernel that
writes past its buffer (a ragged tail, a padding row, an index off by one) fails here even
when the result itself looks right.
"""

import pytest
import torch

import block_sparse_attention_ab_b200 as ab

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps every view 16-byte aligned)
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ab.lib()


class Guarded:
    """A device tensor of `shape` / `dtype` inside a sentinel-filled allocation."""

    def __init__(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        return bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())


def _inputs(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    out = []
    for _ in range(3):
        t = torch.zeros(B, H, N_pad, d)
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g)
        out.append(t.to(torch.bfloat16).cuda())
    return out


@pytest.mark.parametrize("unit", [128, 4])
@pytest.mark.parametrize("d", [128, 64])
def test_outputs_and_workspace_stay_in_bounds(unit, d):
    B, H, N = 1, 3, 1000  # ragged: N_pad = 1024
    q, k, v = _inputs(B, H, N, d, seed=d + unit)
    N_pad = q.shape[2]
    nqb, nku = N_pad // 128, N_pad // unit
    shape = ab.make_shape(q, N)
    ws = Guarded((ab.score_workspace_bytes(shape, 8, unit),), torch.uint8)
    scores = Guarded((B, H, nqb, nku), torch.float32)
    ab.score(q, k, N, 8, 5, workspace=ws.t, out=scores.t, unit=unit)
    assert ws.intact() and scores.intact()
    budget = 3 if unit == 128 else 3 * 32
    for mode in ("sip", "topk"):
        idx = Guarded((B, H, nqb, nku), torch.int32)
        cnt = Guarded((B, H, nqb), torch.int32)
        w = Guarded((B, H, nqb, nku), torch.float32)
        ab.select(scores.t, budget, mode, 7, out=(idx.t, cnt.t, w.t))
        assert idx.intact() and cnt.intact() and w.intact(), mode
        for out_dtype in (torch.bfloat16, torch.float32):
            out = Guarded(q.shape, out_dtype)
            if mode == "sip":
                o, lse = ab.attn_fwd(q, k, v, N, idx.t, cnt.t, w.t, want_lse=True, out=out.t,
                                     out_dtype=out_dtype, unit=unit)
            else:
                o, lse = ab.attn_topk_fwd(q, k, v, N, idx.t, cnt.t, want_lse=True, out=out.t,
                                          out_dtype=out_dtype, unit=unit)
            assert out.intact(), (mode, out_dtype)
            assert torch.isfinite(o.float()).all()
            # padding rows are written as zeros
            assert torch.all(o[:, :, N:] == 0)


def test_host_path_workspace_stays_in_bounds():
    B, H, N, d = 1, 5, 700, 128
    q, k, v = (t.cpu().pin_memory() for t in _inputs(B, H, N, d, seed=3))
    shape = ab.make_shape(q, N)
    ws = Guarded((ab.forward_host_workspace_bytes(shape, 8, 2),), torch.uint8)
    out = ab.forward_host(q, k, v, N, 2, "sip", 1, chunk_heads=2, workspace=ws.t)
    torch.cuda.synchronize()
    assert ws.intact()
    assert torch.all(out[:, :, N:] == 0)
