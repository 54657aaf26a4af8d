"""GPU: the host-buffer entry point ab_forward_host (chunks of head pairs copied in,
scored, selected and attended while neighbouring chunks copy) against the device calls
on the whole tensors, and an oracle spot check of its output.

Bar: bit-exact equality with ab_score -> ab_select -> ab_attn_fwd / ab_attn_topk_fwd on
the same inputs and seed (every stage works per (b, h) and SIP keys its random numbers
by the global (b, h)), for every chunk size, both output dtypes and pageable as well as
page-locked host memory; the oracle check uses the attention tolerances of the parity
tests (max |O - O_ref| <= 1e-2 on fp32 output, Frobenius 5e-3).
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


def _inputs(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    out = []
    for _ in range(3):
        t = torch.zeros(B, H, N_pad, d)
        t[:, :, :N] = torch.randn(B, H, N, d, generator=g)
        out.append(t.to(torch.bfloat16))
    return out


def _device_path(q, k, v, N, budget, mode, seed, out_dtype):
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    s = ab.score(qc, kc, N, 8, 5)
    idx, cnt, w = ab.select(s, budget, mode, seed)
    if mode == "sip":
        o = ab.attn_fwd(qc, kc, vc, N, idx, cnt, w, out_dtype=out_dtype)
    else:
        o = ab.attn_topk_fwd(qc, kc, vc, N, idx, cnt, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return o.cpu(), (idx, cnt, w)


@pytest.mark.parametrize("mode", ["sip", "topk"])
@pytest.mark.parametrize("d", [128, 64])
def test_forward_host_equals_device_calls(mode, d):
    B, H, N = 2, 3, 1000  # ragged tail: N_pad = 1024, 8 blocks
    q, k, v = _inputs(B, H, N, d, seed=3 + d)
    budget, seed = 3, 0x1234_5678_9ABC
    for out_dtype in (torch.float32, torch.bfloat16):
        ref, _ = _device_path(q, k, v, N, budget, mode, seed, out_dtype)
        qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
        for ch in (1, 2, 4, B * H):
            flag = torch.zeros(1, dtype=torch.int32, device="cuda")
            got = ab.forward_host(qp, kp, vp, N, budget, mode, seed, out_dtype=out_dtype,
                                  chunk_heads=ch, dev_flag=flag)
            assert ab.check_flag(flag) == 0
            torch.cuda.synchronize()
            assert torch.equal(got, ref), (mode, d, out_dtype, ch)
        # pageable host memory: same result
        got = ab.forward_host(q, k, v, N, budget, mode, seed, out_dtype=out_dtype, chunk_heads=4)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)


def test_forward_host_against_oracle(orc):
    B, H, N, d = 1, 4, 2000, 128
    q, k, v = _inputs(B, H, N, d, seed=21)
    budget, seed = 6, 77
    ref_dev, (idx, cnt, w) = _device_path(q, k, v, N, budget, "sip", seed, torch.float32)
    # the host buffers must live until the stream is done with them
    pinned = [t.pin_memory() for t in (q, k, v)]
    got = ab.forward_host(*pinned, N, budget, "sip", seed, out_dtype=torch.float32, chunk_heads=3)
    torch.cuda.synchronize()
    assert torch.equal(got, ref_dev)
    nqb = q.shape[2] // 128
    rows = np.arange(0, B * H * nqb, 3, dtype=np.int64)
    ref, _, _, _ = orc.attn_rows(q, k, v, N, idx.cpu().numpy(), cnt.cpu().numpy(), w.cpu().numpy(),
                                 rows=rows)
    og = got.numpy().reshape(B * H * nqb, 128, d)[rows]
    assert np.abs(og - ref).max() <= 1e-2
    assert np.linalg.norm(og - ref) / np.linalg.norm(ref) <= 5e-3


def test_forward_host_repeated_calls_and_reused_workspace():
    # back-to-back calls on one stream reuse the workspace slots and the library's
    # events: each call's output must still be its own
    B, H, N, d = 1, 5, 700, 128
    outs = []
    ws = torch.empty(ab.forward_host_workspace_bytes(ab.Shape(B, H, N, 768, d, ab.AB_BF16), 8, 2),
                     dtype=torch.uint8, device="cuda")
    inputs = [_inputs(B, H, N, d, seed=s) for s in (1, 2, 3)]
    # every call's host buffers stay alive until the stream is done with them
    pinned = [[t.pin_memory() for t in qkv] for qkv in inputs]
    for qp, kp, vp in pinned:
        outs.append(ab.forward_host(qp, kp, vp, N, 2, "sip", 5, chunk_heads=2, workspace=ws))
    torch.cuda.synchronize()
    for (q, k, v), got in zip(inputs, outs):
        ref, _ = _device_path(q, k, v, N, 2, "sip", 5, torch.bfloat16)
        assert torch.equal(got, ref)
