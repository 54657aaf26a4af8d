"""ab_score_noalloc: IBCS scoring for callers that cannot allocate device memory.

Some callers -- a plugin or custom operator inside a host framework that owns all
device memory, or code with no allocator of its own -- can neither call cudaMalloc nor
pass the library a workspace. ab_score_noalloc serves them: it runs the same scoring
kernels as ab_score, with the scratch in a fixed array inside the library. These tests
call it through the C ABI and compare its scores with ab_score's on the same inputs,
for two calls in a row (the second on different inputs, so anything left behind in
the shared scratch by the first call would show), and check the size limit.

The file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import synth

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-4  # the block-score tolerance used by the parity tests


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_ab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ab.lib()


def _inputs(N, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    N_pad = (N + 127) // 128 * 128
    q = torch.zeros(1, H, N_pad, d)
    k = torch.zeros_like(q)
    q[:, :, :N] = torch.randn(1, H, N, d, generator=g)
    k[:, :, :N] = torch.randn(1, H, N, d, generator=g)
    return q.to(torch.bfloat16).cuda(), k.to(torch.bfloat16).cuda()


def _noalloc(lib, q, k, N, C=8, T=5):
    B, H, N_pad, d = q.shape
    nb = N_pad // 128
    out = torch.full((B, H, nb, nb), float("nan"), device=q.device, dtype=torch.float32)
    code = lib.ab_score_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                ab.make_shape(q, N), C, T, ctypes.c_void_p(out.data_ptr()), None,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0, ab.STATUS.get(code, code)
    return out


def _agree(a, b):
    a = a.cpu().numpy()
    b = b.cpu().numpy()
    assert np.all(np.isfinite(a))
    assert np.all(np.abs(a - b) <= SCORE_RTOL * np.abs(b) + 1e-30)


def test_noalloc_matches_ab_score_two_calls(lib):
    w = synth.WORKLOADS["tiny"]
    q1, k1, _ = (t.cuda() for t in synth.make_qkv(w))
    q2, k2 = _inputs(9 * 128 + 40, H=3, d=128, seed=21)
    first = _noalloc(lib, q1, k1, w.N)
    second = _noalloc(lib, q2, k2, 9 * 128 + 40)
    torch.cuda.synchronize()
    _agree(first, ab.score(q1, k1, w.N))
    _agree(second, ab.score(q2, k2, 9 * 128 + 40))


def test_noalloc_wan_sized_call_and_repeat(lib):
    # 4 heads of the Wan2.1-1.3B shape: 4.8 MB of scratch
    N = 32760
    q, k = _inputs(N, H=4, d=128, seed=5)
    ref = ab.score(q, k, N)
    for _ in range(2):
        _agree(_noalloc(lib, q, k, N), ref)


def test_noalloc_rejects_problems_above_the_limit(lib):
    # 24 heads x 118912 tokens (HunyuanVideo shape) needs ~103 MB of scratch
    s = ab.Shape(1, 24, 118800, 118912, 128, ab.AB_BF16)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    n = ctypes.c_size_t(0)
    assert lib.ab_score_workspace_size(s, 8, ctypes.byref(n)) == 0
    assert n.value > 32 * 1024 * 1024
    assert lib.ab_score_noalloc(fake, fake, s, 8, 5, fake, None, None) == 10  # AB_ERR_WORKSPACE
