"""Failure detection without a GPU fault: an in-kernel wait on an mbarrier that nothing
completes must give up after its limit, report AB_FLAG_TIMEOUT through the device flag
and return, leaving the CUDA context usable for the next call (the bounded wait every
pipeline role of the library uses)."""

import time

import numpy as np
import pytest
import torch

import block_sparse_attention_ab_b200 as ab

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_ab_b200 import build
    build.build()
    ab.lib()


def test_wait_that_nothing_completes_times_out_and_reports():
    t0 = time.perf_counter()
    bits, done = ab.selftest_bounded_wait(20000, complete=False)  # 20 ms limit
    elapsed = time.perf_counter() - t0
    assert bits & ab.FLAG_TIMEOUT
    assert done == 2
    assert elapsed < 5.0


def test_completed_wait_reports_nothing():
    bits, done = ab.selftest_bounded_wait(20000, complete=True)
    assert bits == 0
    assert done == 1


def test_context_stays_usable_after_a_timeout(orc):
    ab.selftest_bounded_wait(5000, complete=False)
    # a normal attention call afterwards still matches the oracle
    g = torch.Generator().manual_seed(0)
    N, d = 300, 64
    q, k, v = (torch.zeros(1, 1, 384, d, dtype=torch.bfloat16) for _ in range(3))
    for t in (q, k, v):
        t[:, :, :N] = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    idx = torch.tensor([[[[0, 1, 2], [0, 2, -1], [1, -1, -1]]]], dtype=torch.int32)
    cnt = torch.tensor([[[3, 2, 1]]], dtype=torch.int32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ab.attn_topk_fwd(q.cuda(), k.cuda(), v.cuda(), N, idx.cuda(), cnt.cuda(), dev_flag=flag,
                           out_dtype=torch.float32)
    assert ab.check_flag(flag) == 0
    ref, _, _, _ = orc.attn_rows(q, k, v, N, idx.numpy(), cnt.numpy())
    np.testing.assert_allclose(out.cpu().numpy().reshape(3, 128, d), ref, atol=1e-2)


def test_selftest_argument_checks():
    L = ab.lib()
    assert L.ab_selftest_bounded_wait(0, 0, None, None, None) == 1
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.ab_selftest_bounded_wait(0, 0, ab._ptr(flag), ab._ptr(flag), None) == 5
