"""Host-side checks of the C ABI: the library loads, exports every entry point that
include/ab_attn.h declares, and rejects bad arguments synchronously with the documented
status codes. Nothing here launches a kernel, so it runs without a GPU."""

import ctypes
import os
import re

import pytest

import block_sparse_attention_ab_b200 as ab
from block_sparse_attention_ab_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ab_attn.h")

FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: every call below fails first
MISALIGNED = ctypes.c_void_p(0x10008)


@pytest.fixture(scope="module")
def L():
    build.build()
    return ab.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ab_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert {"ab_score", "ab_select", "ab_attn_fwd", "ab_attn_topk_fwd"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in ab.STATUS.items():
        assert L.ab_status_str(code).decode() == name
    assert L.ab_version() >= 100


def shape(B=1, H=2, N=1000, N_pad=1024, d=64, dtype=ab.AB_BF16):
    return ab.Shape(B, H, N, N_pad, d, dtype)


def test_workspace_size(L):
    n = ctypes.c_size_t(0)
    assert L.ab_score_workspace_size(shape(), 8, ctypes.byref(n)) == 0
    nb = 8
    # mean keys, centroids, cluster weights (fp32), the two fp16 terms of the scaled mean
    # keys and their unscale factors (fp32 rows padded to 256 entries)
    need = 2 * nb * 64 * 4 + 2 * nb * 8 * 64 * 4 + 2 * nb * 8 * 4 + 2 * 2 * nb * 64 * 2 + 2 * 256 * 4
    assert need <= n.value <= need + 5 * 256
    assert L.ab_score_workspace_size(shape(), 9, ctypes.byref(n)) == 4
    assert n.value == 0
    assert L.ab_score_workspace_size(shape(N=1024, N_pad=1000), 8, ctypes.byref(n)) == 2


@pytest.mark.parametrize("bad,code", [
    (dict(B=0), 2), (dict(N=0), 2), (dict(N_pad=1000), 2), (dict(N=1025), 2),
    (dict(N=800), 2),  # N_pad - N >= 128
    (dict(dtype=0), 3), (dict(d=96), 4), (dict(d=256), 4),
    (dict(N=128 * 8193, N_pad=128 * 8193), 5),
])
def test_shape_rejections(L, bad, code):
    s = shape(**bad)
    assert L.ab_attn_topk_fwd(FAKE, FAKE, FAKE, s, FAKE, FAKE, FAKE, ab.AB_BF16, None, None,
                              None) == code
    assert L.ab_attn_fwd(FAKE, FAKE, FAKE, s, FAKE, FAKE, FAKE, FAKE, ab.AB_F32, None, None,
                         None) == code
    assert L.ab_score(FAKE, FAKE, s, 8, 5, FAKE, None, None, None, None, FAKE, 1 << 40, None,
                      None) == code


def test_null_and_alignment(L):
    s = shape()
    B16 = ab.AB_BF16
    assert L.ab_attn_fwd(None, FAKE, FAKE, s, FAKE, FAKE, FAKE, FAKE, B16, None, None, None) == 1
    assert L.ab_attn_fwd(FAKE, FAKE, FAKE, s, FAKE, FAKE, None, FAKE, B16, None, None, None) == 1
    assert L.ab_attn_fwd(FAKE, MISALIGNED, FAKE, s, FAKE, FAKE, FAKE, FAKE, B16, None, None,
                         None) == 9
    assert L.ab_attn_fwd(FAKE, FAKE, FAKE, s, FAKE, FAKE, FAKE, FAKE, 7, None, None, None) == 3
    assert L.ab_attn_topk_fwd(FAKE, FAKE, FAKE, s, FAKE, FAKE, FAKE, 2, None, None, None) == 3
    assert L.ab_score(FAKE, FAKE, s, 8, 5, None, None, None, None, None, FAKE, 1 << 40, None,
                      None) == 1
    assert L.ab_score(FAKE, FAKE, s, 8, 5, MISALIGNED, None, None, None, None, FAKE, 1 << 40,
                      None, None) == 9


def test_score_argument_checks(L):
    s = shape()
    n = ctypes.c_size_t(0)
    L.ab_score_workspace_size(s, 8, ctypes.byref(n))
    assert L.ab_score(FAKE, FAKE, s, 0, 5, FAKE, None, None, None, None, FAKE, n.value, None,
                      None) == 4
    assert L.ab_score(FAKE, FAKE, s, 8, 0, FAKE, None, None, None, None, FAKE, n.value, None,
                      None) == 5
    assert L.ab_score(FAKE, FAKE, s, 8, 5, FAKE, None, None, None, None, None, n.value, None,
                      None) == 10
    assert L.ab_score(FAKE, FAKE, s, 8, 5, FAKE, None, None, None, None, FAKE, n.value - 1,
                      None, None) == 10


def test_select_argument_checks(L):
    u = ctypes.c_uint64(0)
    assert L.ab_select(None, 1, 1, 8, 8, 3, 0, u, FAKE, FAKE, FAKE, None, None, None) == 1
    assert L.ab_select(FAKE, 1, 1, 8, 8, 3, 0, u, FAKE, FAKE, None, None, None, None) == 1
    assert L.ab_select(FAKE, 1, 1, 8, 8, 3, 7, u, FAKE, FAKE, FAKE, None, None, None) == 4
    assert L.ab_select(FAKE, 0, 1, 8, 8, 3, 0, u, FAKE, FAKE, FAKE, None, None, None) == 2
    assert L.ab_select(FAKE, 1, 1, 8, 8, 0, 0, u, FAKE, FAKE, FAKE, None, None, None) == 5
    assert L.ab_select(FAKE, 1, 1, 8, 65537, 3, 1, u, FAKE, FAKE, None, None, None, None) == 5
    assert L.ab_select(MISALIGNED, 1, 1, 8, 8, 3, 1, u, FAKE, FAKE, None, None, None, None) == 9


def test_check_flag_null(L):
    host = ctypes.c_int(0)
    assert L.ab_check_flag(None, ctypes.byref(host), None) == 1


def test_product_path_has_no_fallback(monkeypatch, tmp_path):
    """Without the shared library the binding raises instead of computing on the CPU."""
    monkeypatch.setattr(ab, "_lib", None)
    monkeypatch.setattr(ab, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        ab.lib()


def test_product_package_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "block_sparse_attention_ab_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text and "ab_oracle" not in text, f


def test_unit_entry_points_reject_bad_units(L):
    s = shape()
    n = ctypes.c_size_t(0)
    # key units: 128-token blocks or the page's 4-token units only
    assert L.ab_score_units_workspace_size(s, 8, 8, ctypes.byref(n)) == 4
    assert L.ab_attn_units_fwd(FAKE, FAKE, FAKE, s, 16, FAKE, FAKE, FAKE, FAKE, ab.AB_BF16, None,
                               None, None) == 4
    assert L.ab_attn_units_topk_fwd(FAKE, FAKE, FAKE, s, 2, FAKE, FAKE, FAKE, ab.AB_BF16, None,
                                    None, None) == 4
    # at most AB_MAX_UNITS = 65536 units per head: 4-token units need N_pad <= 262144
    ok = shape(N=262144, N_pad=262144)
    assert L.ab_score_units_workspace_size(ok, 8, 4, ctypes.byref(n)) == 0
    big = shape(N=262144 + 128, N_pad=262144 + 128)
    assert L.ab_score_units_workspace_size(big, 8, 4, ctypes.byref(n)) == 5
    assert L.ab_attn_units_topk_fwd(FAKE, FAKE, FAKE, big, 4, FAKE, FAKE, FAKE, ab.AB_BF16, None,
                                    None, None) == 5
    assert L.ab_score_units(FAKE, FAKE, big, 8, 5, 4, FAKE, None, None, None, None, FAKE, 1 << 40,
                            None, None) == 5
    assert L.ab_attn_units_fwd(FAKE, FAKE, FAKE, s, 4, FAKE, FAKE, None, FAKE, ab.AB_BF16, None,
                               None, None) == 1


def test_select_row_length_limit(L):
    # rows of up to AB_MAX_UNITS entries; a longer row is rejected before any launch
    assert L.ab_select(FAKE, 1, 1, 1, 65537, 4, 0, 0, FAKE, FAKE, FAKE, None, None, None) == 5


def test_unit_workspace_size(L):
    n = ctypes.c_size_t(0)
    assert L.ab_score_units_workspace_size(shape(), 8, 4, ctypes.byref(n)) == 0
    nqb, nku = 8, 256
    # mean keys [2, nku, 64] fp32, centroids and weights per query block, fp16 key terms,
    # unscale factors
    need = 2 * nku * 64 * 4 + 2 * nqb * 8 * 64 * 4 + 2 * nqb * 8 * 4 + 2 * 2 * nku * 64 * 2 + 2 * 256 * 4
    assert need <= n.value <= need + 5 * 256
    m = ctypes.c_size_t(0)
    assert L.ab_score_units_workspace_size(shape(), 8, 128, ctypes.byref(m)) == 0
    L.ab_score_workspace_size(shape(), 8, ctypes.byref(n))
    assert m.value == n.value


def test_forward_host_argument_checks(L):
    # every rejection comes before any CUDA call: no device is touched
    s = ab.Shape(1, 4, 1000, 1024, 128, ab.AB_BF16)
    B16 = ab.AB_BF16
    n = ctypes.c_size_t(0)
    assert L.ab_forward_host_workspace_size(s, 8, 2, B16, ctypes.byref(n)) == 0
    # two slots of Q, K, V (bf16) and O for 2 head pairs, plus one chunk's scoring work
    assert n.value >= 2 * 4 * 2 * 1024 * 128 * 2
    assert L.ab_forward_host_workspace_size(s, 8, 0, B16, ctypes.byref(n)) == 5
    assert L.ab_forward_host_workspace_size(s, 8, 5, B16, ctypes.byref(n)) == 5
    assert L.ab_forward_host_workspace_size(s, 9, 2, B16, ctypes.byref(n)) == 4
    assert L.ab_forward_host_workspace_size(s, 8, 2, 7, ctypes.byref(n)) == 3
    assert L.ab_forward_host_workspace_size(s, 8, 2, B16, None) == 1
    assert L.ab_forward_host_workspace_size(s, 8, 2, B16, ctypes.byref(n)) == 0
    need = n.value
    u = ctypes.c_uint64(1)
    call = L.ab_forward_host
    assert call(None, FAKE, FAKE, s, 8, 5, 0, 3, u, FAKE, B16, 2, FAKE, need, None, None) == 1
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 3, u, None, B16, 2, FAKE, need, None, None) == 1
    assert call(FAKE, FAKE, FAKE, s, 8, 0, 0, 3, u, FAKE, B16, 2, FAKE, need, None, None) == 5
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 0, u, FAKE, B16, 2, FAKE, need, None, None) == 5
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 3, 3, u, FAKE, B16, 2, FAKE, need, None, None) == 4
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 3, u, FAKE, B16, 9, FAKE, need, None, None) == 5
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 3, u, FAKE, B16, 2, MISALIGNED, need, None, None) == 9
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 3, u, FAKE, B16, 2, None, need, None, None) == 10
    assert call(FAKE, FAKE, FAKE, s, 8, 5, 0, 3, u, FAKE, B16, 2, FAKE, need - 1, None, None) == 10
    bad = ab.Shape(1, 4, 1000, 1152, 128, ab.AB_BF16)  # N_pad - N >= 128
    assert call(FAKE, FAKE, FAKE, bad, 8, 5, 0, 3, u, FAKE, B16, 2, FAKE, need, None, None) == 2


def test_attn_bwd_argument_checks(L):
    # every rejection comes before any CUDA call: no device is touched
    s = ab.Shape(1, 2, 1000, 1024, 128, ab.AB_BF16)
    n = ctypes.c_size_t(0)
    assert L.ab_attn_bwd_workspace_size(s, ctypes.byref(n)) == 0
    # D_i and lse_i log2e per query row (fp32), the n_kb x n_qb uint16 mark table and a
    # uint32 count per key block, per head
    need = 2 * 2 * 1024 * 4 + 2 * 8 * 8 * 2 + 2 * 8 * 4
    assert need <= n.value <= need + 4 * 256
    assert L.ab_attn_bwd_workspace_size(s, None) == 1
    assert L.ab_attn_bwd_workspace_size(ab.Shape(1, 2, 1000, 1024, 96, ab.AB_BF16), ctypes.byref(n)) == 4
    assert n.value == 0
    assert L.ab_attn_bwd_workspace_size(s, ctypes.byref(n)) == 0
    need = n.value
    B16 = ab.AB_BF16
    call = L.ab_attn_bwd
    args = [FAKE, FAKE, FAKE, s, FAKE, FAKE, FAKE, FAKE, B16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            need, None, None]

    def with_(**kw):
        a = list(args)
        pos = dict(q=0, k=1, v=2, s=3, idx=4, cnt=5, w=6, out=7, odt=8, lse=9, do=10, dq=11,
                   dk=12, dv=13, ws=14, wsb=15)
        for key, val in kw.items():
            a[pos[key]] = val
        return call(*a)

    for key in ("q", "k", "v", "idx", "cnt", "out", "lse", "do", "dq", "dk", "dv"):
        assert with_(**{key: None}) == 1, key
    assert with_(odt=7) == 3
    assert with_(s=ab.Shape(1, 2, 1000, 1024, 128, 0)) == 3
    assert with_(s=ab.Shape(1, 2, 1000, 1152, 128, B16)) == 2
    assert with_(s=ab.Shape(1, 2, 1000, 1024, 256, B16)) == 4
    for key in ("q", "dq", "do", "lse", "w", "ws"):
        assert with_(**{key: MISALIGNED}) == 9, key
    assert with_(ws=None) == 10
    assert with_(wsb=need - 1) == 10
    assert "ab_attn_bwd" in declared_functions()
    # the wait-limit test entry: a device flag and a limit in 1..1e9 ns are required
    sw = L.ab_selftest_attn_bwd_wait_limit
    base = args[:16]
    assert sw(*base, None, 1000, None) == 1
    assert sw(*base, FAKE, 0, None) == 5
    assert sw(*base, FAKE, 1_000_000_001, None) == 5
    bad = list(base)
    bad[0] = None
    assert sw(*bad, FAKE, 1000, None) == 1
