"""CPU oracle for the AB-Attention hot path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline / reference leg may
import this package. It wraps ``ab_oracle.c`` (plain C, fp64, OpenMP over rows), which
is compiled with gcc into ``liboracle.so`` next to this file. It shares no code with
the CUDA library.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ab_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BLOCK = 128


def build(force: bool = False) -> str:
    """Compile ab_oracle.c with gcc (no fused multiply-add contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-Wall", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, u64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_philox4x32_10.restype = None
        L.orc_mean_key.argtypes = [P, i32, i32, i32, i32, i32, P]
        L.orc_mean_key_u.argtypes = [P, i32, i32, i32, i32, i32, i32, P]
        L.orc_score_u.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, P]
        L.orc_attn_rows_u.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i64, P, P,
                                      P, P, P]
        L.orc_kmeans.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P]
        L.orc_score.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P]
        L.orc_sip.argtypes = [P, i32, i32, i32, i32, i32, u64, P, P, P, P, P]
        L.orc_topk.argtypes = [P, i32, i32, i32, i32, i32, P, P, P]
        L.orc_attn_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P, i64, P, P, P, P,
                                    P]
        L.orc_dense_attn.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P]
        L.orc_attn_bwd.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P]
        L.orc_num_threads.argtypes = []
        for name in ("orc_mean_key", "orc_kmeans", "orc_score", "orc_sip", "orc_topk",
                     "orc_attn_rows", "orc_dense_attn", "orc_num_threads", "orc_mean_key_u",
                     "orc_score_u", "orc_attn_rows_u", "orc_attn_bwd"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 bit patterns as a contiguous uint16 numpy array (accepts torch bf16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16
    return x


def num_threads() -> int:
    return int(lib().orc_num_threads())


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def mean_key(k, N: int, unit: int = BLOCK) -> np.ndarray:
    """Mean key per key unit of `unit` tokens [B, H, N_pad / unit, d] (units with no
    valid token are 0)."""
    kb = _bits(k)
    B, H, N_pad, d = kb.shape
    out = np.zeros((B, H, N_pad // unit, d), dtype=np.float64)
    rc = lib().orc_mean_key_u(_ptr(kb), B, H, N, N_pad, d, unit, _ptr(out))
    if rc:
        raise ValueError(f"orc_mean_key rc={rc}")
    return out


def kmeans(q, N: int, C: int, T: int):
    """Returns (centroids [B,H,nqb,C,d], weights [B,H,nqb,C], assign [B,H,N_pad] uint8,
    min_gap [B,H,nqb], inertia [B,H,nqb,T])."""
    qb = _bits(q)
    B, H, N_pad, d = qb.shape
    nqb = N_pad // BLOCK
    cent = np.zeros((B, H, nqb, C, d), dtype=np.float64)
    wts = np.zeros((B, H, nqb, C), dtype=np.float64)
    assign = np.zeros((B, H, N_pad), dtype=np.uint8)
    gap = np.zeros((B, H, nqb), dtype=np.float64)
    inert = np.zeros((B, H, nqb, T), dtype=np.float64)
    rc = lib().orc_kmeans(_ptr(qb), B, H, N, N_pad, d, C, T, _ptr(cent), _ptr(wts), _ptr(assign),
                          _ptr(gap), _ptr(inert))
    if rc:
        raise ValueError(f"orc_kmeans rc={rc}")
    return cent, wts, assign, gap, inert


def score(cent, wts, kbar, n_valid: int = 0) -> np.ndarray:
    """IBCS scores over the key units of `kbar`; only the first `n_valid` units exist
    (0 = all), the rest score 0."""
    cent = np.ascontiguousarray(cent, dtype=np.float64)
    wts = np.ascontiguousarray(wts, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    B, H, nqb, C, d = cent.shape
    nkb = kbar.shape[2]
    assert kbar.shape == (B, H, nkb, d) and wts.shape == (B, H, nqb, C)
    out = np.zeros((B, H, nqb, nkb), dtype=np.float64)
    rc = lib().orc_score_u(_ptr(cent), _ptr(wts), _ptr(kbar), B, H, nqb, nkb, n_valid or nkb, C,
                           d, _ptr(out))
    if rc:
        raise ValueError(f"orc_score rc={rc}")
    return out


def ibcs_scores(q, k, N: int, C: int = 8, T: int = 5, unit: int = BLOCK) -> np.ndarray:
    """End-to-end oracle IBCS: mean keys per key unit, k-means of the 128-query
    blocks, unit scores (units past the sequence end score 0)."""
    cent, wts, _, _, _ = kmeans(q, N, C, T)
    return score(cent, wts, mean_key(k, N, unit), n_valid=-(-N // unit))


def sip(scores, budget: int, seed: int, with_p: bool = True):
    """Returns (idx, cnt, w, p, bad_rows); scores fp32 [B,H,nqb,nkb]."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    B, H, nqb, nkb = s.shape
    idx = np.zeros((B, H, nqb, nkb), dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    w = np.zeros((B, H, nqb, nkb), dtype=np.float32)
    p = np.zeros((B, H, nqb, nkb), dtype=np.float64) if with_p else None
    bad = np.zeros((B, H, nqb), dtype=np.int32)
    rc = lib().orc_sip(_ptr(s), B, H, nqb, nkb, budget, ctypes.c_uint64(seed & (2**64 - 1)),
                       _ptr(idx), _ptr(cnt), _ptr(w), _ptr(p), _ptr(bad))
    if rc < 0:
        raise ValueError(f"orc_sip rc={rc}")
    return idx, cnt, w, p, bad


def topk(scores, budget: int):
    s = np.ascontiguousarray(scores, dtype=np.float32)
    B, H, nqb, nkb = s.shape
    idx = np.zeros((B, H, nqb, nkb), dtype=np.int32)
    cnt = np.zeros((B, H, nqb), dtype=np.int32)
    w = np.zeros((B, H, nqb, nkb), dtype=np.float32)
    rc = lib().orc_topk(_ptr(s), B, H, nqb, nkb, budget, _ptr(idx), _ptr(cnt), _ptr(w))
    if rc < 0:
        raise ValueError(f"orc_topk rc={rc}")
    return idx, cnt, w


def attn_rows(q, k, v, N: int, idx, cnt, w=None, rows=None, want_num_den: bool = False,
              unit: int = BLOCK):
    """Sparse HT attention over key units of `unit` tokens for the listed (b,h,qb)
    query blocks (flat indices; None = all); idx / w rows have N_pad / unit entries.
    Returns (out [n,128,d], lse [n,128], num, den) in fp64."""
    qb_, kb_, vb_ = _bits(q), _bits(k), _bits(v)
    B, H, N_pad, d = qb_.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    wv = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
    nqb = N_pad // BLOCK
    if rows is None:
        n = B * H * nqb
        rows_a = None
    else:
        rows_a = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_a.shape[0]
    out = np.zeros((n, BLOCK, d), dtype=np.float64)
    lse = np.zeros((n, BLOCK), dtype=np.float64)
    num = np.zeros((n, BLOCK, d), dtype=np.float64) if want_num_den else None
    den = np.zeros((n, BLOCK), dtype=np.float64) if want_num_den else None
    rc = lib().orc_attn_rows_u(_ptr(qb_), _ptr(kb_), _ptr(vb_), B, H, N, N_pad, d, unit,
                               _ptr(idx), _ptr(cnt), _ptr(wv), n, _ptr(rows_a), _ptr(out),
                               _ptr(lse), _ptr(num), _ptr(den))
    if rc:
        raise ValueError(f"orc_attn_rows rc={rc}")
    return out, lse, num, den


def attn_bwd(q, k, v, do, N: int, idx, cnt, w=None):
    """Gradients (dQ, dK, dV), fp64 [B,H,N_pad,d], of the block-sparse HT attention over
    key blocks for the upstream gradient `do` (bf16) of its output; w None = top-k."""
    qb_, kb_, vb_, gb_ = _bits(q), _bits(k), _bits(v), _bits(do)
    B, H, N_pad, d = qb_.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    wv = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
    dq = np.zeros((B, H, N_pad, d), dtype=np.float64)
    dk = np.zeros_like(dq)
    dv = np.zeros_like(dq)
    rc = lib().orc_attn_bwd(_ptr(qb_), _ptr(kb_), _ptr(vb_), _ptr(gb_), B, H, N, N_pad, d,
                            _ptr(idx), _ptr(cnt), _ptr(wv), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError(f"orc_attn_bwd rc={rc}")
    return dq, dk, dv


def dense_attn(q, k, v, N: int):
    qb_, kb_, vb_ = _bits(q), _bits(k), _bits(v)
    B, H, N_pad, d = qb_.shape
    out = np.zeros((B, H, N_pad, d), dtype=np.float64)
    lse = np.zeros((B, H, N_pad), dtype=np.float64)
    rc = lib().orc_dense_attn(_ptr(qb_), _ptr(kb_), _ptr(vb_), B, H, N, N_pad, d, _ptr(out),
                              _ptr(lse))
    if rc:
        raise ValueError(f"orc_dense_attn rc={rc}")
    return out, lse
