"""AB-Attention block-sparse attention on NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/ab_attn.h`` (``libab_attn.so``, built
in-tree by ``build.py``). Every function here only checks and marshals arguments:
all work runs in the library's CUDA kernels on the current torch stream. There is no
fallback: if the library is missing or no CUDA device is present, calls raise.

Steps (AB-Attention news page, section «Три приёма AB-Attention»):
  score()          IBCS block scores from per-block k-means centroids and mean keys
  select()         SIP sampling with inclusion-probability weights, or top-k
  attn_fwd()       block-sparse attention with Horvitz-Thompson weights (logit shift)
  attn_topk_fwd()  the same with all weights 1 (top-k baseline)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import synth  # noqa: F401  (seeded input generators)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libab_attn.so")
BLOCK = 128
MAX_BLOCKS = 8192  # AB_MAX_BLOCKS: key blocks per head
MAX_UNITS = 65536  # AB_MAX_UNITS: 4-token key units per head, and entries per selection row

AB_F32 = 0
AB_BF16 = 1
MODE_SIP = 0
MODE_TOPK = 1
FLAG_BAD_SCORE = 1
FLAG_BAD_INDEX = 2
FLAG_BAD_WEIGHT = 4
FLAG_TIMEOUT = 8
FLAG_SCHED_COLLISION = 16

STATUS = {
    0: "AB_OK", 1: "AB_ERR_NULL", 2: "AB_ERR_SHAPE", 3: "AB_ERR_DTYPE",
    4: "AB_ERR_UNSUPPORTED", 5: "AB_ERR_RANGE", 6: "AB_ERR_CUDA", 7: "AB_ERR_DEVICE_FLAG",
    8: "AB_ERR_TIMEOUT", 9: "AB_ERR_ALIGN", 10: "AB_ERR_WORKSPACE",
}


class AbError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS.get(code, code)}"
        if code == 6 and _lib is not None:
            msg += f" ({_lib.ab_last_cuda_error().decode()})"
        super().__init__(msg)


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("N_pad", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32)]


_lib = None


def lib():
    """Load libab_attn.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m block_sparse_attention_ab_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, Shape
        L.ab_score_workspace_size.argtypes = [S, I, ctypes.POINTER(ctypes.c_size_t)]
        L.ab_score.argtypes = [P, P, S, I, I, P, P, P, P, P, P, ctypes.c_size_t, P, P]
        L.ab_score_noalloc.argtypes = [P, P, S, I, I, P, P, P]
        L.ab_select.argtypes = [P, I, I, I, I, I, I, ctypes.c_uint64, P, P, P, P, P, P]
        L.ab_attn_fwd.argtypes = [P, P, P, S, P, P, P, P, I, P, P, P]
        L.ab_attn_topk_fwd.argtypes = [P, P, P, S, P, P, P, I, P, P, P]
        L.ab_attn_bwd_workspace_size.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
        L.ab_attn_bwd.argtypes = [P, P, P, S, P, P, P, P, I, P, P, P, P, P, P, ctypes.c_size_t,
                                  P, P]
        L.ab_selftest_attn_bwd_wait_limit.argtypes = [P, P, P, S, P, P, P, P, I, P, P, P, P, P, P,
                                                      ctypes.c_size_t, P, I, P]
        L.ab_score_units_workspace_size.argtypes = [S, I, I, ctypes.POINTER(ctypes.c_size_t)]
        L.ab_score_units.argtypes = [P, P, S, I, I, I, P, P, P, P, P, P, ctypes.c_size_t, P, P]
        L.ab_attn_units_fwd.argtypes = [P, P, P, S, I, P, P, P, P, I, P, P, P]
        L.ab_attn_units_topk_fwd.argtypes = [P, P, P, S, I, P, P, P, I, P, P, P]
        L.ab_selftest_bounded_wait.argtypes = [I, I, P, P, P]
        L.ab_selftest_force_counter_slot.argtypes = [I]
        L.ab_selftest_attn_wait_limit.argtypes = [P, P, P, S, I, P, P, P, P, I, P, P, I, P]
        L.ab_forward_host_workspace_size.argtypes = [S, I, I, I, ctypes.POINTER(ctypes.c_size_t)]
        L.ab_forward_host.argtypes = [P, P, P, S, I, I, I, I, ctypes.c_uint64, P, I, I, P,
                                      ctypes.c_size_t, P, P]
        L.ab_check_flag.argtypes = [P, ctypes.POINTER(ctypes.c_int), P]
        L.ab_status_str.argtypes = [I]
        L.ab_status_str.restype = ctypes.c_char_p
        L.ab_version.argtypes = []
        L.ab_last_cuda_error.argtypes = []
        L.ab_last_cuda_error.restype = ctypes.c_char_p
        for name in ("ab_score_workspace_size", "ab_score", "ab_score_noalloc", "ab_select", "ab_attn_fwd",
                     "ab_attn_topk_fwd", "ab_check_flag", "ab_version", "ab_score_units_workspace_size",
                     "ab_score_units", "ab_attn_units_fwd", "ab_attn_units_topk_fwd",
                     "ab_selftest_bounded_wait", "ab_selftest_force_counter_slot",
                     "ab_selftest_attn_wait_limit", "ab_attn_bwd_workspace_size", "ab_attn_bwd",
                     "ab_selftest_attn_bwd_wait_limit"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise AbError(code, where)


def _need(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_shape(q: torch.Tensor, N: int) -> Shape:
    B, H, N_pad, d = q.shape
    return Shape(B, H, int(N), N_pad, d, AB_BF16)


def score_workspace_bytes(shape: Shape, n_clusters: int = 8, unit: int = BLOCK) -> int:
    n = ctypes.c_size_t(0)
    if unit == BLOCK:
        _check(lib().ab_score_workspace_size(shape, n_clusters, ctypes.byref(n)), "ab_score_workspace_size")
    else:
        _check(lib().ab_score_units_workspace_size(shape, n_clusters, unit, ctypes.byref(n)),
               "ab_score_units_workspace_size")
    return int(n.value)


def score(q: torch.Tensor, k: torch.Tensor, N: int, n_clusters: int = 8, iters: int = 5,
          intermediates: bool = False, workspace: Optional[torch.Tensor] = None,
          out: Optional[torch.Tensor] = None, unit: int = BLOCK):
    """IBCS scores [B,H,nqb,N_pad/unit] fp32 over key blocks (unit=128) or 4-token key
    units (unit=4). With intermediates=True also returns (kbar, centroids, cluster
    weights, assignment)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, H, N_pad, d = q.shape
    nb = N_pad // BLOCK
    nku = N_pad // unit
    shape = make_shape(q, N)
    dev = q.device
    scores = out if out is not None else torch.empty(B, H, nb, nku, device=dev, dtype=torch.float32)
    kbar = cent = cw = assign = None
    if intermediates:
        kbar = torch.empty(B, H, nku, d, device=dev, dtype=torch.float32)
        cent = torch.empty(B, H, nb, n_clusters, d, device=dev, dtype=torch.float32)
        cw = torch.empty(B, H, nb, n_clusters, device=dev, dtype=torch.float32)
        assign = torch.empty(B, H, N_pad, device=dev, dtype=torch.uint8)
    if workspace is None:
        workspace = torch.empty(score_workspace_bytes(shape, n_clusters, unit), device=dev,
                                dtype=torch.uint8)
    if unit == BLOCK:
        _check(lib().ab_score(_ptr(q), _ptr(k), shape, n_clusters, iters, _ptr(scores), _ptr(kbar),
                              _ptr(cent), _ptr(cw), _ptr(assign), _ptr(workspace),
                              workspace.numel(), None, _stream()), "ab_score")
    else:
        _check(lib().ab_score_units(_ptr(q), _ptr(k), shape, n_clusters, iters, unit, _ptr(scores),
                                    _ptr(kbar), _ptr(cent), _ptr(cw), _ptr(assign),
                                    _ptr(workspace), workspace.numel(), None, _stream()),
               "ab_score_units")
    if intermediates:
        return scores, kbar, cent, cw, assign
    return scores


def score_noalloc(q: torch.Tensor, k: torch.Tensor, N: int, n_clusters: int = 8, iters: int = 5,
                  out: Optional[torch.Tensor] = None):
    """IBCS block scores through ab_score_noalloc: no workspace argument; the library's
    fixed device scratch is used (see include/ab_attn.h for its size limit)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, H, N_pad, d = q.shape
    nb = N_pad // BLOCK
    scores = out if out is not None else torch.empty(B, H, nb, nb, device=q.device, dtype=torch.float32)
    _check(lib().ab_score_noalloc(_ptr(q), _ptr(k), make_shape(q, N), n_clusters, iters,
                                  _ptr(scores), None, _stream()), "ab_score_noalloc")
    return scores


def select(scores: torch.Tensor, budget: int, mode: str = "sip", seed: int = 0,
           want_p: bool = False, dev_flag: Optional[torch.Tensor] = None, out=None):
    """Returns (idx int32, cnt int32, w fp32[, p fp64]) for SIP or top-k."""
    _need(scores, torch.float32, "scores")
    B, H, nqb, nkb = scores.shape
    dev = scores.device
    if out is not None:
        idx, cnt, w = out[:3]
    else:
        idx = torch.empty(B, H, nqb, nkb, device=dev, dtype=torch.int32)
        cnt = torch.empty(B, H, nqb, device=dev, dtype=torch.int32)
        w = torch.empty(B, H, nqb, nkb, device=dev, dtype=torch.float32)
    p = torch.empty(B, H, nqb, nkb, device=dev, dtype=torch.float64) if want_p else None
    m = {"sip": MODE_SIP, "topk": MODE_TOPK}[mode]
    _check(lib().ab_select(_ptr(scores), B, H, nqb, nkb, int(budget), m,
                           ctypes.c_uint64(int(seed) & (2**64 - 1)), _ptr(idx), _ptr(cnt), _ptr(w),
                           _ptr(p), _ptr(dev_flag), _stream()), "ab_select")
    return (idx, cnt, w, p) if want_p else (idx, cnt, w)


def _out_buffer(q, out, out_dtype):
    if out is not None:
        _need(out, out_dtype, "out")
        return out
    return torch.empty(q.shape, device=q.device, dtype=out_dtype)


def _out_code(out_dtype):
    return {torch.bfloat16: AB_BF16, torch.float32: AB_F32}[out_dtype]


def attn_fwd(q, k, v, N: int, idx, cnt, w, want_lse: bool = False,
             dev_flag: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
             out_dtype=torch.bfloat16, unit: int = BLOCK):
    """Sparse HT-weighted attention over the kept key blocks (unit=128) or 4-token key
    units (unit=4); returns out (bf16 or fp32) [and lse fp32]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(idx, torch.int32, "idx")
    _need(cnt, torch.int32, "cnt")
    _need(w, torch.float32, "w")
    o = _out_buffer(q, out, out_dtype)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32) if want_lse else None
    if unit == BLOCK:
        _check(lib().ab_attn_fwd(_ptr(q), _ptr(k), _ptr(v), make_shape(q, N), _ptr(idx), _ptr(cnt),
                                 _ptr(w), _ptr(o), _out_code(out_dtype), _ptr(lse), _ptr(dev_flag),
                                 _stream()), "ab_attn_fwd")
    else:
        _check(lib().ab_attn_units_fwd(_ptr(q), _ptr(k), _ptr(v), make_shape(q, N), unit, _ptr(idx),
                                       _ptr(cnt), _ptr(w), _ptr(o), _out_code(out_dtype), _ptr(lse),
                                       _ptr(dev_flag), _stream()), "ab_attn_units_fwd")
    return (o, lse) if want_lse else o


def attn_topk_fwd(q, k, v, N: int, idx, cnt, want_lse: bool = False,
                  dev_flag: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  out_dtype=torch.bfloat16, unit: int = BLOCK):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(idx, torch.int32, "idx")
    _need(cnt, torch.int32, "cnt")
    o = _out_buffer(q, out, out_dtype)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32) if want_lse else None
    if unit == BLOCK:
        _check(lib().ab_attn_topk_fwd(_ptr(q), _ptr(k), _ptr(v), make_shape(q, N), _ptr(idx),
                                      _ptr(cnt), _ptr(o), _out_code(out_dtype), _ptr(lse),
                                      _ptr(dev_flag), _stream()), "ab_attn_topk_fwd")
    else:
        _check(lib().ab_attn_units_topk_fwd(_ptr(q), _ptr(k), _ptr(v), make_shape(q, N), unit,
                                            _ptr(idx), _ptr(cnt), _ptr(o), _out_code(out_dtype),
                                            _ptr(lse), _ptr(dev_flag), _stream()),
               "ab_attn_units_topk_fwd")
    return (o, lse) if want_lse else o


def attn_bwd_workspace_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ab_attn_bwd_workspace_size(shape, ctypes.byref(n)), "ab_attn_bwd_workspace_size")
    return n.value


def attn_bwd(q, k, v, N: int, idx, cnt, w, out, lse, dout,
             dev_flag: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
             wait_limit_ns: Optional[int] = None):
    """Gradients (dq, dk, dv), fp32 [B,H,N_pad,d], of attn_fwd (w given) or attn_topk_fwd
    (w None) over key blocks, for the upstream gradient `dout` (bf16) of the output
    `out` (bf16 or fp32) whose lse the forward returned. wait_limit_ns (tests only) runs
    ab_selftest_attn_bwd_wait_limit instead, with the kernels' waits limited to it."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, torch.bfloat16, n)
    _need(idx, torch.int32, "idx")
    _need(cnt, torch.int32, "cnt")
    if w is not None:
        _need(w, torch.float32, "w")
    if not isinstance(out, torch.Tensor) or out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be the forward's bf16 or fp32 output")
    _need(out, out.dtype, "out")
    _need(lse, torch.float32, "lse")
    shape = make_shape(q, N)
    need = attn_bwd_workspace_bytes(shape)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.empty(q.shape, device=q.device, dtype=torch.float32) for _ in range(3))
    args = (_ptr(q), _ptr(k), _ptr(v), shape, _ptr(idx), _ptr(cnt), _ptr(w), _ptr(out),
            _out_code(out.dtype), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(workspace), workspace.numel(), _ptr(dev_flag))
    if wait_limit_ns is None:
        _check(lib().ab_attn_bwd(*args, _stream()), "ab_attn_bwd")
    else:
        _check(lib().ab_selftest_attn_bwd_wait_limit(*args, int(wait_limit_ns), _stream()),
               "ab_selftest_attn_bwd_wait_limit")
    return dq, dk, dv


def selftest_bounded_wait(limit_us: int, complete: bool, device="cuda"):
    """Run the bounded-wait self test (include/ab_attn.h); returns (flag bits, done) with
    done = 1 when the wait succeeded and 2 when it gave up."""
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    done = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib().ab_selftest_bounded_wait(int(limit_us), int(bool(complete)), _ptr(flag), _ptr(done),
                                          _stream()), "ab_selftest_bounded_wait")
    bits = check_flag(flag)
    return bits, int(done.item())


def check_flag(dev_flag: torch.Tensor) -> int:
    """Synchronise the current stream and return the device flag bits."""
    host = ctypes.c_int(0)
    code = lib().ab_check_flag(_ptr(dev_flag), ctypes.byref(host), _stream())
    if code not in (0, 7, 8):
        raise AbError(code, "ab_check_flag")
    return int(host.value)


def ab_attention(q, k, v, N: int, budget: int, mode: str = "sip", seed: int = 0,
                 n_clusters: int = 8, iters: int = 5, unit: int = BLOCK):
    """One pass of the whole path: score -> select -> sparse attention (device tensors).
    `budget` counts selection units (key blocks, or 4-token units when unit=4)."""
    s = score(q, k, N, n_clusters, iters, unit=unit)
    idx, cnt, w = select(s, budget, mode, seed)
    if mode == "sip":
        return attn_fwd(q, k, v, N, idx, cnt, w, unit=unit)
    return attn_topk_fwd(q, k, v, N, idx, cnt, unit=unit)


def forward_host_workspace_bytes(shape: Shape, n_clusters: int, chunk_heads: int,
                                 out_dtype=torch.bfloat16) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ab_forward_host_workspace_size(shape, n_clusters, int(chunk_heads), _out_code(out_dtype),
                                                ctypes.byref(n)), "ab_forward_host_workspace_size")
    return int(n.value)


def default_chunk_heads(shape, device="cuda") -> int:
    """Head pairs per ab_forward_host chunk: the fewest that give each chunk's attention
    launch about four waves of (b, h, query block) items on this GPU. Smaller chunks
    shorten the first copy-in and last copy-out that nothing overlaps."""
    B, H, N_pad = shape[:3]
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    nqb = N_pad // BLOCK
    return max(1, min(B * H, -(-4 * sms // nqb)))


def _need_host(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def forward_host(q, k, v, N: int, budget: int, mode: str = "sip", seed: int = 0,
                 n_clusters: int = 8, iters: int = 5, out: Optional[torch.Tensor] = None,
                 out_dtype=torch.bfloat16, chunk_heads: Optional[int] = None,
                 workspace: Optional[torch.Tensor] = None, dev_flag: Optional[torch.Tensor] = None,
                 device="cuda"):
    """The whole path for host tensors q, k, v (bf16 [B,H,N_pad,d], pinned for overlap):
    chunks of head pairs are copied in, scored, selected and attended on the current CUDA
    stream while the next chunk copies in and the last one's O copies out (ab_forward_host).
    Returns the host output (pinned unless `out` is given); it is ready when the current
    stream is. q, k, v (and `out`) must stay alive and unmodified until then: the copies
    run asynchronously, and a freed pinned buffer may be handed out again at once."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_host(t, torch.bfloat16, n)
    B, H = q.shape[:2]
    ch = int(chunk_heads) if chunk_heads is not None else default_chunk_heads(q.shape, device)
    shape = make_shape(q, N)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype).pin_memory()
    else:
        _need_host(out, out_dtype, "out")
    need = forward_host_workspace_bytes(shape, n_clusters, ch, out_dtype)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    elif workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    m = {"sip": MODE_SIP, "topk": MODE_TOPK}[mode]
    _check(lib().ab_forward_host(_ptr(q), _ptr(k), _ptr(v), shape, int(n_clusters), int(iters), m,
                                 int(budget), ctypes.c_uint64(int(seed) & (2**64 - 1)), _ptr(out),
                                 _out_code(out_dtype), ch, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _ptr(dev_flag), _stream()),
           "ab_forward_host")
    return out
