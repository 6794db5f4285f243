"""Thin ctypes binding over libmisa_b200.so (argument marshalling only).

Every function here has the name of the C entry point it calls (include/misa.h),
takes torch CUDA tensors, allocates the outputs and the workspace through torch,
and passes raw device pointers plus torch's current CUDA stream.  All computation
happens in the library's kernels; there is no CPU path.  A missing library raises
at import time.
"""

from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmisa_b200.so")
INCLUDE_DIR = os.path.join(os.path.dirname(_PKG), "include")
HEADER_PATH = os.path.join(INCLUDE_DIR, "misa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python long_context_block_b200/build.py` "
        "(or __graft_entry__.build()); this package has no fallback path")

_lib = ctypes.CDLL(LIB_PATH)

_c_int, _c_i64, _c_sz, _p = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p

_SIGS = {
    "misa_workspace_size": (_c_sz, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int,
                                    _c_int, _c_int, _c_int]),
    "misa_pool_keys": (_c_int, [_p, _c_int, _c_i64, _c_int, _c_int, _p, _p]),
    "misa_pool_keys_range": (_c_int, [_p, _c_int, _c_i64, _c_int, _c_int, _c_i64, _c_i64, _p,
                                      _p]),
    "misa_route_heads": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_i64,
                                  _c_int, _c_int, _p, _p, _p, _c_sz, _p]),
    "misa_score_topk": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_i64,
                                 _c_int, _c_int, _p, _p, _p, _p, _c_sz, _p]),
    "dsa_score_topk": (_c_int, [_p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int,
                                _p, _p, _p, _p, _c_sz, _p]),
    "misa_dagger_rerank": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_i64,
                                    _c_int, _c_int, _p, _p, _p, _c_sz, _p]),
    "misa_score_rows": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int, _c_i64,
                                 _c_int, _p, _p, _c_sz, _p]),
    "misa_score_topk_noalloc": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int,
                                         _c_i64, _c_int, _c_int, _p, _p, _p, _p]),
    "hisa_block_filter_topk": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int, _c_int,
                                        _c_i64, _c_int, _c_int, _c_int, _p, _p, _p, _p, _c_sz,
                                        _p]),
    "misa_testing_score_simt": (_c_int, [_p, _p, _p, _p, _p, _p, _p, _c_int, _c_int, _c_int,
                                         _c_int, _c_i64, _c_int, _c_i64, _p, _p, _c_sz, _p]),
    "misa_testing_score_rows_wait_expiry": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int,
                                                     _c_int, _c_i64, _c_int, _p, _p, _c_sz,
                                                     ctypes.c_longlong, _c_int, _p]),
    "misa_testing_score_rows_timed": (_c_int, [_p, _p, _p, _p, _p, _c_int, _c_int, _c_int,
                                               _c_int, _c_i64, _c_int, _p, _p, _c_sz,
                                               ctypes.POINTER(ctypes.c_float), _p]),
    "misa_status_string": (ctypes.c_char_p, [_c_int]),
    "misa_check_device_status": (_c_int, [_p, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args

OP_ROUTE_HEADS, OP_SCORE_TOPK, OP_DSA_TOPK, OP_DAGGER_RERANK, OP_SCORE_ROWS = 1, 2, 3, 4, 5
OP_HISA_TOPK = 6
HEAD_DIM = 128


class MisaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: status {status} ({_lib.misa_status_string(status).decode()})")


def declared_symbols() -> list[str]:
    """Function names declared in the headers under include/ (misa.h and misa_testing.h)."""
    names = set()
    for f in sorted(os.listdir(INCLUDE_DIR)):
        if not f.endswith(".h"):
            continue
        text = open(os.path.join(INCLUDE_DIR, f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text))
    return sorted(names - {"if", "sizeof", "defined"})


def library() -> ctypes.CDLL:
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise MisaError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bits(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"{name} must be bf16 (or its int16 bit pattern), got {t.dtype}")
    return _dev(t, name)


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class _Workspace:
    """One zero-initialised scratch buffer per device, grown on demand.

    Every call on a device uses this buffer, so (as the C ABI requires of one workspace)
    calls issued on different streams must not overlap on the GPU: synchronise the streams
    between them, or call the C entry points with a workspace per stream."""

    def __init__(self):
        self._buf = {}
        self._lock = threading.Lock()

    def get(self, nbytes: int, device) -> torch.Tensor:
        dev = torch.device(device)
        with self._lock:
            b = self._buf.get(dev.index)
            if b is None or b.numel() < nbytes:
                b = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
                self._buf[dev.index] = b
            return b


_WS = _Workspace()


def workspace(nbytes: int, device) -> torch.Tensor:
    return _WS.get(nbytes, device)


def misa_workspace_size(op, nseq, T, H, d, L, B, h, topk, kprime) -> int:
    return int(_lib.misa_workspace_size(op, nseq, T, H, d, L, B, h, topk, kprime))


def misa_check_device_status(device=None) -> int:
    """Synchronise, read and clear the workspace status word; raise if it is set."""
    dev = torch.device(device if device is not None else torch.cuda.current_device())
    ws = _WS.get(256, dev)
    st = int(_lib.misa_check_device_status(_ptr(ws), _stream()))
    _check("misa_check_device_status", st)
    return st


def misa_pool_keys(k: torch.Tensor, B: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """Mean-pool k [nseq, L, d] (bf16) into fp32 [nseq, ceil(L/B), d] (Eq. 4)."""
    k = _bits(k, "k")
    nseq, L, d = k.shape
    M = -(-L // B)
    if out is None:
        out = torch.empty((nseq, M, d), dtype=torch.float32, device=k.device)
    _check("misa_pool_keys",
           _lib.misa_pool_keys(_ptr(k), nseq, L, d, B, _ptr(out), _stream()))
    return out


def misa_pool_keys_range(k: torch.Tensor, B: int, k_pool: torch.Tensor, s_begin: int,
                         s_end: int) -> torch.Tensor:
    """Recompute, in place, the pooled blocks of k_pool that meet tokens [s_begin, s_end)
    of every sequence (the keys there changed); other blocks are left as they are."""
    k = _bits(k, "k")
    nseq, L, d = k.shape
    k_pool = _dev(k_pool, "k_pool", torch.float32)
    if tuple(k_pool.shape) != (nseq, -(-L // B), d):
        raise ValueError(f"k_pool must be [{nseq}, {-(-L // B)}, {d}], got {tuple(k_pool.shape)}")
    _check("misa_pool_keys_range",
           _lib.misa_pool_keys_range(_ptr(k), nseq, L, d, B, int(s_begin), int(s_end),
                                     _ptr(k_pool), _stream()))
    return k_pool


def misa_route_heads(q, w, k, k_pool, pos, B: int, h: int, return_E: bool = False,
                     heads: torch.Tensor | None = None, E: torch.Tensor | None = None):
    """Route each query to its top-h heads by block-pooled energy (Eqs. 7-8)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    k_pool = _dev(k_pool, "k_pool", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    if heads is None:
        heads = torch.empty((nseq, T, h), dtype=torch.int32, device=q.device)
    if return_E and E is None:
        E = torch.empty((nseq, T, H), dtype=torch.float32, device=q.device)
    nb = misa_workspace_size(OP_ROUTE_HEADS, nseq, T, H, d, L, B, h, 1, 1)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("misa_route_heads",
           _lib.misa_route_heads(_ptr(q), _ptr(w), _ptr(k), _ptr(k_pool), _ptr(pos), nseq, T, H,
                                 d, L, B, h, _ptr(heads), _ptr(E), _ptr(ws), ws.numel(),
                                 _stream()))
    return (heads, E) if return_E else heads


def _outs(rows_shape, topk, device, idx, vals, want_vals):
    if idx is None:
        idx = torch.empty(rows_shape + (topk,), dtype=torch.int32, device=device)
    if want_vals and vals is None:
        vals = torch.empty(rows_shape + (topk,), dtype=torch.float32, device=device)
    return idx, vals


def misa_score_topk(q, w, k, heads, pos, topk: int, return_vals: bool = True,
                    scores: torch.Tensor | None = None, idx=None, vals=None):
    """Routed scores over each query's prefix and their top-k (Eqs. 9-10)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    heads = _dev(heads, "heads", torch.int32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    h = heads.shape[-1]
    idx, vals = _outs((nseq, T), topk, q.device, idx, vals, return_vals)
    if scores is not None:
        _dev(scores, "scores", torch.float32)
    nb = misa_workspace_size(OP_SCORE_TOPK, nseq, T, H, d, L, 1, h, topk, topk)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("misa_score_topk",
           _lib.misa_score_topk(_ptr(q), _ptr(w), _ptr(k), _ptr(heads), _ptr(pos), nseq, T, H, d,
                                L, h, topk, _ptr(idx), _ptr(vals), _ptr(scores), _ptr(ws),
                                ws.numel(), _stream()))
    return (idx, vals) if return_vals else idx


def dsa_score_topk(q, w, k, pos, topk: int, return_vals: bool = True,
                   scores: torch.Tensor | None = None, idx=None, vals=None):
    """Dense DSA indexer scores (all heads, Eq. 1) and their top-k (Eq. 2)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    idx, vals = _outs((nseq, T), topk, q.device, idx, vals, return_vals)
    if scores is not None:
        _dev(scores, "scores", torch.float32)
    nb = misa_workspace_size(OP_DSA_TOPK, nseq, T, H, d, L, 1, 1, topk, topk)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("dsa_score_topk",
           _lib.dsa_score_topk(_ptr(q), _ptr(w), _ptr(k), _ptr(pos), nseq, T, H, d, L, topk,
                               _ptr(idx), _ptr(vals), _ptr(scores), _ptr(ws), ws.numel(),
                               _stream()))
    return (idx, vals) if return_vals else idx


def misa_score_rows(q, w, k, heads, pos, scores: torch.Tensor | None = None):
    """Token scores without selection: routed (Eq. 9) when heads is given, dense (Eq. 1)
    when heads is None.  Returns fp32 [nseq, T, L]; entries past each query's position
    are left as they were."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    if heads is not None:
        heads = _dev(heads, "heads", torch.int32)
    h = heads.shape[-1] if heads is not None else H
    if scores is None:
        scores = torch.empty((nseq, T, L), dtype=torch.float32, device=q.device)
    _dev(scores, "scores", torch.float32)
    nb = misa_workspace_size(OP_SCORE_ROWS, nseq, T, H, d, L, 1, h, 1, 1)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("misa_score_rows",
           _lib.misa_score_rows(_ptr(q), _ptr(w), _ptr(k), _ptr(heads), _ptr(pos), nseq, T, H, d,
                                L, h, _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return scores


def misa_dagger_rerank(q, w, k, pos, cand, topk: int, return_vals: bool = True, idx=None,
                       vals=None):
    """Re-score candidates with all heads and keep the top-k (Eq. 12)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    cand = _dev(cand, "cand", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    kprime = cand.shape[-1]
    idx, vals = _outs((nseq, T), topk, q.device, idx, vals, return_vals)
    nb = misa_workspace_size(OP_DAGGER_RERANK, nseq, T, H, d, L, 1, 1, topk, kprime)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("misa_dagger_rerank",
           _lib.misa_dagger_rerank(_ptr(q), _ptr(w), _ptr(k), _ptr(pos), _ptr(cand), nseq, T, H,
                                   d, L, kprime, topk, _ptr(idx), _ptr(vals), _ptr(ws),
                                   ws.numel(), _stream()))
    return (idx, vals) if return_vals else idx


def hisa_block_filter_topk(q, w, k, k_pool, pos, B: int, m: int, topk: int,
                           return_vals: bool = True, return_blocks: bool = False, idx=None,
                           vals=None, blocks=None):
    """HISA-style token-axis filter: keep each query's m blocks with the largest
    head-summed affinity G[b] = sum_j w_j ReLU(q_j . kp_b), then the top-k of the
    all-head score (Eq. 1) over their tokens.  k_pool: misa_pool_keys(k, B)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    k_pool = _dev(k_pool, "k_pool", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    idx, vals = _outs((nseq, T), topk, q.device, idx, vals, return_vals)
    if return_blocks and blocks is None:
        blocks = torch.empty((nseq, T, m), dtype=torch.int32, device=q.device)
    nb = misa_workspace_size(OP_HISA_TOPK, nseq, T, H, d, L, B, m, topk, 0)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("hisa_block_filter_topk",
           _lib.hisa_block_filter_topk(_ptr(q), _ptr(w), _ptr(k), _ptr(k_pool), _ptr(pos), nseq,
                                       T, H, d, L, B, m, topk, _ptr(idx), _ptr(vals),
                                       _ptr(blocks), _ptr(ws), ws.numel(), _stream()))
    out = (idx, vals) if return_vals else (idx,)
    if return_blocks:
        out = out + (blocks,)
    return out if len(out) > 1 else out[0]


def misa_score_topk_noalloc(q, w, k, heads, pos, topk: int, return_vals: bool = True, idx=None,
                            vals=None, device_status=None):
    """misa_score_topk for callers that cannot allocate: the library uses its own fixed
    16 MiB scratch (nseq * T * L <= 4,194,304) instead of a workspace.  Outputs are
    allocated here only when not passed in; pass idx / vals / device_status to make
    the call allocation-free from Python too.  Calls whose GPU work overlaps race on
    the shared scratch and must be serialised."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    heads = _dev(heads, "heads", torch.int32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    h = heads.shape[-1]
    idx, vals = _outs((nseq, T), topk, q.device, idx, vals, return_vals)
    _check("misa_score_topk_noalloc",
           _lib.misa_score_topk_noalloc(_ptr(q), _ptr(w), _ptr(k), _ptr(heads), _ptr(pos), nseq,
                                        T, H, d, L, h, topk, _ptr(idx), _ptr(vals),
                                        _ptr(device_status), _stream()))
    return (idx, vals) if return_vals else idx


# ----------------------------------------------------------------- test-only entry points
# (include/misa_testing.h): the CUDA-core scorer on its own, and the tensor-core scorer
# with shortened wait bounds and one key tile never loaded.

def misa_testing_score_simt(q, w, k, heads, pos, gather_ids=None, gather_len=None,
                            scores: torch.Tensor | None = None):
    """The CUDA-core scorer: Eq. (9) under heads (Eq. 1 with heads None) over each
    query's prefix, or over gather_ids[row, :gather_len[row]] when given.  Returns fp32
    [nseq, T, L] (prefix) or [nseq, T, kprime] (gather)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    if heads is not None:
        heads = _dev(heads, "heads", torch.int32)
    h = heads.shape[-1] if heads is not None else H
    if gather_ids is not None:
        gather_ids = _dev(gather_ids, "gather_ids", torch.int32)
        gather_len = _dev(gather_len, "gather_len", torch.int32)
        stride = gather_ids.shape[-1]
    else:
        stride = L
    if scores is None:
        scores = torch.full((nseq, T, stride), float("nan"), dtype=torch.float32,
                            device=q.device)
    ws = _WS.get(256, q.device)
    _check("misa_testing_score_simt",
           _lib.misa_testing_score_simt(_ptr(q), _ptr(w), _ptr(k), _ptr(heads), _ptr(pos),
                                        _ptr(gather_ids), _ptr(gather_len), nseq, T, H, d, L, h,
                                        stride, _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return scores


def misa_testing_score_rows_wait_expiry(q, w, k, heads, pos, wait_cycles: int, skip_tile: int,
                                        scores: torch.Tensor | None = None):
    """misa_score_rows with every wait bounded by wait_cycles and key tile skip_tile never
    loaded (-1: none).  Read the outcome with misa_check_device_status."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    if heads is not None:
        heads = _dev(heads, "heads", torch.int32)
    h = heads.shape[-1] if heads is not None else H
    if scores is None:
        scores = torch.full((nseq, T, L), float("nan"), dtype=torch.float32, device=q.device)
    nb = misa_workspace_size(OP_SCORE_ROWS, nseq, T, H, d, L, 1, h, 1, 1)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    _check("misa_testing_score_rows_wait_expiry",
           _lib.misa_testing_score_rows_wait_expiry(_ptr(q), _ptr(w), _ptr(k), _ptr(heads),
                                                    _ptr(pos), nseq, T, H, d, L, h,
                                                    _ptr(scores), _ptr(ws), ws.numel(),
                                                    int(wait_cycles), int(skip_tile), _stream()))
    return scores


def misa_testing_score_rows_timed(q, w, k, heads, pos, scores: torch.Tensor | None = None):
    """misa_score_rows on the tensor-core scorer; returns the device milliseconds of its
    scoring kernel alone (CUDA events around that launch; the call waits for it)."""
    q, k = _bits(q, "q"), _bits(k, "k")
    w = _dev(w, "w", torch.float32)
    pos = _dev(pos, "pos", torch.int32)
    nseq, T, H, d = q.shape
    L = k.shape[1]
    if heads is not None:
        heads = _dev(heads, "heads", torch.int32)
    h = heads.shape[-1] if heads is not None else H
    if scores is None:
        scores = torch.empty((nseq, T, L), dtype=torch.float32, device=q.device)
    nb = misa_workspace_size(OP_SCORE_ROWS, nseq, T, H, d, L, 1, h, 1, 1)
    if nb == 0:
        raise MisaError("misa_workspace_size", 1)
    ws = _WS.get(nb, q.device)
    ms = ctypes.c_float(0.0)
    _check("misa_testing_score_rows_timed",
           _lib.misa_testing_score_rows_timed(_ptr(q), _ptr(w), _ptr(k), _ptr(heads), _ptr(pos),
                                              nseq, T, H, d, L, h, _ptr(scores), _ptr(ws),
                                              ws.numel(), ctypes.byref(ms), _stream()))
    return float(ms.value)
