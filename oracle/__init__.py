"""Plain fp64 CPU oracle for the DashAttention forward path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package.  The CUDA library never does: the two share no code.

The arithmetic lives in ``dash_oracle.c`` (fp64, OpenMP over rows); this module only
marshals numpy/torch arrays into it.  Every function widens its inputs to float64 (bf16
inputs widen exactly) and returns float64 numpy arrays.

Parity status per function (pins live in ``tests/test_oracle_pins.py``):
  stage0            pinned (mean pooling at head_cls = 0, SDPA special case, arg-max limit)
  entmax / stage1   pinned (sum to one, sort closed forms, brute-force supports, softmax limit)
  stage2            pinned (dense causal attention special case, variational optimum,
                    exact zero weight of masked chunks)
  decode            pinned (equals the prefill row at the same position)
  decode_route      pinned (equals decode's routing, which recomputes the summaries)
  backward          pinned (central finite differences of sum(O dO) for every input; dense
                    mode against torch autograd of SDPA in float64)
  topk              pinned (numpy's stable argsort on the negated scores; uniform prior)
  estimate_diagonal pinned (diagonal summary = single-query SDPA over the visible keys of the
                    diagonal chunk; at a chunk's last row it is Stage 0's summary; routing =
                    entmax of the scores written out independently)
  diagonal branch, GQA score averaging, bias = sigma * log p: parity unpinned by the pages
  (they rest on stated readings; the tests pin the library to those readings).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dash_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dbl_p = ctypes.POINTER(ctypes.c_double)
_i64_p = ctypes.POINTER(ctypes.c_int64)
_L = ctypes.c_long


def build(force: bool = False) -> str:
    """Compile dash_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_stage0.argtypes = [_dbl_p, _dbl_p, _L, _L, _L, _L, _L, _dbl_p]
        lib.oracle_stage0.restype = None
        for name in ("oracle_entmax", "oracle_entmax_bisect"):
            getattr(lib, name).argtypes = (
                [_dbl_p, _L, ctypes.c_double, _dbl_p] if name == "oracle_entmax"
                else [_dbl_p, _L, ctypes.c_double, _dbl_p])
            getattr(lib, name).restype = ctypes.c_double
        for name in ("oracle_sparsemax_sort", "oracle_entmax15_sort", "oracle_softmax"):
            getattr(lib, name).argtypes = [_dbl_p, _L, _dbl_p]
            getattr(lib, name).restype = ctypes.c_double
        lib.oracle_stage1.argtypes = [_dbl_p, _dbl_p, _L, _L, _L, _L, _L, _L, ctypes.c_double,
                                      ctypes.c_double, _i64_p, _L, _dbl_p, _dbl_p, _dbl_p]
        lib.oracle_stage1.restype = None
        lib.oracle_stage1_diag.argtypes = [_dbl_p, _dbl_p, _dbl_p, _dbl_p, _L, _L, _L, _L, _L, _L,
                                           ctypes.c_double, ctypes.c_double, _L, _i64_p, _L,
                                           _dbl_p, _dbl_p, _dbl_p]
        lib.oracle_topk.argtypes = [_dbl_p, _L, _L, _dbl_p]
        lib.oracle_topk.restype = ctypes.c_double
        lib.oracle_stage1_diag.restype = None
        lib.oracle_stage2.argtypes = [_dbl_p, _dbl_p, _dbl_p, _dbl_p, _L, _L, _L, _L, _L, _L,
                                      ctypes.c_double, ctypes.c_int, _i64_p, _L, _dbl_p]
        lib.oracle_stage2.restype = None
        lib.oracle_decode.argtypes = [_dbl_p, _dbl_p, _dbl_p, _dbl_p, _i64_p, _L, _L, _L, _L,
                                      _L, _L, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int, _L, _dbl_p, _dbl_p,
                                      _dbl_p, _dbl_p]
        lib.oracle_decode.restype = None
        lib.oracle_decode_route.argtypes = [_dbl_p, _dbl_p, _dbl_p, _dbl_p, _i64_p, _L, _L, _L,
                                            _L, _L, _L, _L, ctypes.c_double, ctypes.c_double, _L,
                                            _dbl_p, _dbl_p, _dbl_p]
        lib.oracle_decode_route.restype = None
        lib.oracle_backward.argtypes = [_dbl_p] * 5 + [_L] * 6 + [ctypes.c_double] * 3 + [_dbl_p] * 4
        lib.oracle_backward.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Widen a torch tensor or array-like to a C-contiguous float64 numpy array."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dbl_p)


def num_threads() -> int:
    return int(_get().oracle_num_threads())


# --------------------------------------------------------------------------- stage 0
def stage0(K, head_cls, chunk_size: int) -> np.ndarray:
    """Chunk summaries [B,Hkv,T//Bc,D] of every complete chunk (gist.science summary,
    "Stufe 0: Lokale Chunk-Zusammenfassung")."""
    K = _f64(K)
    hc = _f64(head_cls)
    B, Hkv, T, D = K.shape
    out = np.zeros((B, Hkv, T // chunk_size, D))
    _get().oracle_stage0(_ptr(K), _ptr(hc), B, Hkv, T, D, chunk_size, _ptr(out))
    return out


# --------------------------------------------------------------------------- entmax
def entmax(s, alpha: float, method: str = "auto"):
    """alpha-entmax of one score vector s: returns (p, tau).

    method: "auto" (exact sort algorithm for alpha in {1.5, 2}, softmax for 1, bisection
    otherwise), "bisect", "sort15", "sparsemax", "softmax"."""
    s = _f64(s).ravel()
    n = s.size
    p = np.zeros(n)
    lib = _get()
    if method == "auto":
        tau = lib.oracle_entmax(_ptr(s), n, float(alpha), _ptr(p))
    elif method == "bisect":
        tau = lib.oracle_entmax_bisect(_ptr(s), n, float(alpha), _ptr(p))
    elif method == "sort15":
        tau = lib.oracle_entmax15_sort(_ptr(s), n, _ptr(p))
    elif method == "sparsemax":
        tau = lib.oracle_sparsemax_sort(_ptr(s), n, _ptr(p))
    elif method == "softmax":
        tau = lib.oracle_softmax(_ptr(s), n, _ptr(p))
    else:
        raise ValueError(method)
    return p, float(tau)


def topk(s, k: int):
    """Top-k routing of one score vector: (p, theta) with p uniform (1/min(k, n)) on the k
    highest scores (ties: lower index first) and theta the k-th highest score."""
    s = _f64(s).ravel()
    p = np.zeros(s.size)
    theta = _get().oracle_topk(_ptr(s), s.size, int(k), _ptr(p))
    return p, float(theta)


# --------------------------------------------------------------------------- stage 1
def stage1(Q, summary, seq_len: int, chunk_size: int, alpha: float, gamma: float = 1.0,
           rows=None, estimate_diagonal: bool = False, K=None, head_cls=None, topk: int = 0):
    """Routing of the given rows (default: all).  Returns (p, m, tau):
    p, m [B,Hkv,nrows,C] (m = margin (alpha-1)s - tau on routable chunks, NaN elsewhere),
    tau [B,Hkv,nrows].  (gist.science summary, "Stufe 1: Entmax-Chunk-Routing").
    estimate_diagonal (needs K and head_cls): the diagonal chunk takes part in the entmax
    normalisation with its summary estimated from the keys the row can see (p[.., c_t] is
    then its probability; aiexpert.news interface paragraph).  topk > 0: top-k routing
    (p uniform over the k highest scores, m = s - theta) instead of alpha-entmax."""
    Q = _f64(Q)
    S = _f64(summary)
    B, Hq, T, D = Q.shape
    assert T == seq_len
    Hkv = S.shape[1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(
        np.asarray(rows, dtype=np.int64))
    C = (T + chunk_size - 1) // chunk_size
    nr = rows.size
    p = np.zeros((B, Hkv, nr, C))
    m = np.zeros((B, Hkv, nr, C))
    tau = np.zeros((B, Hkv, nr))
    if estimate_diagonal or topk:
        Kd = hc = None
        if estimate_diagonal:
            Kd, hc = _f64(K), _f64(head_cls)
            assert Kd.shape == (B, Hkv, T, D) and hc.shape == (Hkv, D)
        _get().oracle_stage1_diag(_ptr(Q), _ptr(S), _ptr(Kd) if Kd is not None else None,
                                  _ptr(hc) if hc is not None else None, B, Hq, Hkv, T, D,
                                  chunk_size, float(alpha), float(gamma), int(topk),
                                  rows.ctypes.data_as(_i64_p), nr, _ptr(p), _ptr(m), _ptr(tau))
    else:
        _get().oracle_stage1(_ptr(Q), _ptr(S), B, Hq, Hkv, T, D, chunk_size, float(alpha),
                             float(gamma), rows.ctypes.data_as(_i64_p), nr, _ptr(p), _ptr(m),
                             _ptr(tau))
    return p, m, tau


# --------------------------------------------------------------------------- stage 2
def stage2(Q, K, V, p, chunk_size: int, sigma: float = 1.0, rows=None, dense: bool = False):
    """Prior-induced block-sparse softmax attention for the given rows: O [B,Hq,nrows,D].
    p is [B,Hkv,nrows,C] (ignored when dense).  (gist.science summary, "Stufe 2:
    Prior-induzierte spaerliche Softmax")."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, Hq, T, D = Q.shape
    Hkv = K.shape[1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(
        np.asarray(rows, dtype=np.int64))
    nr = rows.size
    out = np.zeros((B, Hq, nr, D))
    if dense:
        pp = None
    else:
        pp = _f64(p)
        assert pp.shape[:3] == (B, Hkv, nr)
    _get().oracle_stage2(_ptr(Q), _ptr(K), _ptr(V), _ptr(pp) if pp is not None else None,
                         B, Hq, Hkv, T, D, chunk_size, float(sigma), int(dense),
                         rows.ctypes.data_as(_i64_p), nr, _ptr(out))
    return out


def prefill(Q, K, V, head_cls, chunk_size: int, alpha: float, gamma: float = 1.0,
            sigma: float = 1.0, rows=None, dense: bool = False,
            estimate_diagonal: bool = False, topk: int = 0):
    """Whole forward pass for the given rows: dict(O, p, m, tau, summary).  With topk > 0 the
    routing is top-k and Stage 2 attends the selection with a uniform prior (sigma = 0)."""
    T = _f64(Q).shape[2] if not hasattr(Q, "shape") else Q.shape[2]
    summary = stage0(K, head_cls, chunk_size)
    p, m, tau = stage1(Q, summary, T, chunk_size, alpha, gamma, rows,
                       estimate_diagonal=estimate_diagonal, K=K, head_cls=head_cls, topk=topk)
    O = stage2(Q, K, V, p, chunk_size, 0.0 if topk else sigma, rows, dense)
    return dict(O=O, p=p, m=m, tau=tau, summary=summary)


# --------------------------------------------------------------------------- decode
def decode(q, K_cache, V_cache, head_cls, seq_lens, chunk_size: int, alpha: float,
           gamma: float = 1.0, sigma: float = 1.0, estimate_diagonal: bool = False,
           topk: int = 0):
    """One decode step: the row t = seq_lens[b]-1 of every sequence.  Returns dict(O
    [B,Hq,D], p, m [B,Hkv,Ccap], tau [B,Hkv])."""
    q, K, V, hc = _f64(q), _f64(K_cache), _f64(V_cache), _f64(head_cls)
    B, Hq, D = q.shape
    Hkv, cap = K.shape[1], K.shape[2]
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int64))
    Ccap = (cap + chunk_size - 1) // chunk_size
    O = np.zeros((B, Hq, D))
    p = np.zeros((B, Hkv, Ccap))
    m = np.zeros((B, Hkv, Ccap))
    tau = np.zeros((B, Hkv))
    _get().oracle_decode(_ptr(q), _ptr(K), _ptr(V), _ptr(hc), sl.ctypes.data_as(_i64_p), B, Hq,
                         Hkv, cap, D, chunk_size, float(alpha), float(gamma),
                         0.0 if topk else float(sigma), int(estimate_diagonal), int(topk),
                         _ptr(O), _ptr(p), _ptr(m), _ptr(tau))
    return dict(O=O, p=p, m=m, tau=tau)


def decode_route(q, summary, seq_lens, cap: int, chunk_size: int, alpha: float,
                 gamma: float = 1.0, estimate_diagonal: bool = False, K_cache=None,
                 head_cls=None, topk: int = 0):
    """Routing alone of one decode step from cached summaries [B,Hkv,Cs,D]: the row
    t = seq_lens[b]-1 of every sequence over its complete chunks (plus, with
    estimate_diagonal, its diagonal chunk estimated from K_cache [B,Hkv,cap,D]).  Returns
    dict(p, m [B,Hkv,Ccap] with Ccap = ceil(cap/Bc), tau [B,Hkv]) -- the same values as
    decode()."""
    q, S = _f64(q), _f64(summary)
    B, Hq, D = q.shape
    Hkv, Cs = S.shape[1], S.shape[2]
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int64))
    assert (sl >= 1).all() and ((sl - 1) // chunk_size <= Cs).all()
    Ccap = (cap + chunk_size - 1) // chunk_size
    p = np.zeros((B, Hkv, Ccap))
    m = np.zeros((B, Hkv, Ccap))
    tau = np.zeros((B, Hkv))
    Kd = hc = None
    if estimate_diagonal:
        Kd, hc = _f64(K_cache), _f64(head_cls)
        assert Kd.shape[:2] == (B, Hkv) and Kd.shape[2] == cap
    _get().oracle_decode_route(_ptr(q), _ptr(S), _ptr(Kd) if Kd is not None else None,
                               _ptr(hc) if hc is not None else None,
                               sl.ctypes.data_as(_i64_p), B, Hq, Hkv, Cs, cap, D, chunk_size,
                               float(alpha), float(gamma), int(topk), _ptr(p), _ptr(m), _ptr(tau))
    return dict(p=p, m=m, tau=tau)


# --------------------------------------------------------------------------- backward
def backward(Q, K, V, head_cls, dO, chunk_size: int, alpha: float, gamma: float = 1.0,
             sigma: float = 1.0):
    """Gradients of sum(O * dO) w.r.t. Q, K, V, head_cls through Stages 2, 1 and 0 (default
    routing mode).  Returns dict(dQ [B,Hq,T,D], dK, dV [B,Hkv,T,D], dhc [Hkv,D]).
    (gist.science summary, "Stufe 1": gradients flow through the routing back to Stage 0.)"""
    Q, K, V, hc, dO = (_f64(x) for x in (Q, K, V, head_cls, dO))
    B, Hq, T, D = Q.shape
    Hkv = K.shape[1]
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dhc = np.zeros_like(hc)
    _get().oracle_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(hc), _ptr(dO), B, Hq, Hkv, T, D,
                           chunk_size, float(alpha), float(gamma), float(sigma), _ptr(dQ),
                           _ptr(dK), _ptr(dV), _ptr(dhc))
    return dict(dQ=dQ, dK=dK, dV=dV, dhc=dhc)
