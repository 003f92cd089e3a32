"""DashAttention forward path on B200: Python binding of libdash (the C ABI in include/dash.h).

This module only marshals torch tensors into pointers, sizes and the current CUDA stream;
every step of the computation runs in libdash's sm_100a kernels.  There is no fallback: if
libdash.so is missing, importing this package raises.

    import sparse_hierarchical_attention_stage0_b200 as dash
    out = dash.prefill(q, k, v, head_cls, chunk_size=64, alpha=1.5, enable_gqa=True)

The interface follows the pages' description of the reference one (aiexpert.news
"DashAttention alcanca 75% de esparsidade ...": q, k, v, a per-head head_cls vector,
chunk_size, estimate_diagonal, enable_gqa, optional active_blocks).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdash.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python sparse_hierarchical_attention_stage0_b200/build.py` (there is no fallback)")

LIB_DEBUG_PATH = os.path.join(_HERE, "libdash_debug.so")

DASH_OK = 0
STATUS_NAMES = {0: "DASH_OK", 1: "DASH_ERR_INVALID_ARGUMENT", 2: "DASH_ERR_UNSUPPORTED",
                3: "DASH_ERR_WORKSPACE_TOO_SMALL", 4: "DASH_ERR_CUDA",
                5: "DASH_ERR_DEVICE_TIMEOUT", 6: "DASH_ERR_RANGE_CLAMPED", 7: "DASH_ERR_BOUNDS"}
FLAG_DENSE = 1
FLAG_FORCE_ALL_ACTIVE = 2
FLAG_ESTIMATE_DIAGONAL = 4
FLAG_TEST_NEWTON_CAP = 8          # test hook: Newton solve capped at one iteration
FLAG_TEST_STALL_WAIT = 16         # test hook: Stage 0's bounded copy wait runs out
FLAG_FUSE_ROUTE = 32              # Stage 1 inside the Stage 2 kernel where it applies (off by default)

# Every symbol include/dash.h declares.
EXPORTS = ("dash_prefill_workspace_size", "dash_prefill", "dash_prefill_host", "dash_stage0", "dash_route",
           "dash_attend_workspace_size", "dash_attend", "dash_update_chunk_cache", "dash_decode_workspace_size",
           "dash_decode", "dash_read_device_status", "dash_status_string", "dash_prefill_static_ws",
           "dash_static_ws_read_status", "dash_attend_kernel_name", "dash_prefill_kernel_count", "dash_decode_paged",
           "dash_update_chunk_cache_paged", "dash_backward_workspace_size", "dash_backward",
           "dash_stage2_kernel_ran", "dash_decode_step_workspace_size", "dash_decode_step",
           "dash_decode_step_paged")


class Params(ctypes.Structure):
    """dash_params_t."""
    _fields_ = [("batch", ctypes.c_int), ("heads_q", ctypes.c_int), ("heads_kv", ctypes.c_int),
                ("seq_len", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("chunk_size", ctypes.c_int), ("alpha", ctypes.c_float),
                ("gamma", ctypes.c_float), ("sigma", ctypes.c_float),
                ("enable_gqa", ctypes.c_int), ("flags", ctypes.c_uint), ("topk", ctypes.c_int)]


_vp = ctypes.c_void_p
_P = ctypes.POINTER(Params)
_sz = ctypes.c_size_t


def load_library(path: str) -> ctypes.CDLL:
    """Load a build of libdash (libdash.so, or the bounds-checking libdash_debug.so) and
    declare its C signatures."""
    lib = ctypes.CDLL(path)
    _declare(lib)
    return lib


def _declare(lib):
    lib.dash_prefill_workspace_size.argtypes = [_P]
    lib.dash_prefill_workspace_size.restype = _sz
    lib.dash_attend_workspace_size.argtypes = [_P]
    lib.dash_attend_workspace_size.restype = _sz
    lib.dash_decode_workspace_size.argtypes = [_P]
    lib.dash_decode_workspace_size.restype = _sz
    lib.dash_prefill.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_prefill_host.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                      ctypes.c_int, _vp, _vp, _vp]
    lib.dash_stage0.argtypes = [_P, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_route.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_attend.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_update_chunk_cache.argtypes = [_P, _vp, _vp, _vp, ctypes.c_int, _vp, _vp, _sz, _vp]
    lib.dash_decode.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_read_device_status.argtypes = [_vp, _vp]
    lib.dash_backward_workspace_size.argtypes = [_P]
    lib.dash_backward_workspace_size.restype = _sz
    lib.dash_backward.argtypes = [_P] + [_vp] * 11 + [_sz, _vp]
    lib.dash_backward.restype = ctypes.c_int
    lib.dash_decode_paged.argtypes = [_P, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp,
                                      _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_decode_step_workspace_size.argtypes = [_P]
    lib.dash_decode_step_workspace_size.restype = _sz
    lib.dash_decode_step.argtypes = [_P] + [_vp] * 12 + [_sz, _vp]
    lib.dash_decode_step_paged.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int,
                                           _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dash_update_chunk_cache_paged.argtypes = [_P, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int,
                                                  _vp, ctypes.c_int, _vp, _vp, _sz, _vp]
    lib.dash_status_string.argtypes = [ctypes.c_int]
    lib.dash_attend_kernel_name.argtypes = [_P, _sz]
    lib.dash_attend_kernel_name.restype = ctypes.c_char_p
    lib.dash_stage2_kernel_ran.argtypes = [_vp, _vp]
    lib.dash_stage2_kernel_ran.restype = ctypes.c_char_p
    lib.dash_prefill_kernel_count.argtypes = [_P, _sz]
    lib.dash_prefill_kernel_count.restype = ctypes.c_int
    lib.dash_status_string.restype = ctypes.c_char_p
    for _f in ("dash_prefill", "dash_stage0", "dash_route", "dash_attend",
               "dash_update_chunk_cache", "dash_decode", "dash_read_device_status",
               "dash_decode_paged", "dash_update_chunk_cache_paged"):
        getattr(lib, _f).restype = ctypes.c_int


lib = load_library(LIB_PATH)


class DashError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def _check(code: int, where: str):
    if code != DASH_OK:
        raise DashError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_params(batch, heads_q, heads_kv, seq_len, head_dim, chunk_size=64, alpha=1.5,
                gamma=1.0, sigma=1.0, enable_gqa=False, flags=0, topk=0) -> Params:
    return Params(int(batch), int(heads_q), int(heads_kv), int(seq_len), int(head_dim),
                  int(chunk_size), float(alpha), float(gamma), float(sigma),
                  1 if enable_gqa else 0, int(flags), int(topk))


def _flags(dense, force_all_active, estimate_diagonal):
    return ((FLAG_DENSE if dense else 0) | (FLAG_FORCE_ALL_ACTIVE if force_all_active else 0)
            | (FLAG_ESTIMATE_DIAGONAL if estimate_diagonal else 0))


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


def prefill_workspace_size(params: Params) -> int:
    return int(lib.dash_prefill_workspace_size(ctypes.byref(params)))


def attend_workspace_size(params: Params) -> int:
    return int(lib.dash_attend_workspace_size(ctypes.byref(params)))


def decode_workspace_size(params: Params) -> int:
    return int(lib.dash_decode_workspace_size(ctypes.byref(params)))


def attend_kernel_name(params: Params, ws_bytes: int) -> str:
    """Name of the Stage 2 kernel dash_attend launches with a workspace of ws_bytes."""
    return lib.dash_attend_kernel_name(ctypes.byref(params), int(ws_bytes)).decode()


def stage2_kernel_ran(ws) -> str:
    """The Stage 2 kernel a run-time choice ran in the last call with workspace ws ("" if that
    call made no run-time choice); synchronises the current stream."""
    return lib.dash_stage2_kernel_ran(_ptr(ws), _stream(ws.device)).decode()


def prefill_kernel_count(params: Params, ws_bytes: int) -> int:
    """Kernels one dash_prefill call launches with a workspace of ws_bytes."""
    return int(lib.dash_prefill_kernel_count(ctypes.byref(params), int(ws_bytes)))


def workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def prefill(q, k, v, head_cls, chunk_size=64, alpha=1.5, gamma=1.0, sigma=1.0,
            enable_gqa=False, return_p=False, return_active_blocks=False,
            return_summary=False, dense=False, force_all_active=False,
            estimate_diagonal=False, out=None, ws=None, topk=0, fuse_route=False):
    """Causal prefill.  q [B,Hq,T,D], k/v [B,Hkv,T,D] bf16 CUDA; head_cls [Hkv,D] fp32.

    Returns out [B,Hq,T,D] bf16, or a dict with out and the requested p [B,Hkv,T,C] fp32,
    active_blocks [B,Hkv,T,W] int64 (bit-packed uint64 words) and summary [B,Hkv,T//Bc,D]."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    C = (T + chunk_size - 1) // chunk_size
    W = (C + 63) // 64
    dev = q.device
    prm = make_params(B, Hq, Hkv, T, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(dense, force_all_active, estimate_diagonal)
                      | (FLAG_FUSE_ROUTE if fuse_route else 0), topk)
    _need(q, torch.bfloat16, (B, Hq, T, D), "q")
    _need(k, torch.bfloat16, (B, Hkv, T, D), "k")
    _need(v, torch.bfloat16, (B, Hkv, T, D), "v")
    if not dense:
        _need(head_cls, torch.float32, (Hkv, D), "head_cls")
    if out is None:
        out = torch.empty_like(q)
    p = torch.empty(B, Hkv, T, C, dtype=torch.float32, device=dev) if return_p else None
    mask = (torch.empty(B, Hkv, T, W, dtype=torch.int64, device=dev)
            if return_active_blocks else None)
    summ = (torch.empty(B, Hkv, T // chunk_size, D, dtype=torch.float32, device=dev)
            if return_summary else None)
    if ws is None:
        ws = workspace(prefill_workspace_size(prm), dev)
    _check(lib.dash_prefill(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v),
                            _ptr(head_cls) if head_cls is not None else None, _ptr(out),
                            _ptr(summ), _ptr(p), _ptr(mask), _ptr(ws), ws.numel(),
                            _stream(dev)), "dash_prefill")
    if not (return_p or return_active_blocks or return_summary):
        return out
    return dict(out=out, p=p, active_blocks=mask, summary=summ, ws=ws)


_copy_streams = {}


def prefill_host(q_host, k_host, v_host, head_cls_host, out_host, q, k, v, head_cls, out,
                 chunk_size=64, alpha=1.5, gamma=1.0, sigma=1.0, enable_gqa=False,
                 dense=False, force_all_active=False, n_slices=8, ws=None, fuse_route=False):
    """Causal prefill with inputs and output in page-locked host tensors (q_host, k_host,
    v_host, head_cls_host in; out_host out), the copies overlapped with the computation in
    row slices.  q, k, v, head_cls, out are the device buffers it fills and uses (same
    shapes).  Enqueued on the current stream (two copy streams of its own per device); out_host
    is valid once the current stream is synchronised."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    dev = q.device
    prm = make_params(B, Hq, Hkv, T, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(dense, force_all_active, False) | (FLAG_FUSE_ROUTE if fuse_route else 0))
    for name, h, d, dt in (("q", q_host, q, torch.bfloat16), ("k", k_host, k, torch.bfloat16),
                           ("v", v_host, v, torch.bfloat16), ("out", out_host, out, torch.bfloat16)):
        _need(d, dt, tuple(d.shape), name)
        if h.shape != d.shape or h.dtype != dt or h.device.type != "cpu" or not h.is_contiguous():
            raise ValueError(f"{name}_host must be a contiguous CPU {dt} tensor of shape {tuple(d.shape)}")
    if ws is None:
        ws = workspace(prefill_workspace_size(prm), dev)
    if dev not in _copy_streams:
        _copy_streams[dev] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    hs, ds = _copy_streams[dev]
    hc = None if head_cls is None else head_cls
    _check(lib.dash_prefill_host(ctypes.byref(prm), q_host.data_ptr(), k_host.data_ptr(),
                                 v_host.data_ptr(),
                                 None if head_cls_host is None else head_cls_host.data_ptr(),
                                 out_host.data_ptr(), _ptr(q), _ptr(k), _ptr(v), _ptr(hc), _ptr(out),
                                 _ptr(ws), ws.numel(), int(n_slices), _stream(dev),
                                 ctypes.c_void_p(hs.cuda_stream), ctypes.c_void_p(ds.cuda_stream)),
           "dash_prefill_host")
    return out_host


def stage0(k, head_cls, chunk_size=64, ws=None, summary=None):
    B, Hkv, T, D = k.shape
    prm = make_params(B, Hkv, Hkv, T, D, chunk_size)
    if summary is None:
        summary = torch.empty(B, Hkv, T // chunk_size, D, dtype=torch.float32, device=k.device)
    if ws is None:
        ws = workspace(256, k.device)
    _check(lib.dash_stage0(ctypes.byref(prm), _ptr(k), _ptr(head_cls), _ptr(summary), _ptr(ws),
                           ws.numel(), _stream(k.device)), "dash_stage0")
    return summary


def route(q, summary, heads_kv, chunk_size=64, alpha=1.5, gamma=1.0, enable_gqa=True,
          return_p=True, ws=None, topk=0):
    """Stage 1 alone: returns dict(tau [B,Hkv,T], active_blocks [B,Hkv,T,W], p or None)."""
    B, Hq, T, D = q.shape
    C = (T + chunk_size - 1) // chunk_size
    W = (C + 63) // 64
    prm = make_params(B, Hq, heads_kv, T, D, chunk_size, alpha, gamma, 1.0, enable_gqa, 0, topk)
    dev = q.device
    tau = torch.empty(B, heads_kv, T, dtype=torch.float32, device=dev)
    mask = torch.empty(B, heads_kv, T, W, dtype=torch.int64, device=dev)
    p = torch.empty(B, heads_kv, T, C, dtype=torch.float32, device=dev) if return_p else None
    if ws is None:
        ws = workspace(256, dev)
    _check(lib.dash_route(ctypes.byref(prm), _ptr(q), _ptr(summary), _ptr(tau), _ptr(p),
                          _ptr(mask), _ptr(ws), ws.numel(), _stream(dev)), "dash_route")
    return dict(tau=tau, active_blocks=mask, p=p, ws=ws)


def attend(q, k, v, summary, tau, active_blocks, chunk_size=64, alpha=1.5, gamma=1.0,
           sigma=1.0, enable_gqa=True, dense=False, force_all_active=False, ws=None, out=None,
           topk=0):
    """Stage 2 alone from a given routing."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    prm = make_params(B, Hq, Hkv, T, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(dense, force_all_active, False), topk)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = workspace(lib.dash_attend_workspace_size(ctypes.byref(prm)), q.device)
    _check(lib.dash_attend(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(summary),
                           _ptr(tau), _ptr(active_blocks), _ptr(out), _ptr(ws), ws.numel(),
                           _stream(q.device)), "dash_attend")
    return out


def update_chunk_cache(k_cache, head_cls, seq_lens, summary_cache, heads_q, chunk_size=64,
                       n_recent=1, ws=None):
    """Stage 0 over each sequence's last n_recent complete chunks (in place)."""
    B, Hkv, cap, D = k_cache.shape
    prm = make_params(B, heads_q, Hkv, cap, D, chunk_size, enable_gqa=True)
    if ws is None:
        ws = workspace(256, k_cache.device)
    _check(lib.dash_update_chunk_cache(ctypes.byref(prm), _ptr(k_cache), _ptr(head_cls),
                                       _ptr(seq_lens), int(n_recent), _ptr(summary_cache),
                                       _ptr(ws), ws.numel(), _stream(k_cache.device)),
           "dash_update_chunk_cache")
    return summary_cache


def decode(q, k_cache, v_cache, seq_lens, summary_cache, chunk_size=64, alpha=1.5, gamma=1.0,
           sigma=1.0, enable_gqa=True, return_p=False, return_active_blocks=False, out=None,
           ws=None, p=None, active_blocks=None, estimate_diagonal=False, head_cls=None, topk=0):
    """One decode step for the token at seq_lens[b]-1 of every sequence.  q [B,Hq,D];
    head_cls [Hkv,D] fp32 is needed with estimate_diagonal."""
    B, Hq, D = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    Ccap = (cap + chunk_size - 1) // chunk_size
    Wcap = (Ccap + 63) // 64
    dev = q.device
    prm = make_params(B, Hq, Hkv, cap, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(False, False, estimate_diagonal), topk)
    if out is None:
        out = torch.empty_like(q)
    if return_p and p is None:
        p = torch.empty(B, Hkv, Ccap, dtype=torch.float32, device=dev)
    if return_active_blocks and active_blocks is None:
        active_blocks = torch.empty(B, Hkv, Wcap, dtype=torch.int64, device=dev)
    if ws is None:
        ws = workspace(decode_workspace_size(prm), dev)
    _check(lib.dash_decode(ctypes.byref(prm), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                           _ptr(seq_lens), _ptr(summary_cache), _ptr(head_cls), _ptr(out), _ptr(p),
                           _ptr(active_blocks), _ptr(ws), ws.numel(), _stream(dev)),
           "dash_decode")
    if not (return_p or return_active_blocks):
        return out
    return dict(out=out, p=p, active_blocks=active_blocks)


def update_chunk_cache_paged(k_pool, head_cls, block_table, seq_lens, summary_pool, heads_q,
                             chunk_size=64, n_recent=1, ws=None):
    """Stage 0 over each sequence's last n_recent complete chunks of a paged cache (in place):
    k_pool [n_pages,Hkv,Bc,D] bf16, block_table [B,max_blocks] int32, summary_pool
    [n_pages,Hkv,D] fp32."""
    n_pages, Hkv, Bc, D = k_pool.shape
    B, max_blocks = block_table.shape
    prm = make_params(B, heads_q, Hkv, max_blocks * chunk_size, D, chunk_size, enable_gqa=True)
    if ws is None:
        ws = workspace(256, k_pool.device)
    _check(lib.dash_update_chunk_cache_paged(ctypes.byref(prm), _ptr(k_pool), _ptr(head_cls),
                                             _ptr(block_table), int(max_blocks), int(n_pages),
                                             _ptr(seq_lens), int(n_recent), _ptr(summary_pool),
                                             _ptr(ws), ws.numel(), _stream(k_pool.device)),
           "dash_update_chunk_cache_paged")
    return summary_pool


def decode_paged(q, k_pool, v_pool, block_table, seq_lens, summary_pool, chunk_size=64,
                 alpha=1.5, gamma=1.0, sigma=1.0, enable_gqa=True, return_p=False,
                 return_active_blocks=False, out=None, ws=None, estimate_diagonal=False,
                 head_cls=None, topk=0):
    """One decode step on a paged cache (see update_chunk_cache_paged for the layouts)."""
    B, Hq, D = q.shape
    n_pages, Hkv = k_pool.shape[0], k_pool.shape[1]
    max_blocks = block_table.shape[1]
    cap = max_blocks * chunk_size
    Ccap = max_blocks
    Wcap = (Ccap + 63) // 64
    dev = q.device
    prm = make_params(B, Hq, Hkv, cap, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(False, False, estimate_diagonal), topk)
    out = torch.empty_like(q) if out is None else out
    p = torch.empty(B, Hkv, Ccap, dtype=torch.float32, device=dev) if return_p else None
    mask = torch.empty(B, Hkv, Wcap, dtype=torch.int64, device=dev) if return_active_blocks else None
    if ws is None:
        ws = workspace(decode_workspace_size(prm), dev)
    _check(lib.dash_decode_paged(ctypes.byref(prm), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                 _ptr(block_table), int(max_blocks), int(n_pages), _ptr(seq_lens),
                                 _ptr(summary_pool), _ptr(head_cls), _ptr(out), _ptr(p), _ptr(mask),
                                 _ptr(ws), ws.numel(), _stream(dev)), "dash_decode_paged")
    if not (return_p or return_active_blocks):
        return out
    return dict(out=out, p=p, active_blocks=mask)


def decode_step(q, k_new, v_new, k_cache, v_cache, seq_lens, summary_cache, head_cls,
                chunk_size=64, alpha=1.5, gamma=1.0, sigma=1.0, enable_gqa=True, return_p=False,
                return_active_blocks=False, out=None, ws=None, estimate_diagonal=False, topk=0,
                block_table=None, p=None, active_blocks=None):
    """A whole decode step in one launch: k_new, v_new [B,Hkv,D] bf16 are appended at row
    seq_lens[b] of the caches, q [B,Hq,D] attends over seq_lens[b] + 1 tokens, a chunk the new
    token completes gets its summary, and seq_lens is incremented (all in place).  With
    block_table the caches are page pools (see update_chunk_cache_paged).  A ws passed in
    must have been zero-filled before its first step; the step does not clear its status
    word (read_device_status does)."""
    B, Hq, D = q.shape
    dev = q.device
    if block_table is None:
        Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    else:
        Hkv = k_cache.shape[1]
        cap = block_table.shape[1] * chunk_size
    Ccap = (cap + chunk_size - 1) // chunk_size
    Wcap = (Ccap + 63) // 64
    prm = make_params(B, Hq, Hkv, cap, D, chunk_size, alpha, gamma, sigma, enable_gqa,
                      _flags(False, False, estimate_diagonal), topk)
    out = torch.empty_like(q) if out is None else out
    if p is None and return_p:
        p = torch.empty(B, Hkv, Ccap, dtype=torch.float32, device=dev)
    mask = active_blocks
    if mask is None and return_active_blocks:
        mask = torch.empty(B, Hkv, Wcap, dtype=torch.int64, device=dev)
    if ws is None:       # zero-filled before its first step (the arrival counters)
        ws = torch.zeros(max(256, lib.dash_decode_step_workspace_size(ctypes.byref(prm))),
                         dtype=torch.uint8, device=dev)
    if block_table is None:
        _check(lib.dash_decode_step(ctypes.byref(prm), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(seq_lens), _ptr(summary_cache), _ptr(head_cls),
                                    _ptr(out), _ptr(p), _ptr(mask), _ptr(ws), ws.numel(), _stream(dev)),
               "dash_decode_step")
    else:
        _check(lib.dash_decode_step_paged(ctypes.byref(prm), _ptr(q), _ptr(k_new), _ptr(v_new),
                                          _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                          int(block_table.shape[1]), int(k_cache.shape[0]),
                                          _ptr(seq_lens), _ptr(summary_cache), _ptr(head_cls), _ptr(out),
                                          _ptr(p), _ptr(mask), _ptr(ws), ws.numel(), _stream(dev)),
               "dash_decode_step_paged")
    if not (return_p or return_active_blocks):
        return out
    return dict(out=out, p=p, active_blocks=mask)


def backward(q, k, v, head_cls, out, dout, chunk_size=64, alpha=1.5, gamma=1.0, sigma=1.0,
             enable_gqa=True, ws=None):
    """Gradients of sum(out * dout) w.r.t. q, k, v, head_cls (fp32 tensors) through the three
    stages.  out is the forward's output for the same arguments."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    dev = q.device
    prm = make_params(B, Hq, Hkv, T, D, chunk_size, alpha, gamma, sigma, enable_gqa)
    for name, t_, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                         ("out", out, torch.bfloat16), ("dout", dout, torch.bfloat16)):
        _need(t_, dt, tuple(t_.shape), name)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    dhc = torch.empty(head_cls.shape, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(lib.dash_backward_workspace_size(ctypes.byref(prm)), dev)
    _check(lib.dash_backward(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(head_cls), _ptr(out),
                             _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dhc), _ptr(ws), ws.numel(),
                             _stream(dev)), "dash_backward")
    return dict(dq=dq, dk=dk, dv=dv, dhc=dhc, ws=ws)


def read_device_status(ws) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    return int(lib.dash_read_device_status(_ptr(ws), _stream(ws.device)))
