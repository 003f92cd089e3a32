"""dash_prefill_static_ws: the prefill entry point for callers that cannot allocate device
memory (for example a plugin whose host application owns every device allocation, or a
latency-bound loop that cannot afford cudaMalloc's blocking).  Its scratch lives in a
library-owned device array of DASH_STATIC_WS_BYTES.  The test calls it through the C ABI
twice in a row and checks both results against dash_prefill, which takes a caller-provided
workspace.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from dash_inputs import PrefillConfig, make_prefill
from parity_util import O_MAX_TOL, O_MEAN_TOL, P_TOL

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 16 << 20      # DASH_STATIC_WS_BYTES in include/dash.h


def _bind(lib):
    f = lib.dash_prefill_static_ws
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.c_void_p] + [vp] * 9
    f.restype = ctypes.c_int
    return f


def test_static_workspace_prefill_matches_dash_prefill_twice():
    import sparse_hierarchical_attention_stage0_b200 as dash
    f = _bind(dash.lib)
    dev = "cuda"
    cfg = PrefillConfig("nz", 1, 32, 2, 4096 + 48, 128, 64, 1.5, planted=True, n_max=12, seed=77)
    q, k, v, hc = (x.to(dev) for x in make_prefill(cfg))
    B, Hq, T, D = q.shape
    Hkv, C = k.shape[1], (T + 63) // 64
    ref = dash.prefill(q, k, v, hc, 64, 1.5, enable_gqa=True, return_p=True)
    prm = dash.make_params(B, Hq, Hkv, T, D, 64, 1.5, 1.0, 1.0, True)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        p = torch.full((B, Hkv, T, C), float("nan"), device=dev)
        rc = f(ctypes.addressof(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), hc.data_ptr(),
               out.data_ptr(), None, p.data_ptr(), None, stream)
        assert rc == 0, dash.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        err = (out.float() - ref["out"].float()).abs()
        assert torch.isfinite(out.float()).all(), f"call {call}"
        assert err.max().item() <= O_MAX_TOL and err.mean().item() <= O_MEAN_TOL, f"call {call}"
        assert (p - ref["p"]).abs().max().item() <= P_TOL, f"call {call}"


def test_static_workspace_refuses_sizes_beyond_its_array():
    import sparse_hierarchical_attention_stage0_b200 as dash
    f = _bind(dash.lib)
    # 128K rows x 2 KV heads: tau (1 MiB) + summaries (2 MiB) + mask words (64 MiB) > 16 MiB
    prm = dash.make_params(1, 32, 2, 131072, 128, 64, 1.5, 1.0, 1.0, True)
    fake = 1 << 20
    rc = f(ctypes.addressof(prm), fake, fake, fake, fake, fake, None, None, None, None)
    assert rc == 3                                                   # WORKSPACE_TOO_SMALL
    need = 256 + 131072 * 2 * 4 + 2048 * 2 * 128 * 4 + 131072 * 2 * 32 * 8
    assert need > STATIC_WS_BYTES
