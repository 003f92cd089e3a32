"""dash_prefill_static_ws: the prefill entry point for callers that cannot allocate device
memory (for example a plugin whose host application owns every device allocation, or a
latency-bound loop that cannot afford cudaMalloc's blocking).  Its scratch lives in a
library-owned device array of DASH_STATIC_WS_BYTES, and dash_static_ws_read_status reads its
device status word.  The tests call both through the C ABI.  A first call with another shape,
chunk size, alpha and data leaves different contents in the shared array; the next two calls
must still match dash_prefill (which takes a caller-provided workspace) and the oracle.  This
file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from dash_inputs import PrefillConfig, make_prefill
from parity_util import O_MAX_TOL, O_MEAN_TOL, P_TOL, check_output

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 16 << 20      # DASH_STATIC_WS_BYTES in include/dash.h
FLAG_TEST_STALL_WAIT = 16


def _bind(lib):
    f = lib.dash_prefill_static_ws
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.c_void_p] + [vp] * 9
    f.restype = ctypes.c_int
    r = lib.dash_static_ws_read_status
    r.argtypes = [vp]
    r.restype = ctypes.c_int
    return f, r


def _call(f, prm, q, k, v, hc, out, p, stream):
    return f(ctypes.addressof(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), hc.data_ptr(),
             out.data_ptr(), None, None if p is None else p.data_ptr(), None, stream)


def test_static_workspace_prefill_matches_dash_prefill_twice():
    import sparse_hierarchical_attention_stage0_b200 as dash
    f, read_status = _bind(dash.lib)
    dev = "cuda"
    stream = torch.cuda.current_stream().cuda_stream
    # A first call with other sizes and data: chunk 128, alpha 2, more rows, other seed.
    cfg0 = PrefillConfig("pre", 1, 16, 2, 6144 + 100, 128, 128, 2.0, planted=True, n_max=6, seed=5)
    q0, k0, v0, hc0 = (x.to(dev) for x in make_prefill(cfg0))
    prm0 = dash.make_params(1, 16, 2, q0.shape[2], 128, 128, 2.0, 1.0, 1.0, True)
    out0 = torch.empty_like(q0)
    assert _call(f, prm0, q0, k0, v0, hc0, out0, None, stream) == 0
    assert read_status(stream) == 0

    cfg = PrefillConfig("nz", 1, 32, 2, 4096 + 48, 128, 64, 1.5, planted=True, n_max=12, seed=77)
    q_h, k_h, v_h, hc_h = make_prefill(cfg)
    q, k, v, hc = (x.to(dev) for x in (q_h, k_h, v_h, hc_h))
    B, Hq, T, D = q.shape
    Hkv, C = k.shape[1], (T + 63) // 64
    ref = dash.prefill(q, k, v, hc, 64, 1.5, enable_gqa=True, return_p=True)
    prm = dash.make_params(B, Hq, Hkv, T, D, 64, 1.5, 1.0, 1.0, True)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        p = torch.full((B, Hkv, T, C), float("nan"), device=dev)
        rc = _call(f, prm, q, k, v, hc, out, p, stream)
        assert rc == 0, dash.STATUS_NAMES.get(rc, rc)
        assert read_status(stream) == 0, f"call {call}"
        err = (out.float() - ref["out"].float()).abs()
        assert torch.isfinite(out.float()).all(), f"call {call}"
        assert err.max().item() <= O_MAX_TOL and err.mean().item() <= O_MEAN_TOL, f"call {call}"
        assert (p - ref["p"]).abs().max().item() <= P_TOL, f"call {call}"
    # The last call against the oracle on sampled rows.
    rows = np.unique(np.r_[0, 63, 64, 65, 1000, 2047, 2048, 3333, np.arange(T - 8, T)])
    orc = oracle.prefill(q_h, k_h, v_h, hc_h, 64, 1.5, rows=rows)
    rt = torch.from_numpy(rows).to(dev)
    assert np.abs(p.index_select(2, rt).cpu().double().numpy() - orc["p"]).max() <= P_TOL
    check_output(out.index_select(2, rt).cpu().float().numpy(), orc["O"], tag="static ws")


def test_static_workspace_status_word_reports_a_device_timeout():
    """The Stage 0 test hook makes its bounded copy wait run out (2 s): the fault lands in the
    status word inside the static array, dash_static_ws_read_status returns it once (then
    DASH_OK, the read clears it), and the next call runs clean."""
    import sparse_hierarchical_attention_stage0_b200 as dash
    f, read_status = _bind(dash.lib)
    dev = "cuda"
    stream = torch.cuda.current_stream().cuda_stream
    q, k, v, hc = (x.to(dev) for x in make_prefill(
        PrefillConfig("st", 1, 2, 2, 256, 128, 64, 1.5, seed=62)))      # 4 chunks: one CTA waits
    out = torch.empty_like(q)
    for flags, want in ((FLAG_TEST_STALL_WAIT, 5), (0, 0)):
        prm = dash.make_params(1, 2, 2, 256, 128, 64, 1.5, 1.0, 1.0, False, flags=flags)
        assert _call(f, prm, q, k, v, hc, out, None, stream) == 0
        assert read_status(stream) == want, flags
        assert read_status(stream) == 0
    ref = dash.prefill(q, k, v, hc, 64, 1.5)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_static_workspace_refuses_sizes_beyond_its_array():
    import sparse_hierarchical_attention_stage0_b200 as dash
    f, _ = _bind(dash.lib)
    # 128K rows x 2 KV heads: tau (1 MiB) + summaries (2 MiB) + mask words (64 MiB) > 16 MiB
    prm = dash.make_params(1, 32, 2, 131072, 128, 64, 1.5, 1.0, 1.0, True)
    fake = 1 << 20
    rc = f(ctypes.addressof(prm), fake, fake, fake, fake, fake, None, None, None, None)
    assert rc == 3                                                   # WORKSPACE_TOO_SMALL
    need = 256 + 131072 * 2 * 4 + 2048 * 2 * 128 * 4 + 131072 * 2 * 32 * 8
    assert need > STATIC_WS_BYTES
    # Bad parameters keep their own status (head_dim 96 is unsupported, not too large).
    prm = dash.make_params(1, 2, 2, 256, 96, 64, 1.5, 1.0, 1.0, False)
    rc = f(ctypes.addressof(prm), fake, fake, fake, fake, fake, None, None, None, None)
    assert rc == 2                                                   # UNSUPPORTED
