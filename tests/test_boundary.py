"""The C-ABI library: it loads, exports every symbol include/dash.h declares, and its host-side
argument checks return the documented status codes before any launch (CPU only: no call
here reaches a CUDA API)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dash.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dash_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def dash():
    import sparse_hierarchical_attention_stage0_b200 as d
    return d


def test_header_declares_the_documented_entry_points():
    names = _declared()
    for n in ("dash_prefill", "dash_decode", "dash_update_chunk_cache", "dash_stage0",
              "dash_route", "dash_attend", "dash_read_device_status", "dash_status_string",
              "dash_prefill_workspace_size", "dash_decode_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(dash):
    for name in _declared():
        assert hasattr(dash.lib, name), name          # ctypes resolves via dlsym
    assert set(dash.EXPORTS) == set(_declared())


def test_status_strings(dash):
    for code, name in dash.STATUS_NAMES.items():
        assert dash.lib.dash_status_string(code).decode() == name
    assert dash.lib.dash_status_string(99).decode() == "DASH_ERR_UNKNOWN"


def _p(dash, **kw):
    base = dict(batch=1, heads_q=32, heads_kv=2, seq_len=4096, head_dim=128, chunk_size=64,
                alpha=1.5, gamma=1.0, sigma=1.0, enable_gqa=True, flags=0)
    base.update(kw)
    return dash.make_params(**base)


def test_workspace_sizes(dash):
    prm = _p(dash, heads_q=2)
    B, Hkv, T, D, Bc = 1, 2, 4096, 128, 64
    C = T // Bc
    W = (C + 63) // 64
    r = lambda x: (x + 255) // 256 * 256
    expect = 256 + r(B * Hkv * T * 4) + r(B * Hkv * (T // Bc) * D * 4) + r(B * Hkv * T * W * 8)
    assert dash.prefill_workspace_size(prm) == expect
    assert dash.attend_workspace_size(prm) == 256
    g16 = _p(dash, heads_q=32, heads_kv=2, seq_len=1001)
    T2 = 1001
    C2 = (T2 + Bc - 1) // Bc
    W2 = (C2 + 63) // 64
    vt2 = r(B * Hkv * D * ((T2 + 7) // 8 * 8) * 2)
    assert dash.attend_workspace_size(g16) == 256 + vt2
    assert dash.prefill_workspace_size(g16) == (256 + r(B * Hkv * T2 * 4) + r(B * Hkv * (T2 // Bc) * D * 4)
                                                + r(B * Hkv * T2 * W2 * 8) + vt2)
    assert dash.attend_workspace_size(_p(dash, head_dim=96)) == 0
    assert dash.decode_workspace_size(prm) == 256
    assert dash.prefill_workspace_size(_p(dash, head_dim=96)) == 0


FAKE = 1 << 20      # a 256-aligned fake device address; never dereferenced on these paths


@pytest.mark.parametrize("kw,code", [
    (dict(heads_q=31), 1),                      # heads_q % heads_kv != 0
    (dict(enable_gqa=False), 1),                # GQA disabled with Hq != Hkv
    (dict(alpha=0.5), 1),
    (dict(alpha=float("nan")), 1),
    (dict(gamma=0.0), 1),
    (dict(sigma=-1.0), 1),
    (dict(flags=64), 1),                        # unknown flag bit
    (dict(flags=128), 1),
    (dict(topk=-1), 1),
    (dict(topk=8, flags=4), 2),                 # top-k with estimate_diagonal
    (dict(head_dim=96), 2),
    (dict(chunk_size=32), 2),
    (dict(heads_q=6, heads_kv=2), 2),           # G = 3 neither divides 16 nor is a multiple
    (dict(batch=0), 1),
    (dict(seq_len=0), 1),
    (dict(seq_len=64 * 200000), 2),             # too many chunks for the routing kernel
])
def test_prefill_rejects_bad_parameters_before_launch(dash, kw, code):
    prm = _p(dash, **kw)
    rc = dash.lib.dash_prefill(ctypes.byref(prm), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                               FAKE, 1 << 40, None)
    assert rc == code


def test_estimate_diagonal_is_accepted_by_prefill_and_refused_by_route(dash):
    prm = _p(dash, flags=dash.FLAG_ESTIMATE_DIAGONAL)
    assert dash.prefill_workspace_size(prm) == dash.prefill_workspace_size(_p(dash))
    rc = dash.lib.dash_route(ctypes.byref(prm), FAKE, FAKE, FAKE, None, FAKE, FAKE, 256, None)
    assert rc == 2                                  # needs the keys: dash_prefill only
    # decode with the flag needs head_cls
    rc = dash.lib.dash_decode(ctypes.byref(prm), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                              None, FAKE, 256, None)
    assert rc == 1


def test_test_hook_flags_are_accepted(dash):
    for f in (dash.FLAG_TEST_NEWTON_CAP, dash.FLAG_TEST_STALL_WAIT):
        prm = _p(dash, flags=f)
        assert dash.prefill_workspace_size(prm) == dash.prefill_workspace_size(_p(dash))


def test_prefill_rejects_bad_pointers_and_small_workspace(dash):
    prm = _p(dash)
    f = dash.lib.dash_prefill
    assert f(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, 1 << 40, None) == 1
    assert f(ctypes.byref(prm), None, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, 1 << 40,
             None) == 1
    assert f(ctypes.byref(prm), FAKE + 8, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE,
             1 << 40, None) == 1                                    # misaligned q
    assert f(ctypes.byref(prm), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE + 16,
             1 << 40, None) == 1                                    # misaligned workspace
    # the V^T scratch is optional: the smallest accepted workspace leaves it out
    need = dash.prefill_workspace_size(prm) - dash.attend_workspace_size(prm) + 256
    assert f(ctypes.byref(prm), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, need - 1,
             None) == 3
    dense = _p(dash, flags=1)
    assert f(ctypes.byref(dense), FAKE, FAKE, FAKE, None, FAKE, None, None, FAKE, FAKE, 1 << 40,
             None) == 1                                             # dense + routing output


def test_prefill_host_rejects_bad_arguments_before_any_copy(dash):
    prm = _p(dash)
    f = dash.lib.dash_prefill_host
    big = 1 << 40
    h = [FAKE] * 5                                   # q, k, v, head_cls, out on the host
    d = [FAKE] * 5                                   # their device buffers
    assert f(ctypes.byref(prm), *h, *d, FAKE, big, 0, None, None, None) == 1  # n_slices < 1
    assert f(ctypes.byref(prm), None, *h[1:], *d, FAKE, big, 8, None, None, None) == 1
    assert f(ctypes.byref(prm), *h[:4], None, *d, FAKE, big, 8, None, None, None) == 1
    assert f(ctypes.byref(prm), *h, FAKE + 8, *d[1:], FAKE, big, 8, None, None, None) == 1
    assert f(ctypes.byref(prm), *h, *d, FAKE, dash.prefill_workspace_size(prm) - 1, 8,
             None, None, None) == 3
    dense = _p(dash, flags=1)                        # no head_cls needed in dense mode
    assert f(ctypes.byref(dense), *h[:3], None, h[4], *d[:3], None, d[4], FAKE, big, 0,
             None, None, None) == 1


def test_decode_and_cache_reject_bad_arguments(dash):
    prm = _p(dash, seq_len=65792)
    d = dash.lib.dash_decode
    assert d(ctypes.byref(prm), FAKE, FAKE, FAKE, None, FAKE, None, FAKE, None, None, FAKE, 256,
             None) == 1                                             # no seq_lens
    assert d(ctypes.byref(prm), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, FAKE, 255,
             None) == 3
    dense = _p(dash, seq_len=65792, flags=1)
    assert d(ctypes.byref(dense), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, FAKE, 256,
             None) == 2
    wide = _p(dash, heads_q=64, heads_kv=2, seq_len=65792)         # G = 32: decode is G <= 16
    assert d(ctypes.byref(wide), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, FAKE, 256,
             None) == 2
    u = dash.lib.dash_update_chunk_cache
    assert u(ctypes.byref(prm), FAKE, FAKE, FAKE, 0, FAKE, FAKE, 256, None) == 1   # n_recent 0
    assert u(ctypes.byref(prm), FAKE, FAKE, FAKE + 2, 1, FAKE, FAKE, 256, None) == 1


def test_stage_entry_points_reject_missing_outputs(dash):
    prm = _p(dash)
    assert dash.lib.dash_stage0(ctypes.byref(prm), FAKE, FAKE, None, FAKE, 256, None) == 1
    assert dash.lib.dash_route(ctypes.byref(prm), FAKE, FAKE, FAKE, None, None, FAKE, 256,
                               None) == 1
    assert dash.lib.dash_attend(ctypes.byref(prm), FAKE, FAKE, FAKE, None, None, None, FAKE,
                                FAKE, 256, None) == 1       # routed mode needs the routing
    assert dash.lib.dash_read_device_status(None, None) == 1


def test_attend_kernel_name_follows_the_dispatch(dash):
    """The library names the Stage 2 kernel it picks (host only, nothing launched)."""
    big = 1 << 40
    assert dash.attend_kernel_name(_p(dash), big) == "k_attend_fa"
    assert dash.attend_kernel_name(_p(dash), 256) == "k_attend_tc"          # no room for V^T
    assert dash.attend_kernel_name(_p(dash, flags=1), big) == "k_attend_pair"
    assert dash.attend_kernel_name(_p(dash, flags=2), big) == "k_attend_pair"
    assert dash.attend_kernel_name(_p(dash, heads_q=8), big) == "k_attend_fa|k_attend"  # G = 4: chosen at run time
    assert dash.attend_kernel_name(_p(dash, heads_q=8), 256) == "k_attend"    # no V^T room, G < 8
    assert dash.attend_kernel_name(_p(dash, heads_q=8, flags=1), big) == "k_attend_pair"
    assert dash.attend_kernel_name(_p(dash, heads_q=4, flags=1), big) == "k_attend_fa"  # G = 2, chunk 64
    assert dash.attend_kernel_name(_p(dash, heads_q=4, chunk_size=128, flags=2), big) == "k_attend_pair"
    assert dash.attend_kernel_name(_p(dash, heads_q=2), big) == "k_attend"     # G = 1: 128 tokens per tile
    assert dash.attend_kernel_name(_p(dash, head_dim=64), big) == "k_attend"   # D = 64
    assert dash.attend_kernel_name(_p(dash, head_dim=96), big) == ""
    assert dash.attend_kernel_name(_p(dash), 255) == ""


def test_prefill_kernel_count_follows_the_dispatch(dash):
    """The library counts the kernels one dash_prefill call launches (host only)."""
    big = 1 << 40
    assert dash.prefill_kernel_count(_p(dash), big) == 4              # stage 0, route, V^T, 128-key blocks
    assert dash.prefill_kernel_count(_p(dash, flags=32), big) == 3    # fused route + attend on request
    assert dash.prefill_kernel_count(_p(dash), 256) == 3              # stage 0, route, 64-key blocks
    assert dash.prefill_kernel_count(_p(dash, flags=1), big) == 2     # dense: V^T, SM pairs
    assert dash.prefill_kernel_count(_p(dash, head_dim=64), big) == 3  # stage 0, route, warp MMA
    assert dash.prefill_kernel_count(_p(dash, flags=4 | 32), big) == 4   # estimated diagonal: never fused
    assert dash.prefill_kernel_count(_p(dash, head_dim=96), big) == 0
    # G = 4: stage 0, route, cost kernel, V^T, both Stage 2 kernels (one exits per CTA)
    assert dash.prefill_kernel_count(_p(dash, heads_q=8), big) == 6
    assert dash.prefill_kernel_count(_p(dash, heads_q=8, flags=1), big) == 2   # dense: V^T, SM pairs
