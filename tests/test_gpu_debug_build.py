"""The bounds-checking build libdash_debug.so (the same kernels compiled with DASH_DEBUG: every
checked index is compared with its buffer's bounds, a failed check reports DASH_ERR_BOUNDS
through the status word and skips the access).  On odd shapes (ragged sequence lengths,
batch > 1, every Stage 2 kernel, sliced prefill from host memory, decode with ragged cache
lengths) it must report no violation and give the release library's output bit for bit."""
import pytest
import torch

from dash_inputs import PrefillConfig, make_prefill

pytestmark = pytest.mark.gpu
dev = "cuda"


@pytest.fixture(scope="module")
def libs():
    import sparse_hierarchical_attention_stage0_b200 as dash
    return dash, dash.lib, dash.load_library(dash.LIB_DEBUG_PATH)


def _both(dash, rel, dbg, monkeypatch, fn):
    """fn() run with the release and then the debug library behind the binding."""
    monkeypatch.setattr(dash, "lib", rel)
    a = fn()
    torch.cuda.synchronize()
    monkeypatch.setattr(dash, "lib", dbg)
    b = fn()
    torch.cuda.synchronize()
    monkeypatch.setattr(dash, "lib", rel)
    return a, b


@pytest.mark.parametrize("B,G,D,Bc,T,flags", [
    (2, 16, 128, 64, 1100 + 5, {}),                          # two-tile tensor-core kernel
    (1, 8, 128, 128, 1500 + 3, {}),
    (1, 4, 128, 128, 777, {}),                               # warp-MMA kernel
    (2, 1, 64, 64, 333, {}),
    (2, 8, 128, 128, 700, {"dense": True}),                  # pairs of SMs
    (1, 16, 128, 64, 640 + 17, {"estimate_diagonal": True}),
])
def test_debug_build_matches_release_without_violations(libs, monkeypatch, B, G, D, Bc, T, flags):
    dash, rel, dbg = libs
    Hkv = 2
    q, k, v, hc = (x.to(dev) for x in make_prefill(
        PrefillConfig("dbg", B, G * Hkv, Hkv, T, D, Bc, 1.5, planted=True, n_max=6, seed=90 + G)))
    dense = flags.get("dense", False)
    fl = (dash.FLAG_DENSE if dense else 0) | (dash.FLAG_ESTIMATE_DIAGONAL if flags.get("estimate_diagonal") else 0)
    prm = dash.make_params(B, G * Hkv, Hkv, T, D, Bc, 1.5, enable_gqa=True, flags=fl)

    def run():
        ws = dash.workspace(dash.prefill_workspace_size(prm), dev)
        r = dash.prefill(q, k, v, None if dense else hc, Bc, 1.5, enable_gqa=True, ws=ws,
                         return_active_blocks=not dense, return_p=not dense, **flags)
        r = r if isinstance(r, dict) else {"out": r}
        r["status"] = dash.read_device_status(ws)
        return r

    a, b = _both(dash, rel, dbg, monkeypatch, run)
    assert a["status"] == 0 and b["status"] == 0, (a["status"], b["status"])
    for key in ("out", "p", "active_blocks"):
        if a.get(key) is not None:
            assert torch.equal(a[key], b[key]), key


def test_debug_build_host_prefill_and_decode(libs, monkeypatch):
    dash, rel, dbg = libs
    B, Hkv, G, L, D, Bc = 3, 2, 16, 1300 + 9, 128, 64
    q, k, v, hc = make_prefill(PrefillConfig("dbg", B, G * Hkv, Hkv, L, D, Bc, 1.5, planted=True,
                                             n_max=6, seed=99))
    qd, kd, vd, hcd = (x.to(dev) for x in (q, k, v, hc))
    hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
    prm = dash.make_params(B, G * Hkv, Hkv, L, D, Bc, 1.5, enable_gqa=True)
    ws = dash.workspace(dash.prefill_workspace_size(prm), dev)

    def host():
        ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        bo = torch.empty_like(qd)
        dash.prefill_host(hq, hk, hv, hhc, ho, qd.clone(), kd.clone(), vd.clone(), hcd.clone(), bo,
                          Bc, 1.5, enable_gqa=True, n_slices=5, ws=ws, fuse_route=True)
        torch.cuda.current_stream().synchronize()
        assert dash.read_device_status(ws) == 0
        return ho

    a, b = _both(dash, rel, dbg, monkeypatch, host)
    assert torch.equal(a, b)

    cap = L + 100
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    kc[:, :, :L] = kd
    vc[:, :, :L] = vd
    lens = [L, Bc * 5, 17]
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    qs = torch.stack([qd[b, :, lens[b] - 1] for b in range(B)])

    def dec():
        cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
        wsu, wsd = dash.workspace(256, dev), dash.workspace(256, dev)
        dash.update_chunk_cache(kc, hcd, seq, cache, heads_q=G * Hkv, chunk_size=Bc,
                                n_recent=cap // Bc, ws=wsu)
        r = dash.decode(qs, kc, vc, seq, cache, Bc, return_p=True, return_active_blocks=True, ws=wsd)
        assert dash.read_device_status(wsu) == 0 and dash.read_device_status(wsd) == 0
        r["cache"] = cache
        return r

    a, b = _both(dash, rel, dbg, monkeypatch, dec)
    for key in ("out", "p", "active_blocks", "cache"):
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("Bc,L", [(64, 1300 + 9), (128, 900 + 3)])
def test_debug_build_four_heads_per_kv_head(libs, monkeypatch, Bc, L):
    """G = 4 at low sparsity (alpha 1.25): the 128-key-block kernel with 32-token tiles, whose
    routing biases come from two warps over summary rows staged in shared memory, through the
    full-range prefill (chosen at run time) and the sliced prefill from host memory (with the
    routing fused).  Ragged lengths leave a diagonal chunk without a summary row."""
    dash, rel, dbg = libs
    B, Hkv, G, D, alpha = 2, 2, 4, 128, 1.25
    q, k, v, hc = make_prefill(PrefillConfig("dbg", B, G * Hkv, Hkv, L, D, Bc, alpha, planted=True,
                                             n_max=6, seed=101 + Bc))
    qd, kd, vd, hcd = (x.to(dev) for x in (q, k, v, hc))
    hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
    prm = dash.make_params(B, G * Hkv, Hkv, L, D, Bc, alpha, enable_gqa=True)

    def run():
        ws = dash.workspace(dash.prefill_workspace_size(prm), dev)
        r = dash.prefill(qd, kd, vd, hcd, Bc, alpha, enable_gqa=True, ws=ws, return_active_blocks=True)
        st = dash.read_device_status(ws)
        ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        dash.prefill_host(hq, hk, hv, hhc, ho, qd.clone(), kd.clone(), vd.clone(), hcd.clone(),
                          torch.empty_like(qd), Bc, alpha, enable_gqa=True, n_slices=3, ws=ws,
                          fuse_route=True)
        torch.cuda.current_stream().synchronize()
        return {"out": r["out"], "active_blocks": r["active_blocks"], "host": ho,
                "status": (st, dash.read_device_status(ws))}

    a, b = _both(dash, rel, dbg, monkeypatch, run)
    assert a["status"] == (0, 0) and b["status"] == (0, 0), (a["status"], b["status"])
    for key in ("out", "active_blocks", "host"):
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("G,D,Bc,T", [(16, 128, 64, 300 + 5), (4, 128, 128, 607), (1, 64, 64, 333)])
def test_debug_build_backward_without_violations(libs, monkeypatch, G, D, Bc, T):
    """dash_backward (routing, the per-chunk token lists, query- and key-side kernels) under the
    bounds-checking build first, then the release build: no violation, and the same gradients
    up to the order of the atomic sums (d log p over head groups, dhc over chunks)."""
    dash, rel, dbg = libs
    Hkv = 2
    q, k, v, hc = (x.to(dev) for x in make_prefill(
        PrefillConfig("dbg", 1, G * Hkv, Hkv, T, D, Bc, 1.5, planted=True, n_max=6, seed=70 + G)))
    g_ = torch.Generator().manual_seed(5)
    dout = torch.randn(q.shape, generator=g_).to(torch.bfloat16).to(dev)
    res = {}
    for name, lib in (("debug", dbg), ("release", rel)):
        monkeypatch.setattr(dash, "lib", lib)
        out = dash.prefill(q, k, v, hc, Bc, 1.5, enable_gqa=True)
        gr = dash.backward(q, k, v, hc, out, dout, Bc, 1.5)
        torch.cuda.synchronize()
        assert dash.read_device_status(gr["ws"]) == 0, name
        res[name] = gr
    monkeypatch.setattr(dash, "lib", rel)
    for key in ("dq", "dk", "dv", "dhc"):
        a, b = res["debug"][key], res["release"][key]
        scale = b.abs().max().item()
        assert (a - b).abs().max().item() <= 1e-4 * max(scale, 1e-30), key
