"""The benchmark workloads at full size against the fp64 oracle, through the C ABI (via the
binding), in the launch configuration bench.py times:

  * 32K GQA and 128K prefill: the active-block mask and p on every row, O on a sampled row
    set, the sliced prefill from host memory equal bit for bit;
  * the incremental decode workload (16 sequences x 64K cached tokens, 256 steps, the
    chunk-representation cache updated whenever a chunk completes): mask and p every step,
    O at steps 1, 63, 64, 65, 128 and 256;
  * the six alpha x chunk_size cells of the 64K sweep (B = 2, H_kv = 8): mask, p and O on
    sampled rows; all blocks forced active against the oracle's dense causal attention and
    against the library's own dense path, bit for bit.
"""
import json
import os
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from dash_inputs import CONFIGS, SWEEP_DENSE_SEED, make_decode, make_prefill, sweep_config
from parity_util import check_output, check_routing, unpack_mask

pytestmark = pytest.mark.gpu

dev = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def dash():
    import sparse_hierarchical_attention_stage0_b200 as d
    return d


def _sample_rows(T, Bc, n_rand, seed):
    """The first and last 16 rows, the ends and starts of the first chunks and of a chunk in
    the middle, and n_rand uniform rows."""
    rng = np.random.default_rng(seed)
    mid = (T // 2) // Bc * Bc
    r = list(range(16)) + [Bc - 1, Bc, 2 * Bc - 1, 2 * Bc, mid - 1, mid] + list(range(T - 16, T))
    r += list(rng.integers(0, T, n_rand))
    return np.unique(np.array(r, dtype=np.int64))


def _routing_every_row(res, q64, S_or, cfg, slice_rows=4096):
    """Mask and p of every row against the oracle's Stage 1 (on the oracle's own summaries),
    slice by slice.  Returns the number of excused near-threshold mask mismatches."""
    T, Bc = cfg.seq_len, cfg.chunk_size
    C = (T + Bc - 1) // Bc
    n_ex = 0
    for r0 in range(0, T, slice_rows):
        rows = np.arange(r0, min(T, r0 + slice_rows))
        p_or, m_or, _ = oracle.stage1(q64, S_or, T, Bc, cfg.alpha, cfg.gamma, rows=rows)
        bits = unpack_mask(res["active_blocks"][:, :, r0:r0 + rows.size], C)
        p = res["p"][:, :, r0:r0 + rows.size].cpu().double().numpy()
        n_ex += check_routing(bits, p, p_or, m_or, rows, Bc, cfg.alpha, tag=f"{cfg.name} rows {r0}+")
    return n_ex


@pytest.mark.parametrize("name,n_rand", [("gqa32k", 96), ("prefill128k", 32)])
def test_full_size_prefill_every_row(dash, name, n_rand):
    """The 32K and 128K workloads at full size, through dash_prefill with the workspace the
    bench times (V^T scratch included: Stage 2 on a 128-key-block kernel).  Mask and p on
    every row, O on sampled rows; the sliced prefill from host memory equal bit for bit."""
    cfg = CONFIGS[name]
    if name == "prefill128k":
        with open(os.path.join(GOLDEN, "gamma_prefill128k.json")) as f:
            cfg = replace(cfg, gamma=json.load(f)["gamma"])
    q, k, v, hc = make_prefill(cfg)
    B, Hq, T, D = q.shape
    Hkv, Bc = k.shape[1], cfg.chunk_size
    qd, kd, vd, hcd = (x.to(dev) for x in (q, k, v, hc))
    prm = dash.make_params(B, Hq, Hkv, T, D, Bc, cfg.alpha, cfg.gamma, enable_gqa=True)
    assert dash.attend_kernel_name(prm, dash.prefill_workspace_size(prm)) == "k_attend_fa"
    res = dash.prefill(qd, kd, vd, hcd, Bc, cfg.alpha, cfg.gamma, enable_gqa=True,
                       return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    q64 = oracle._f64(q)
    S_or = oracle.stage0(k, hc, Bc)
    n_ex = _routing_every_row(res, q64, S_or, cfg)
    assert n_ex <= 1e-5 * B * Hkv * T * T / Bc / 2, n_ex       # near-threshold flips are rare
    rows = _sample_rows(T, Bc, n_rand, seed=cfg.seed + 100)
    rt = torch.from_numpy(rows).to(dev)
    ref = oracle.prefill(q64, k, v, hc, Bc, cfg.alpha, cfg.gamma, rows=rows)
    check_output(res["out"].index_select(2, rt).cpu().float().numpy(), ref["O"], tag=name)
    del res["p"]
    # The same workload from host memory in 16 row slices.
    hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    bo = torch.empty_like(qd)
    ws = dash.workspace(dash.prefill_workspace_size(prm), qd.device)
    dash.prefill_host(hq, hk, hv, hhc, ho, qd, kd, vd, hcd, bo, Bc, cfg.alpha, cfg.gamma,
                      enable_gqa=True, n_slices=16, ws=ws)
    torch.cuda.current_stream().synchronize()
    assert dash.read_device_status(ws) == 0
    assert torch.equal(bo, res["out"])
    assert torch.equal(ho, res["out"].cpu())


def test_decode_workload_at_full_size(dash):
    """16 sequences with 65536 cached tokens, 256 decode steps as bench.py runs them: each step
    appends its token's K/V, updates the chunk-representation cache when a chunk completes
    (L % 64 == 0), then decodes.  Mask and p of every step against the oracle's routing from
    its own summaries; O at steps 1, 63, 64, 65, 128 and 256; the cached summaries against the
    oracle's Stage 0, the newly completed chunks included, which the next steps can route to."""
    cfg = CONFIGS["decode64k"]
    d = make_decode(cfg)
    B, Hq, Hkv, D, Bc = cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.head_dim, cfg.chunk_size
    L0, S, cap = d["prefix_len"], d["steps"], d["capacity"]
    Ccap = (cap + Bc - 1) // Bc
    Wcap = (Ccap + 63) // 64
    k_all, v_all, hc = d["k_all"].to(dev), d["v_all"].to(dev), d["head_cls"].to(dev)
    q_steps = d["q_steps"].to(dev)
    kc = torch.zeros_like(k_all)
    vc = torch.zeros_like(v_all)
    kc[:, :, :L0] = k_all[:, :, :L0]
    vc[:, :, :L0] = v_all[:, :, :L0]
    cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
    seq = torch.full((B,), L0, dtype=torch.int32, device=dev)
    dash.update_chunk_cache(kc, hc, seq, cache, Hq, Bc, n_recent=L0 // Bc)
    ws, ws_u = dash.workspace(256, dev), dash.workspace(256, dev)
    o_steps = {1, 63, 64, 65, 128, 256}
    p_all = torch.empty(S, B, Hkv, Ccap, device=dev)
    m_all = torch.empty(S, B, Hkv, Wcap, dtype=torch.int64, device=dev)
    outs = {}
    for s in range(S):
        L = L0 + s + 1
        kc[:, :, L - 1] = k_all[:, :, L - 1]
        vc[:, :, L - 1] = v_all[:, :, L - 1]
        seq.fill_(L)
        if L % Bc == 0:
            dash.update_chunk_cache(kc, hc, seq, cache, Hq, Bc, n_recent=1, ws=ws_u)
        r = dash.decode(q_steps[s], kc, vc, seq, cache, Bc, cfg.alpha, return_p=True,
                        return_active_blocks=True, ws=ws, p=p_all[s], active_blocks=m_all[s])
        if s + 1 in o_steps:
            outs[s + 1] = r["out"].clone()
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0 and dash.read_device_status(ws_u) == 0
    completed = [L for L in range(L0 + 1, cap + 1) if L % Bc == 0]
    assert len(completed) == 4                                   # chunks 1024-1027 complete
    S_or = oracle.stage0(d["k_all"], d["head_cls"], Bc)          # [B,Hkv,cap/Bc,D]
    rel = np.abs(cache.cpu().double().numpy() - S_or).max() / np.abs(S_or).max()
    assert rel <= 1e-5, rel
    bits = unpack_mask(m_all, Ccap)                              # [S,B,Hkv,Ccap]
    p_gpu = p_all.cpu().double().numpy()
    routed_new = 0
    for s in range(S):
        L = L0 + s + 1
        t = L - 1
        ro = oracle.decode_route(d["q_steps"][s], S_or, [L] * B, cap, Bc, cfg.alpha)
        check_routing(bits[s][:, :, None], p_gpu[s][:, :, None], ro["p"][:, :, None],
                      ro["m"][:, :, None], [t], Bc, cfg.alpha, tag=f"decode step {s + 1}")
        if t // Bc > L0 // Bc:                                   # chunk 1024 is routable
            routed_new += int((ro["p"][:, :, L0 // Bc] > 0).sum())
    assert routed_new > 0                                        # some rows route to it
    k64, v64 = oracle._f64(d["k_all"]), oracle._f64(d["v_all"])
    for step in sorted(o_steps):
        L = L0 + step
        ref = oracle.decode(d["q_steps"][step - 1], k64, v64, d["head_cls"], [L] * B, Bc, cfg.alpha)
        check_output(outs[step].cpu().float().numpy(), ref["O"], tag=f"decode step {step}")


@pytest.mark.parametrize("cell", range(6))
def test_sweep_cell_every_row(dash, cell):
    """One alpha x chunk_size cell of the 64K sweep (B = 2, H_q = 32, H_kv = 8: four query
    heads per KV head): mask and p on every row of both sequences, O on sampled rows."""
    cfg = sweep_config(cell)
    q, k, v, hc = make_prefill(cfg)
    B, Hq, T, D = q.shape
    Hkv, Bc = k.shape[1], cfg.chunk_size
    qd, kd, vd, hcd = (x.to(dev) for x in (q, k, v, hc))
    res = dash.prefill(qd, kd, vd, hcd, Bc, cfg.alpha, cfg.gamma, enable_gqa=True,
                       return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    n_ex = _routing_every_row(res, oracle._f64(q), oracle.stage0(k, hc, Bc), cfg)
    assert n_ex <= 1e-5 * B * Hkv * T * T / Bc / 2, n_ex       # near-threshold flips are rare
    del res["p"]
    rows = _sample_rows(T, Bc, 64, seed=cfg.seed + 100)
    rt = torch.from_numpy(rows).to(dev)
    ref = oracle.prefill(q, k, v, hc, Bc, cfg.alpha, cfg.gamma, rows=rows)
    check_output(res["out"].index_select(2, rt).cpu().float().numpy(), ref["O"], tag=cfg.name)


@pytest.mark.parametrize("chunk_size", [64, 128])
def test_sweep_forced_all_active_equals_dense(dash, chunk_size):
    """The sweep's shape with every block forced active and a uniform prior: the same output
    as the library's dense path bit for bit, and the oracle's dense causal attention on
    sampled rows."""
    cfg = replace(sweep_config(0 if chunk_size == 64 else 1), seed=SWEEP_DENSE_SEED)
    q, k, v, hc = make_prefill(cfg)
    T, Bc = q.shape[2], cfg.chunk_size
    qd, kd, vd, hcd = (x.to(dev) for x in (q, k, v, hc))
    o_dense = dash.prefill(qd, kd, vd, None, Bc, enable_gqa=True, dense=True)
    o_force = dash.prefill(qd, kd, vd, hcd, Bc, cfg.alpha, enable_gqa=True, force_all_active=True)
    torch.cuda.synchronize()
    assert torch.equal(o_dense, o_force)
    rows = _sample_rows(T, Bc, 48, seed=cfg.seed + 100)
    rt = torch.from_numpy(rows).to(dev)
    ref = oracle.stage2(q, k, v, None, Bc, rows=rows, dense=True)
    check_output(o_dense.index_select(2, rt).cpu().float().numpy(), ref, tag="sweep dense")
