#!/usr/bin/env python
"""Benchmark of the DashAttention forward path on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dash|reference]
                    [--workload prefill128k|gqa32k|tiny|sweep|decode64k] [--no-decode]

A step is one causal prefill (Stage 0 -> Stage 1 -> Stage 2) over the workload's synthetic
seeded inputs, already resident in HBM.  value = prefill tokens/s over all ranks (replicas:
every rank runs the same workload on its own GPU, no data-path collective).  Also reported:
active-FLOP TFLOP/s of Stage 2, per-stage times and roofline fractions, the library's own
dense path, the end-to-end time through host buffers, a 256-step decode captured in one CUDA
graph, and the fp64 oracle timed on the host cores on a bounded row sample.  With
--workload sweep the line covers the six alpha x chunk_size cells of the 64K sweep instead
(per cell: tokens/s, active TFLOP/s, sparsity, Stage 0-1 GB/s, speedup vs the dense path,
union waste).

--impl reference times the oracle (plain fp64 C on the host cores) on the same workload and
metric: each step runs the oracle over a bounded sample of rows, extrapolated to the
workload's tokens/s.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from dash_inputs import CONFIGS, make_decode, make_prefill  # noqa: E402

METRIC = "prefill tokens/s & active-FLOP TFLOP/s at 128K; decode tok/s; % roofline"
GAMMA_FILE = os.path.join(ROOT, "tests", "golden", "gamma_prefill128k.json")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
E2E_SLICES = 16         # row slices of the end-to-end prefill from host memory (8: 130 ms, 16: 128 ms at 128K)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(name):
    if name == "sweep64k":
        from dash_inputs import sweep_config
        return sweep_config(2)                    # the reference arm times the alpha 1.5, chunk 64 cell
    cfg = CONFIGS[name]
    if name == "prefill128k":
        try:
            with open(GAMMA_FILE) as f:
                g = json.load(f)["gamma"]
            from dataclasses import replace
            cfg = replace(cfg, gamma=float(g))
        except (OSError, ValueError, KeyError):
            log("warning: no calibrated gamma for prefill128k; using 1.0")
    return cfg


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons during a region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if not self.proc:
            return None
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], swp=f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 250] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(loaded)}


# ------------------------------------------------------------------------------ helpers
def popcount_words(words: torch.Tensor) -> torch.Tensor:
    """Per-row popcount of int64 mask words [..., W] -> int64 [...]."""
    b = words.contiguous().view(torch.uint8)
    table = torch.tensor([bin(i).count("1") for i in range(256)], dtype=torch.int64,
                         device=words.device)
    return table[b.long()].view(*words.shape[:-1], -1).sum(-1)


def active_stats(dash, q, k, v, hc, cfg):
    """Realised routing of one run: active routed chunks per (b, g, t), block-weighted
    sparsity over the routed (visible) chunks, and Stage 2's active FLOPs."""
    res = dash.prefill(q, k, v, hc, cfg.chunk_size, cfg.alpha, cfg.gamma, enable_gqa=True,
                       return_active_blocks=True)
    words = res["active_blocks"]
    cnt = popcount_words(words) - 1                          # minus the diagonal bit
    del res
    T, Bc, D, G = cfg.seq_len, cfg.chunk_size, cfg.head_dim, cfg.group
    t = torch.arange(T, device=q.device)
    ct = t // Bc
    visible = ct.to(torch.float64).sum() * cfg.batch * cfg.heads_kv
    active = cnt.to(torch.float64).sum()
    diag_keys = (t - ct * Bc + 1).to(torch.float64).sum() * cfg.batch * cfg.heads_kv
    flops = 4.0 * D * G * (Bc * active + diag_keys)
    dense_flops = 4.0 * D * G * cfg.batch * cfg.heads_kv * (T * (T + 1) / 2.0)
    sparsity = 1.0 - float(active / visible) if visible > 0 else 0.0
    return dict(active_flops=float(flops), dense_flops=float(dense_flops), sparsity=sparsity,
                active_chunks=float(active), visible_chunks=float(visible), words=words,
                support=support_histogram(cnt))


def support_histogram(cnt: torch.Tensor) -> dict:
    """Entmax support sizes (routed active chunks per row, diagonal excluded) as a histogram
    over power-of-two bins, with quantiles: how adaptive the routing was."""
    c = cnt.flatten().to(torch.int64)
    edges = [0, 1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192]
    bins = {}
    for lo, hi in zip(edges[:-1], edges[1:]):
        n = int(((c >= lo) & (c < hi)).sum())
        if n:
            bins[f"{lo}-{hi - 1}"] = n
    n_big = int((c >= edges[-1]).sum())
    if n_big:
        bins[f">={edges[-1]}"] = n_big
    q = torch.quantile(c[:1 << 24].to(torch.float64), torch.tensor([0.1, 0.5, 0.9, 0.99], dtype=torch.float64, device=c.device))
    return {"rows": int(c.numel()), "bins": bins, "mean": float(c.to(torch.float64).mean()),
            "p10": float(q[0]), "p50": float(q[1]), "p90": float(q[2]), "p99": float(q[3]),
            "max": int(c.max()) if c.numel() else 0}


def tokens_per_tile(kernel: str, G: int) -> int:
    """Tokens whose rows share one Stage 2 work unit (and so walk the union of their routed
    chunks) in the named kernel: 128 rows of G heads per tile (two tiles per SM pair), or 16
    rows per warp in the warp-MMA kernel."""
    if kernel == "k_attend_pair":
        return max(1, 256 // G)
    if kernel in ("k_attend_fa", "k_attend_tc"):
        return max(1, 128 // G)
    return max(1, 16 // G)


def union_stats(words: torch.Tensor, chunk_size: int, head_dim: int, G: int, tpt: int):
    """Union waste of a Stage 2 kernel whose work units hold `tpt` consecutive tokens: each
    unit walks the OR of its tokens' mask words, so it executes (routed chunks of the union) x
    (its tokens) token-chunk pairs against the sum of the tokens' own active chunks.
    words: int64 [B, Hkv, T, W].  Returns dict(factor = executed / active routed pairs,
    executed_flops = 4 D G (Bc x executed pairs + Bc x tokens for the diagonal block))."""
    B, Hkv, T, W = words.shape
    pad = (-T) % tpt
    w = words
    if pad:
        w = torch.cat([w, torch.zeros(B, Hkv, pad, W, dtype=w.dtype, device=w.device)], 2)
    w = w.view(B, Hkv, (T + pad) // tpt, tpt, W)
    u = w[:, :, :, 0]
    for i in range(1, tpt):
        u = u | w[:, :, :, i]
    tok = torch.full(((T + pad) // tpt,), tpt, dtype=torch.float64, device=words.device)
    if pad:
        tok[-1] = tpt - pad
    union = (popcount_words(u) - 1).clamp_min(0).to(torch.float64)      # [B,Hkv,units]
    executed = float((union * tok).sum())
    active = float((popcount_words(words) - 1).clamp_min(0).to(torch.float64).sum())
    diag = float(B * Hkv * T) * chunk_size
    return dict(factor=executed / active if active > 0 else 1.0,
                executed_flops=4.0 * head_dim * G * (chunk_size * executed + diag),
                tokens_per_unit=tpt)


def stage01_bytes(cfg):
    """Algorithmic HBM bytes of Stages 0-1: K read, summaries written and read once, Q read
    once, mask words and tau written."""
    B, Hq, Hkv, T, D, Bc = (cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.seq_len, cfg.head_dim,
                            cfg.chunk_size)
    C = (T + Bc - 1) // Bc
    W = (C + 63) // 64
    k_bytes = B * Hkv * T * D * 2
    summ = B * Hkv * (T // Bc) * D * 4
    q_bytes = B * Hq * T * D * 2
    mask = B * Hkv * T * W * 8
    tau = B * Hkv * T * 4
    return dict(stage0=k_bytes + summ, stage1=q_bytes + summ + mask + tau)


def stage1_score_flops(cfg):
    """FLOPs of Stage 1's scores: qbar . summary_c (2 D) for every row and routable chunk
    c < c_t (the group mean and the entmax solve not counted)."""
    B, Hkv, T, D, Bc = cfg.batch, cfg.heads_kv, cfg.seq_len, cfg.head_dim, cfg.chunk_size
    Cf = T // Bc
    pairs = Bc * Cf * (Cf - 1) // 2 + (T - Cf * Bc) * Cf       # sum over t of floor(t / Bc)
    return 2.0 * D * B * Hkv * pairs


# FP32 FMA peak of the CUDA cores: 148 SMs x 128 FMA lanes x 2 FLOP x the maximum SM clock
# (1965 MHz); the Stage 1 scores run there (fp32 FMA chains in a fixed order).
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def max_over_ranks(x: float, device) -> float:
    """The maximum of x over the ranks of the default process group (x itself when there is
    none): every multi-rank time is the slowest rank's.  device is where the reduction runs
    (CUDA for NCCL, CPU for gloo)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank_step: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each processed `steps` steps of
    `tokens_per_rank_step` tokens in at most max_ms milliseconds."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def traffic_for(kernel, cfg_name):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        e = d[kernel][cfg_name]
        csrc = os.path.join(ROOT, "sparse_hierarchical_attention_stage0_b200", "csrc")
        blob = b"".join(open(os.path.join(csrc, n), "rb").read() for n in e["sources"])
        h = hashlib.sha256(blob).hexdigest()[:16]
        return e["bytes_per_launch"] if h == e["source_sha256_16"] else None
    except (OSError, ValueError, KeyError):
        return None


def timed(fn, steps, stream, flush=None):
    """Per-step device times (ms) with CUDA events on `stream`; flush runs between steps."""
    times = []
    for _ in range(steps):
        if flush is not None:
            flush()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    return times


def bench_backward(dash, q, k, v, hc, out, cfg, stream, flush, stats):
    """dash_backward (gradients w.r.t. q, k, v, head_cls of sum(out * dout) through the three
    stages) on the same inputs, L2 flushed before each call.  Algorithmic FLOPs: the five
    products of attention backward per attended (token, key, head) (S, dP, dQ, dK, dV:
    10 D) = 2.5 x the forward's active FLOPs; the routing backward is not counted."""
    dash.prefill(q, k, v, hc, cfg.chunk_size, cfg.alpha, cfg.gamma, enable_gqa=True, out=out)
    dout = torch.randn(q.shape, generator=torch.Generator(device=q.device).manual_seed(1),
                       device=q.device).to(torch.bfloat16)
    prm = dash.make_params(q.shape[0], q.shape[1], k.shape[1], q.shape[2], q.shape[3], cfg.chunk_size,
                           cfg.alpha, cfg.gamma, 1.0, True)
    ws = dash.workspace(dash.lib.dash_backward_workspace_size(ctypes.byref(prm)), q.device)

    def run():
        dash.backward(q, k, v, hc, out, dout, cfg.chunk_size, cfg.alpha, cfg.gamma, ws=ws)

    run()
    ms = statistics.mean(timed(run, 2, stream, flush))
    assert dash.read_device_status(ws) == 0
    flops = 2.5 * stats["active_flops"]
    del ws, dout
    torch.cuda.empty_cache()
    return {"ms": ms, "tflops": flops / (ms / 1e3) / 1e12, "algorithmic_flop": flops,
            "kernels": "k_stage0, k_route (with p), k_bwd_q, k_bwd_lists x2, k_bwd_scan, k_bwd_kv, "
                       "k_bwd_route, k_bwd_dsum, k_bwd_stage0 (warp-level MMA)",
            "note": "2.5 x the forward's active FLOPs (S, dP, dQ, dK, dV per attended pair)"}


# ------------------------------------------------------------------------------ decode
def graph_us(body, stream, reset=None, replays=3):
    """Median device time (us) of one replay of a CUDA graph of body(), timed with events on
    `stream`; reset() (outside the timing) restores the state body() mutates."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        if reset is not None:
            reset()
        body()                                        # warm-up outside the capture
        if reset is not None:
            reset()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            body()
    torch.cuda.synchronize()
    ts = []
    for _ in range(replays):
        with torch.cuda.stream(stream):
            if reset is not None:
                reset()
            st = torch.cuda.Event(enable_timing=True)
            en = torch.cuda.Event(enable_timing=True)
            st.record(stream)
            g.replay()                                # replay launches on the current stream
            en.record(stream)
        en.synchronize()
        ts.append(st.elapsed_time(en) * 1e3)
    del g
    return statistics.median(ts)


def bench_decode(dash, dev, steps_cap=256, warmup=3):
    """The decode workload: 256 steps of dash_decode_step (append the new K/V, route, attend,
    summarise a completed chunk, advance seq_lens: one launch per step), in one CUDA graph."""
    cfg = CONFIGS["decode64k"]
    t0 = time.time()
    d = make_decode(cfg)
    log(f"decode inputs drawn in {time.time() - t0:.1f}s")
    B, Hq, Hkv, D, Bc = cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.head_dim, cfg.chunk_size
    L0, S, cap = d["prefix_len"], min(d["steps"], steps_cap), d["capacity"]
    k_all = d["k_all"].to(dev)
    v_all = d["v_all"].to(dev)
    hc = d["head_cls"].to(dev)
    q_steps = d["q_steps"].to(dev)
    k_new = k_all[:, :, L0:L0 + S].permute(2, 0, 1, 3).contiguous()       # [S, B, Hkv, D]
    v_new = v_all[:, :, L0:L0 + S].permute(2, 0, 1, 3).contiguous()
    kc = torch.zeros_like(k_all)
    vc = torch.zeros_like(v_all)
    kc[:, :, :L0] = k_all[:, :, :L0]
    vc[:, :, :L0] = v_all[:, :, :L0]
    cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
    seq = torch.full((B,), L0, dtype=torch.int32, device=dev)
    dash.update_chunk_cache(kc, hc, seq, cache, Hq, Bc, n_recent=L0 // Bc)
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    prm = dash.make_params(B, Hq, Hkv, cap, D, Bc, cfg.alpha, enable_gqa=True)
    ws = torch.zeros(max(256, dash.lib.dash_decode_step_workspace_size(ctypes.byref(prm))),
                     dtype=torch.uint8, device=dev)             # zeroed before the first step

    def reset():
        seq.fill_(L0)

    def steps(masks=None, flush=None):
        for s in range(S):
            if flush is not None:
                flush()
            dash.decode_step(q_steps[s], k_new[s], v_new[s], kc, vc, seq, cache, hc, Bc, cfg.alpha,
                             out=out, ws=ws, active_blocks=None if masks is None else masks[s])

    # Routing of every step (untimed pass) for the algorithmic byte count.
    Wcap = ((cap + Bc - 1) // Bc + 63) // 64
    masks = torch.zeros(S, B, Hkv, Wcap, dtype=torch.int64, device=dev)
    reset()
    steps(masks)
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0
    assert int(seq.min()) == L0 + S
    act = (popcount_words(masks) - 1).to(torch.float64)          # routed active per (s,b,g)
    L = torch.arange(L0 + 1, L0 + S + 1, device=dev, dtype=torch.float64)
    t = L - 1
    ct = torch.floor(t / Bc)
    diag_keys = t - ct * Bc + 1                                  # [S]
    per_bg = (ct[:, None, None] * D * 4 + act * 2 * Bc * D * 2 + diag_keys[:, None, None] * 2 * D * 2
              + 2 * (Hq // Hkv) * D * 2)
    alg_bytes = float(per_bg.sum())
    visible = float(ct.sum() * B * Hkv)
    sparsity = 1.0 - float(act.sum()) / visible

    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    warm_us = graph_us(steps, stream, reset)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush = flush_buf.zero_
    cold_us = graph_us(lambda: steps(flush=flush), stream, reset) - graph_us(lambda: [flush() for _ in range(S)], stream)
    assert dash.read_device_status(ws) == 0
    ms = warm_us / 1e3
    paged_us = bench_decode_paged(dash, dev, d, cfg, S, k_new, v_new, stream)
    return dict(tokens_per_s=B * S / (ms / 1e3), ms_per_step=ms / S, steps=S, batch=B,
                paged={"ms_per_step": paged_us / 1e3 / S, "tokens_per_s": B * S / (paged_us / 1e6),
                       "layout": "pages of one chunk, scattered through the pools by a random "
                                 "block table"},
                cache_len=L0, realised_sparsity=sparsity,
                hbm_bytes_per_step=alg_bytes / S,
                achieved_gbs=alg_bytes / (ms / 1e3) / 1e9, launches=S,
                kernel=dict(us_l2_warm=warm_us / S, us_l2_cold=cold_us / S,
                            gbs_l2_cold=alg_bytes / (cold_us / 1e6) / 1e9,
                            note="cold: each step after a 256 MiB L2-flushing write, the graph "
                                 "of writes alone subtracted"),
                note="one dash_decode_step launch per step (append, route, attend, chunk "
                     "summary, length update); steps consecutive, L2 warm across them")


def bench_decode_paged(dash, dev, d, cfg, S, k_new, v_new, stream):
    """The same 256 steps on a paged cache (pages of one chunk, a random block table),
    captured in one graph; returns the median graph time in us."""
    B, Hq, Hkv, D, Bc = cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.head_dim, cfg.chunk_size
    L0, cap = d["prefix_len"], d["capacity"]
    nb = cap // Bc
    n_pages = B * nb
    gen = torch.Generator().manual_seed(11)
    table = torch.randperm(n_pages, generator=gen).view(B, nb).to(torch.int32).to(dev)
    k_all, v_all = d["k_all"].to(dev), d["v_all"].to(dev)
    hc, q_steps = d["head_cls"].to(dev), d["q_steps"].to(dev)
    # pool[table[b, c]] = chunk c of sequence b (positions >= L0 zero until appended)
    flat = table.view(-1).long()
    kp = torch.zeros(n_pages, Hkv, Bc, D, dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    src_k = k_all.clone()
    src_v = v_all.clone()
    src_k[:, :, L0:] = 0
    src_v[:, :, L0:] = 0
    kp[flat] = src_k.view(B, Hkv, nb, Bc, D).permute(0, 2, 1, 3, 4).reshape(n_pages, Hkv, Bc, D)
    vp[flat] = src_v.view(B, Hkv, nb, Bc, D).permute(0, 2, 1, 3, 4).reshape(n_pages, Hkv, Bc, D)
    sp = torch.zeros(n_pages, Hkv, D, device=dev)
    seq = torch.full((B,), L0, dtype=torch.int32, device=dev)
    dash.update_chunk_cache_paged(kp, hc, table, seq, sp, Hq, Bc, n_recent=L0 // Bc)
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    prm = dash.make_params(B, Hq, Hkv, cap, D, Bc, cfg.alpha, enable_gqa=True)
    ws = torch.zeros(max(256, dash.lib.dash_decode_step_workspace_size(ctypes.byref(prm))),
                     dtype=torch.uint8, device=dev)             # zeroed before the first step

    def steps():
        for s in range(S):
            dash.decode_step(q_steps[s], k_new[s], v_new[s], kp, vp, seq, sp, hc, Bc, cfg.alpha,
                             out=out, ws=ws, block_table=table)

    us = graph_us(steps, stream, lambda: seq.fill_(L0))
    assert dash.read_device_status(ws) == 0
    return us


# ------------------------------------------------------------------------------ oracle
def oracle_sample(cfg, q, k, v, hc, n_rows, seed=0):
    """Time the fp64 oracle on n_rows sampled rows (all heads) plus Stage 0 over every chunk;
    extrapolate linearly in rows to the workload's tokens/s."""
    import oracle
    q, k, v, hc = (oracle._f64(x) for x in (q, k, v, hc))     # widen outside the timing
    g = torch.Generator().manual_seed(seed)
    T = cfg.seq_len
    rows = torch.sort(torch.randint(0, T, (n_rows,), generator=g)).values.numpy()
    t0 = time.perf_counter()
    S = oracle.stage0(k, hc, cfg.chunk_size)
    t1 = time.perf_counter()
    p, m, tau = oracle.stage1(q, S, T, cfg.chunk_size, cfg.alpha, cfg.gamma, rows)
    oracle.stage2(q, k, v, p, cfg.chunk_size, 1.0, rows)
    t2 = time.perf_counter()
    total = (t1 - t0) + (t2 - t1) * T / n_rows
    return dict(value=cfg.batch * T / total, unit="tokens/s", cores=oracle.num_threads(),
                kind="oracle", seconds=t2 - t0,
                sample=f"Stage 0 over all {T // cfg.chunk_size} chunks per KV head + Stages 1-2 "
                       f"for {n_rows} uniformly sampled rows (all {cfg.heads_q} heads), "
                       f"extrapolated linearly to {T} rows")


def reference_decode_line(args):
    """The oracle's decode on the host cores: each step one decode of the 16 sequences at a
    sampled step of the workload (its summaries recomputed by the oracle, as decode does)."""
    import oracle
    cfg = CONFIGS["decode64k"]
    d = make_decode(cfg)
    k64, v64 = oracle._f64(d["k_all"]), oracle._f64(d["v_all"])
    times = []
    for i in range(args.warmup + args.steps):
        s = (37 * i) % d["steps"]
        L = d["prefix_len"] + s + 1
        t0 = time.perf_counter()
        oracle.decode(d["q_steps"][s], k64, v64, d["head_cls"], [L] * cfg.batch, cfg.chunk_size,
                      cfg.alpha)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    value = cfg.batch / statistics.median(times)
    sample = f"{args.steps} decode steps of all {cfg.batch} sequences (oracle recomputes summaries)"
    return {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / value * cfg.batch, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.batch, "cache_len": cfg.prefix_len},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dash", choices=["dash", "reference"])
    ap.add_argument("--workload", default="prefill128k",
                    choices=["prefill128k", "gqa32k", "tiny", "sweep", "decode64k"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--oracle-rows", type=int, default=0, help="0: pick by workload")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = workload_config({"sweep": "sweep64k", "decode64k": "gqa32k"}.get(args.workload, args.workload))
    n_rows = args.oracle_rows or {"prefill128k": 96, "gqa32k": 256, "tiny": 1024,
                                  "sweep": 32, "decode64k": 0}[args.workload]

    if args.impl == "reference" and args.workload == "decode64k":
        if rank == 0:
            print(json.dumps(reference_decode_line(args)), flush=True)
        return
    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        q, k, v, hc = (oracle._f64(x) for x in make_prefill(cfg))
        times = []
        for i in range(args.warmup + args.steps):
            r = oracle_sample(cfg, q, k, v, hc, max(8, n_rows // 4), seed=i)
            if i >= args.warmup:
                times.append(r)
        value = statistics.median(x["value"] for x in times)
        secs = sum(x["seconds"] for x in times)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": cfg.batch * cfg.seq_len / value * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded planted-evidence generator)",
                "config": {"workload": cfg.name, "batch": cfg.batch, "heads_q": cfg.heads_q,
                           "heads_kv": cfg.heads_kv, "seq_len": cfg.seq_len,
                           "head_dim": cfg.head_dim, "chunk_size": cfg.chunk_size,
                           "alpha": cfg.alpha, "gamma": cfg.gamma, "parallelism": "replicas"},
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": times[0]["cores"],
                                 "kind": "oracle", "sample": times[0]["sample"]},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "oracle_seconds": secs}
        print(json.dumps(line), flush=True)
        return

    import sparse_hierarchical_attention_stage0_b200 as dash
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    if args.workload == "sweep":
        line = bench_sweep(dash, args, dev, world, rank)
    elif args.workload == "decode64k":
        line = bench_decode_line(dash, args, dev, world)
    else:
        line = bench_prefill(dash, cfg, args, dev, world, rank, full=True)
        if not args.no_decode and args.workload == "prefill128k":
            torch.cuda.empty_cache()
            pk, _ = peaks()
            dec = bench_decode(dash, dev)
            kg = dec["kernel"]["gbs_l2_cold"]
            dec["roofline"] = {"bound": "hbm", "kernel": "k_decode (alone, L2 flushed before each launch)",
                               "achieved": kg, "peak": pk["hbm_gbs"], "unit": "GB/s",
                               "frac": kg / pk["hbm_gbs"],
                               "traffic": traffic_for("k_decode", "decode64k")}
            line["decode"] = dec
        if rank == 0 and world == 1:
            q_h, k_h, v_h, hc_h = make_prefill(cfg)
            line["cpu_baseline"] = oracle_sample(cfg, q_h, k_h, v_h, hc_h, n_rows)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_prefill(dash, cfg, args, dev, world, rank, full=True):
    """Time `args.steps` routed prefills of `cfg` (inputs resident in HBM, L2 flushed before
    each), the stages one by one, the dense path, and with full=True the end-to-end prefill
    from host buffers.  Returns the JSON line's fields (without decode and cpu_baseline)."""
    t0 = time.time()
    q_h, k_h, v_h, hc_h = make_prefill(cfg)
    log(f"[rank {rank}] {cfg.name}: inputs drawn in {time.time() - t0:.1f}s")
    q, k, v, hc = (x.to(dev) for x in (q_h, k_h, v_h, hc_h))
    B, Hq, Hkv, T, D, Bc = cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.seq_len, cfg.head_dim, cfg.chunk_size
    prm = dash.make_params(B, Hq, Hkv, T, D, Bc, cfg.alpha, cfg.gamma, 1.0, True)
    ws = dash.workspace(dash.prefill_workspace_size(prm), dev)
    out = torch.empty_like(q)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.zero_()                               # noqa: E731
    stream = torch.cuda.current_stream(dev)

    def prefill():
        dash.prefill(q, k, v, hc, Bc, cfg.alpha, cfg.gamma, enable_gqa=True, out=out, ws=ws)

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms = timed(prefill, args.steps, stream, flush)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(step_ms), dev)
    if world > 1:
        torch.distributed.barrier()
    value = job_tokens_per_s(world, B * T, args.steps, total_ms)

    # Per-stage times through the stage entry points (same kernels as dash_prefill).
    summ = torch.empty(B, Hkv, T // Bc, D, device=dev)
    C = (T + Bc - 1) // Bc
    W = (C + 63) // 64
    tau = torch.empty(B, Hkv, T, device=dev)
    mask = torch.empty(B, Hkv, T, W, dtype=torch.int64, device=dev)
    ws_s = dash.workspace(256, dev)
    ws_a = dash.workspace(dash.attend_workspace_size(prm), dev)
    import ctypes

    def run_route():
        dash._check(dash.lib.dash_route(ctypes.byref(prm), dash._ptr(q), dash._ptr(summ),
                                        dash._ptr(tau), None, dash._ptr(mask), dash._ptr(ws_s),
                                        256, dash._stream(dev)), "dash_route")

    st_ms = {"stage0": [], "stage1": [], "stage2": []}
    for i in range(args.warmup + args.steps):
        flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        dash.stage0(k, hc, Bc, ws=ws_s, summary=summ)
        ev[1].record(stream)
        run_route()
        ev[2].record(stream)
        dash.attend(q, k, v, summ, tau, mask, Bc, cfg.alpha, cfg.gamma, 1.0, True, ws=ws_a, out=out)
        ev[3].record(stream)
        ev[3].synchronize()
        if i >= args.warmup:
            for j, name in enumerate(("stage0", "stage1", "stage2")):
                st_ms[name].append(ev[j].elapsed_time(ev[j + 1]))
    stage = {k_: statistics.mean(v_) for k_, v_ in st_ms.items()}
    del mask, tau

    stats = active_stats(dash, q, k, v, hc, cfg)
    # The Stage 2 kernel dash_attend runs with the bench's workspace (the library names it);
    # the 128-key-block kernels also transpose V (timed together with them as Stage 2).
    s2_dispatch = dash.attend_kernel_name(prm, ws_a.numel())
    with_vt = s2_dispatch in ("k_attend_fa", "k_attend_pair", "k_attend_fa|k_attend")
    # Chosen at run time (fewer than 8 query heads per KV head): the kernel the timed calls ran.
    s2_kernel = (dash.stage2_kernel_ran(ws_a) or s2_dispatch) if "|" in s2_dispatch else s2_dispatch
    s2_note = ", V^T transpose included" if with_vt else ""
    # k_stage0, [k_route,] [k_vtranspose,] Stage 2: as the library reports for this workspace
    launches_per_step = dash.prefill_kernel_count(prm, ws.numel())
    un = union_stats(stats.pop("words"), Bc, D, cfg.group, tokens_per_tile(s2_kernel, cfg.group))

    def dense():
        dash.prefill(q, k, v, None, Bc, enable_gqa=True, dense=True, out=out, ws=ws)

    for _ in range(2):
        dense()
    dense_ms = statistics.mean(timed(dense, max(2, min(args.steps, 3)), stream, flush))
    dprm = dash.make_params(B, Hq, Hkv, T, D, Bc, enable_gqa=True, flags=1)
    dense_kernel = dash.attend_kernel_name(dprm, ws.numel())

    pk, pk_kind = peaks()
    s2_tflops = stats["active_flops"] / (stage["stage2"] / 1e3) / 1e12
    sb = stage01_bytes(cfg)
    s01_gbs = (sb["stage0"] + sb["stage1"]) / ((stage["stage0"] + stage["stage1"]) / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded planted-evidence generator, see dash_inputs)",
        "config": {"workload": cfg.name, "batch": B, "heads_q": Hq, "heads_kv": Hkv,
                   "seq_len": T, "head_dim": D, "chunk_size": Bc, "alpha": cfg.alpha,
                   "gamma": cfg.gamma, "parallelism": f"replicas x{world}",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "active_tflops": s2_tflops,
        "realised_sparsity": stats["sparsity"],
        "support": stats.pop("support"),
        "stage_ms": stage,
        "stage01_gbs": s01_gbs,
        "dense_ms": dense_ms,
        "dense_kernel": dense_kernel,
        "dense_tflops": stats["dense_flops"] / (dense_ms / 1e3) / 1e12,
        "speedup_vs_dense": dense_ms / (total_ms / args.steps),
        "union": {"kernel": s2_kernel, "tokens_per_unit": un["tokens_per_unit"],
                  "factor": un["factor"],
                  "executed_tflops": un["executed_flops"] / (stage["stage2"] / 1e3) / 1e12,
                  "note": "executed / active routed token-chunk pairs: each work unit walks "
                          "the union of its tokens' chunks"},
        "roofline": {"bound": "tensor", "kernel": f"{s2_kernel} (Stage 2{s2_note})",
                     "achieved": s2_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": s2_tflops / pk["bf16_tflops"],
                     "traffic": traffic_for(s2_kernel, cfg.name),
                     "peak_source": f"{pk_kind} bf16 burst",
                     "algorithmic": f"{stats['active_flops']:.4e} active FLOP per launch"},
        "roofline_stage01": {"bound": "hbm", "achieved": s01_gbs, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": s01_gbs / pk["hbm_gbs"],
                             "frac_of_8tbs_nominal": s01_gbs / 8000.0,
                             "bytes": sb["stage0"] + sb["stage1"]},
        "roofline_stage1_alu": {"bound": "alu",
                                "achieved": stage1_score_flops(cfg) / (stage["stage1"] / 1e3) / 1e12,
                                "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                                "frac": stage1_score_flops(cfg) / (stage["stage1"] / 1e3) / 1e12 / FP32_PEAK_TFLOPS,
                                "note": "Stage 1's score FLOPs (2 D per row and routable chunk) over its "
                                        "time through dash_route, against the fp32 FMA peak of the CUDA "
                                        "cores (148 SMs x 128 lanes x 2 x 1965 MHz)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if full:
        # The routing variants, each timed as the main prefill (L2 flushed before each step):
        # top-k routing at the entmax's mean active-chunk count (equal sparsity), and the
        # estimated diagonal.
        k_eq = max(1, int(round(stats["active_chunks"] / (B * Hkv * T))))
        variants = {}
        for name, kw in (("topk", dict(topk=k_eq)), ("estimate_diagonal", dict(estimate_diagonal=True))):
            def run_variant(kw=kw):
                dash.prefill(q, k, v, hc, Bc, cfg.alpha, cfg.gamma, enable_gqa=True, out=out,
                             ws=ws, **kw)
            for _ in range(2):
                run_variant()
            vms = statistics.mean(timed(run_variant, max(2, min(args.steps, 3)), stream, flush))
            variants[name] = {"ms_per_step": vms, "tokens_per_s": B * T / (vms / 1e3), **kw}
        torch.cuda.synchronize()
        assert dash.read_device_status(ws) == 0
        line["routing_variants"] = variants
        line["backward"] = bench_backward(dash, q, k, v, hc, out, cfg, stream, flush, stats)
        # End to end through host buffers: dash_prefill_host copies q, k, v, head_cls from
        # pinned host memory and out back, in row slices overlapped with the computation.
        hq, hk, hv, hhc = (x.pin_memory() for x in (q_h, k_h, v_h, hc_h))
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e():
            dash.prefill_host(hq, hk, hv, hhc, ho, q, k, v, hc, out, Bc, cfg.alpha, cfg.gamma,
                              enable_gqa=True, n_slices=E2E_SLICES, ws=ws)

        e2e()
        if world > 1:
            torch.distributed.barrier()
        e2e_ms = max_over_ranks(statistics.mean(timed(e2e, args.steps, stream, flush)), dev)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hhc))
        d2h = ho.numel() * ho.element_size()
        line["e2e"] = {"value": job_tokens_per_s(world, B * T, 1, e2e_ms), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                       "call": f"dash_prefill_host, {E2E_SLICES} row slices"}
        del hq, hk, hv, ho
    del q, k, v, out, ws, flush_buf, ws_a
    torch.cuda.empty_cache()
    return line


DECODE_METRIC = "decode tok/s (16 sequences x 64K cached tokens, 256 steps in one CUDA graph)"


def bench_decode_line(dash, args, dev, world):
    """The decode workload alone as the JSON line (value = decode tokens/s over all ranks)."""
    pk, pk_kind = peaks()
    with ClockSampler(torch.cuda.current_device()) as clk:
        dec = bench_decode(dash, dev)
    ms = max_over_ranks(dec["ms_per_step"] * dec["steps"], dev)
    cfg = CONFIGS["decode64k"]
    return {"metric": DECODE_METRIC, "value": world * dec["batch"] * dec["steps"] / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": dec["steps"], "warmup": 3,
            "ms_per_step": ms / dec["steps"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded planted-evidence generator, see dash_inputs)",
            "config": {"workload": cfg.name, "batch": cfg.batch, "heads_q": cfg.heads_q,
                       "heads_kv": cfg.heads_kv, "cache_len": cfg.prefix_len, "steps": cfg.steps,
                       "head_dim": cfg.head_dim, "chunk_size": cfg.chunk_size, "alpha": cfg.alpha,
                       "parallelism": f"replicas x{world}",
                       "l2": "not flushed between steps (one graph of 256 steps)"},
            "roofline": {"bound": "hbm", "kernel": "k_decode (alone, L2 flushed before each launch)",
                         "achieved": dec["kernel"]["gbs_l2_cold"],
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": dec["kernel"]["gbs_l2_cold"] / pk["hbm_gbs"],
                         "traffic": traffic_for("k_decode", "decode64k"),
                         "peak_source": f"{pk_kind} copy bandwidth",
                         "algorithmic": f"{dec['hbm_bytes_per_step']:.4e} bytes per launch"},
            "decode": dec, "gpu_launches": dec["launches"], "clocks": clk.summary()}


SWEEP_METRIC = ("sweep at 64K (B=2, H_kv=8): prefill tokens/s over the alpha x chunk_size "
                "cells; per cell active TFLOP/s, sparsity, Stage 0-1 GB/s, speedup vs dense")


def bench_sweep(dash, args, dev, world, rank):
    """The six alpha x chunk_size cells of the 64K sweep, each timed as bench_prefill does
    (without the host-memory leg); value = all cells' tokens over their summed step times."""
    from dash_inputs import SWEEP_ALPHAS, SWEEP_CHUNKS, sweep_config
    cells, tokens, ms = [], 0, 0.0
    for i in range(len(SWEEP_ALPHAS) * len(SWEEP_CHUNKS)):
        cfg = sweep_config(i)
        r = bench_prefill(dash, cfg, args, dev, world, rank, full=False)
        cells.append({"alpha": cfg.alpha, "chunk_size": cfg.chunk_size, "ms_per_step": r["ms_per_step"],
                      "tokens_per_s": r["value"], "active_tflops": r["active_tflops"],
                      "realised_sparsity": r["realised_sparsity"], "support": r["support"],
                      "stage_ms": r["stage_ms"],
                      "stage01_gbs": r["stage01_gbs"], "dense_ms": r["dense_ms"],
                      "dense_kernel": r["dense_kernel"], "speedup_vs_dense": r["speedup_vs_dense"],
                      "union": r["union"], "stage2_kernel": r["union"]["kernel"],
                      "gpu_launches": r["gpu_launches"], "clocks": r["clocks"]})
        tokens += cfg.batch * cfg.seq_len * args.steps * world
        ms += r["ms_per_step"] * args.steps
    cfg0 = sweep_config(0)
    return {"metric": SWEEP_METRIC, "value": tokens / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded planted-evidence generator, see dash_inputs)",
            "config": {"workload": "sweep64k", "batch": cfg0.batch, "heads_q": cfg0.heads_q,
                       "heads_kv": cfg0.heads_kv, "seq_len": cfg0.seq_len,
                       "head_dim": cfg0.head_dim, "alphas": list(SWEEP_ALPHAS),
                       "chunk_sizes": list(SWEEP_CHUNKS), "parallelism": f"replicas x{world}",
                       "l2": "flushed (256 MiB write) before every timed step"},
            "gpu_launches": sum(c["gpu_launches"] for c in cells),
            "cells": cells}


if __name__ == "__main__":
    main()
