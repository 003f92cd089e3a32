"""Calibrate the Stage 1 factor gamma of the 128K prefill workload (oracle only).

The pages tune the Stage 1 factor to reach a target sparsity (liuzhao09.github.io
"DashAttention 精读", section 4: the method matches the baselines' ~75% sparsity through the
Stage 1 factor; aixai.ru "DashAttention ...", FAQ: gamma is chosen for the target sparsity).
This script draws the 128K workload, builds the oracle's fp64 chunk summaries, and bisects
log(gamma) on [1e-3, 1e3] until the oracle's block-weighted sparsity over 4096 sampled rows
per KV group is 0.75 +- 0.02.  Sparsity = 1 - (active routed chunks) / (visible routed
chunks), summed over the sampled rows.  It writes gamma_prefill128k.json beside itself.

    python tests/golden/calibrate_gamma.py
"""
import json
import math
import os
import sys
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from dash_inputs import CONFIGS, make_prefill  # noqa: E402

TARGET, TOL, ROWS, SEED = 0.75, 0.02, 4096, 1234


def sparsity(Q, S, T, Bc, alpha, gamma, rows):
    p, m, tau = oracle.stage1(Q, S, T, Bc, alpha, gamma, rows)
    ct = rows // Bc
    visible = ct.sum() * p.shape[0] * p.shape[1]
    active = (p > 0).sum()
    return 1.0 - active / visible


def main():
    cfg = CONFIGS["prefill128k"]
    t0 = time.time()
    q, k, v, hc = make_prefill(cfg)
    Q = q.double().numpy()
    S = oracle.stage0(k, hc, cfg.chunk_size)
    print(f"inputs + summaries in {time.time() - t0:.1f}s", flush=True)
    rng = np.random.default_rng(SEED)
    rows = np.sort(rng.integers(cfg.chunk_size, cfg.seq_len, ROWS)).astype(np.int64)
    lo, hi = math.log(1e-3), math.log(1e3)
    g, s = 1.0, None
    for it in range(40):
        mid = 0.5 * (lo + hi)
        g = math.exp(mid)
        s = sparsity(Q, S, cfg.seq_len, cfg.chunk_size, cfg.alpha, g, rows)
        print(f"iter {it}: gamma {g:.6g} sparsity {s:.4f}", flush=True)
        if abs(s - TARGET) <= TOL / 4:
            break
        if s < TARGET:
            lo = mid          # support shrinks as gamma grows
        else:
            hi = mid
    assert abs(s - TARGET) <= TOL, s
    out = {"gamma": float(np.float32(g)), "oracle_sparsity_on_sample": float(s),
           "target": TARGET, "tolerance": TOL, "rows_per_group": ROWS, "row_seed": SEED,
           "workload": cfg.name, "alpha": cfg.alpha, "chunk_size": cfg.chunk_size,
           "written_by": "tests/golden/calibrate_gamma.py (oracle only)"}
    with open(os.path.join(HERE, "gamma_prefill128k.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
