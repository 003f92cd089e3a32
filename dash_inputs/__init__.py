"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the attention method itself: it only draws tensors.
Everything is drawn on the CPU from one ``torch.Generator`` per call, in a fixed order
(K, V, query noise z, head_cls, evidence counts, evidence indices) and rounded to bf16 last.

Planted-evidence queries (the long-context workloads): for every token t whose own chunk
c_t = t // chunk_size is at least 1, draw a count n_t uniform in {1..n_max} (clipped to c_t)
and a set E_t of n_t distinct earlier chunks, uniform without replacement from [0, c_t).
Every query head of KV group g then gets  q = z + scale * sqrt(D) * u_g,  where u_g is the
unit vector along the sum of the mean keys of the chunks in E_t (group g's keys).  The
evidence set is per token and shared by all heads of that token, so the routing support
varies per query.  These synthetic tensors stand in for the long-context benchmark suites
the pages evaluate on (RULER, HELMET), which need trained models; only the context lengths
and sparsity levels are taken from them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["PrefillConfig", "DecodeConfig", "CONFIGS", "make_prefill", "make_decode",
           "sample_rows"]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seq_len: int
    head_dim: int
    chunk_size: int
    alpha: float
    gamma: float = 1.0
    planted: bool = False
    n_max: int = 24
    scale: float = 3.0
    seed: int = 0

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    prefix_len: int
    steps: int
    head_dim: int
    chunk_size: int
    alpha: float
    gamma: float = 1.0
    n_max: int = 24
    scale: float = 3.0
    seed: int = 3

    @property
    def capacity(self) -> int:
        return self.prefix_len + self.steps


# The five workloads.  gamma of the 128K config is calibrated by
# tests/golden/calibrate_gamma.py (oracle only) and read back from tests/golden.
CONFIGS = {
    "tiny": PrefillConfig("tiny", 1, 4, 4, 1024, 64, 64, 1.5, seed=0),
    "gqa32k": PrefillConfig("gqa32k", 1, 32, 2, 32768, 128, 64, 1.5, planted=True, n_max=24,
                            seed=1),
    "prefill128k": PrefillConfig("prefill128k", 1, 32, 2, 131072, 128, 64, 1.5, planted=True,
                                 n_max=24, seed=2),
    "decode64k": DecodeConfig("decode64k", 16, 32, 2, 65536, 256, 128, 64, 1.5, n_max=24,
                              seed=3),
}
SWEEP_ALPHAS = (1.25, 1.5, 2.0)
SWEEP_CHUNKS = (64, 128)


def sweep_config(index: int) -> PrefillConfig:
    """Cell `index` (0..5) of the alpha x chunk_size sweep at 64K, B=2, Hq=32, Hkv=8."""
    a = SWEEP_ALPHAS[index // len(SWEEP_CHUNKS)]
    bc = SWEEP_CHUNKS[index % len(SWEEP_CHUNKS)]
    return PrefillConfig(f"sweep64k_a{a}_c{bc}", 2, 32, 8, 65536, 128, bc, a, planted=True,
                         n_max=32, seed=4 + index)


SWEEP_DENSE_SEED = 10


def _evidence(gen: torch.Generator, mu: torch.Tensor, tokens: torch.Tensor, chunk_size: int,
              n_max: int, counts: torch.Tensor, block: int = 2048) -> torch.Tensor:
    """Unit evidence directions u [len(tokens), Hkv, D] for the given tokens.

    mu: [Hkv, Cf, D] fp32 chunk-mean keys.  counts: [len(tokens)] already clipped."""
    Hkv, Cf, D = mu.shape
    out = torch.empty(tokens.numel(), Hkv, D, dtype=torch.float32)
    kmax = min(n_max, Cf) if Cf > 0 else 0
    for s in range(0, tokens.numel(), block):
        tt = tokens[s:s + block]
        nb = tt.numel()
        ct = (tt // chunk_size).clamp(max=Cf)
        ncols = int(ct.max().item())
        keys = torch.rand(nb, ncols, generator=gen)
        col = torch.arange(ncols).unsqueeze(0)
        keys = torch.where(col < ct.unsqueeze(1), keys, torch.full_like(keys, 2.0))
        kk = min(kmax, ncols)
        idx = torch.topk(keys, kk, dim=1, largest=False, sorted=True).indices  # [nb, kk]
        take = torch.arange(kk).unsqueeze(0) < counts[s:s + block].unsqueeze(1)  # [nb, kk]
        g = mu[:, idx]                                        # [Hkv, nb, kk, D]
        g = (g * take.unsqueeze(0).unsqueeze(-1)).sum(2)      # [Hkv, nb, D]
        g = g / g.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        out[s:s + nb] = g.permute(1, 0, 2)
    return out


def make_prefill(cfg: PrefillConfig, seed: int | None = None, seq_len: int | None = None,
                 batch: int | None = None):
    """Draw (q, k, v, head_cls) for a prefill workload.

    Returns CPU tensors: q [B,Hq,T,D] bf16, k/v [B,Hkv,T,D] bf16, head_cls [Hkv,D] fp32."""
    if seq_len is not None or batch is not None:
        cfg = replace(cfg, seq_len=seq_len or cfg.seq_len, batch=batch or cfg.batch)
    seed = cfg.seed if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, T, D, Bc = (cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.seq_len, cfg.head_dim,
                            cfg.chunk_size)
    G = Hq // Hkv
    k = torch.randn(B, Hkv, T, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, D, generator=gen).to(torch.bfloat16)
    z = torch.randn(B, Hq, T, D, generator=gen)
    head_cls = torch.randn(Hkv, D, generator=gen)
    if cfg.planted and T > Bc:
        Cf = T // Bc
        tokens = torch.arange(Bc, T)
        for b in range(B):
            counts = torch.randint(1, cfg.n_max + 1, (tokens.numel(),), generator=gen)
            counts = torch.minimum(counts, (tokens // Bc).clamp(max=Cf))
            mu = k[b, :, :Cf * Bc].float().view(Hkv, Cf, Bc, D).mean(2)
            u = _evidence(gen, mu, tokens, Bc, cfg.n_max, counts)      # [n, Hkv, D]
            add = cfg.scale * math.sqrt(D) * u                          # [n, Hkv, D]
            add = add.repeat_interleave(G, dim=1).permute(1, 0, 2)      # [Hq, n, D]
            z[b, :, Bc:] += add
    q = z.to(torch.bfloat16)
    return q, k, v, head_cls


def make_decode(cfg: DecodeConfig, seed: int | None = None, steps: int | None = None,
                prefix_len: int | None = None, batch: int | None = None):
    """Draw a decode workload.

    Returns dict with k_all, v_all [B,Hkv,cap,D] bf16 (positions < prefix_len are the
    pre-filled cache, position prefix_len+s is the token appended at step s), q_steps
    [steps,B,Hq,D] bf16 (planted over the complete chunks before each step's own chunk),
    head_cls [Hkv,D] fp32, and the integer sizes."""
    if steps is not None or prefix_len is not None or batch is not None:
        cfg = replace(cfg, steps=steps or cfg.steps, prefix_len=prefix_len or cfg.prefix_len,
                      batch=batch or cfg.batch)
    seed = cfg.seed if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, D, Bc = cfg.batch, cfg.heads_q, cfg.heads_kv, cfg.head_dim, cfg.chunk_size
    G = Hq // Hkv
    cap = cfg.capacity
    k_all = torch.randn(B, Hkv, cap, D, generator=gen).to(torch.bfloat16)
    v_all = torch.randn(B, Hkv, cap, D, generator=gen).to(torch.bfloat16)
    z = torch.randn(cfg.steps, B, Hq, D, generator=gen)
    head_cls = torch.randn(Hkv, D, generator=gen)
    tokens = torch.arange(cfg.prefix_len, cap)                 # t of step s = prefix_len + s
    for b in range(B):
        Cf = cap // Bc
        counts = torch.randint(1, cfg.n_max + 1, (cfg.steps,), generator=gen)
        counts = torch.minimum(counts, (tokens // Bc).clamp(max=Cf))
        mu = k_all[b, :, :Cf * Bc].float().view(Hkv, Cf, Bc, D).mean(2)
        u = _evidence(gen, mu, tokens, Bc, cfg.n_max, counts)           # [steps, Hkv, D]
        add = cfg.scale * math.sqrt(D) * u.repeat_interleave(G, dim=1)  # [steps, Hq, D]
        z[:, b] += add
    return dict(k_all=k_all, v_all=v_all, q_steps=z.to(torch.bfloat16), head_cls=head_cls,
                prefix_len=cfg.prefix_len, steps=cfg.steps, capacity=cap)


def sample_rows(seq_len: int, chunk_size: int, seed: int, n_random: int = 512) -> torch.Tensor:
    """Row set R for sampled output checks: rows 0-63, 64 rows at random chunk starts and
    ends, the last 64 rows, and n_random uniform rows (drawn from seed + 100); sorted, unique."""
    gen = torch.Generator().manual_seed(seed + 100)
    T, Bc = seq_len, chunk_size
    C = (T + Bc - 1) // Bc
    parts = [torch.arange(min(64, T)), torch.arange(max(0, T - 64), T)]
    cs = torch.randint(0, C, (32,), generator=gen)
    parts += [(cs * Bc).clamp(max=T - 1), (cs * Bc + Bc - 1).clamp(max=T - 1)]
    parts.append(torch.randint(0, T, (n_random,), generator=gen))
    return torch.unique(torch.cat(parts)).to(torch.int64)
