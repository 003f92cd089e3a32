"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped 1/sqrt(D), a wrong
sign or index, a transposed operand, a wrong support rule, a mishandled diagonal) fails at
least one test:
  * hand-derived examples (tests/golden/hand_examples.json);
  * closed forms and library routines: torch SDPA in float64 for Stage 0 and for dense
    causal attention, scipy softmax for the alpha -> 1 limit;
  * brute force over all supports for tiny entmax problems;
  * variational optimality: entmax maximises p.s + Tsallis entropy; the prior softmax
    maximises z.w - KL(w || g) (gist.science "DashAttention ...", Technische
    Zusammenfassung, "Stufe 2", variational formulation);
  * invariants: sum to one, KKT, masked chunks contribute exactly nothing, decode == prefill.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from dash_inputs import CONFIGS, make_prefill

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
RNG = np.random.default_rng(12345)


# ----------------------------------------------------------------------------- entmax
@pytest.mark.parametrize("case", json.load(open(GOLD))["entmax"], ids=lambda c: str(c["s"]))
def test_entmax_hand_examples(case):
    p, tau = oracle.entmax(np.array(case["s"]), case["alpha"])
    np.testing.assert_allclose(p, case["p"], atol=1e-13)
    assert abs(tau - case["tau"]) < 1e-13


@pytest.mark.parametrize("alpha", [1.0, 1.25, 1.5, 1.75, 2.0, 2.5])
@pytest.mark.parametrize("n", [1, 2, 7, 64, 1000])
def test_entmax_sums_to_one_and_kkt(alpha, n):
    s = RNG.normal(size=n) * 3
    p, tau = oracle.entmax(s, alpha)
    assert abs(p.sum() - 1.0) < 1e-12
    assert (p >= 0).all()
    if alpha > 1:
        x = (alpha - 1) * s
        sup = p > 0
        # on the support p^(alpha-1) = x - tau; off it x <= tau
        np.testing.assert_allclose(p[sup] ** (alpha - 1), x[sup] - tau, rtol=1e-9, atol=1e-12)
        assert (x[~sup] <= tau + 1e-12).all()


def _brute_force(s, alpha):
    """Enumerate every support S, solve sum_{S}(x - tau)^beta = 1 in closed form (beta = 2 or
    1), keep the self-consistent S (x > tau on S, x <= tau off S)."""
    x = (alpha - 1) * np.asarray(s, dtype=np.float64)
    n = x.size
    found = []
    for k in range(1, n + 1):
        for S in itertools.combinations(range(n), k):
            xs = x[list(S)]
            if alpha == 2.0:
                tau = (xs.sum() - 1) / k
            else:  # alpha == 1.5: k tau^2 - 2 tau sum + sum sq - 1 = 0, smaller root
                a, b, c = k, -2 * xs.sum(), (xs ** 2).sum() - 1
                disc = b * b - 4 * a * c
                if disc < 0:
                    continue
                tau = (-b - math.sqrt(disc)) / (2 * a)
            inside = np.zeros(n, bool)
            inside[list(S)] = True
            if (x[inside] > tau).all() and (x[~inside] <= tau).all():
                found.append(tau)
    assert len(found) == 1, found          # the problem is strictly convex: one solution
    tau = found[0]
    beta = 1 / (alpha - 1)
    return np.where(x > tau, np.maximum(x - tau, 0) ** beta, 0.0), tau


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("trial", range(12))
def test_entmax_brute_force(alpha, trial):
    n = 2 + trial % 10
    s = RNG.normal(size=n) * (0.5 + trial)
    pb, tb = _brute_force(s, alpha)
    for method in ("auto", "bisect"):
        p, tau = oracle.entmax(s, alpha, method=method)
        np.testing.assert_allclose(p, pb, atol=1e-12)
        assert abs(tau - tb) < 1e-12


@pytest.mark.parametrize("n", [3, 50, 2047])
def test_sort_algorithms_agree_with_bisection(n):
    s = RNG.normal(size=n) * 2
    for alpha, method in ((1.5, "sort15"), (2.0, "sparsemax")):
        p1, t1 = oracle.entmax(s, alpha, method=method)
        p2, t2 = oracle.entmax(s, alpha, method="bisect")
        np.testing.assert_allclose(p1, p2, atol=1e-12)
        assert abs(t1 - t2) < 1e-12


def _tsallis_objective(p, s, alpha):
    return p @ s + (p - p ** alpha).sum() / (alpha * (alpha - 1))


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
def test_entmax_is_the_tsallis_maximiser(alpha):
    """alpha-entmax(s) = argmax over the simplex of p.s + (1/(alpha(alpha-1))) sum(p - p^alpha)
    (Peters, Niculae & Martins 2019); no feasible perturbation may do better."""
    s = RNG.normal(size=9) * 2
    p, _ = oracle.entmax(s, alpha)
    f0 = _tsallis_objective(p, s, alpha)
    for _ in range(2000):
        y = p + RNG.normal(size=9) * RNG.choice([1e-3, 1e-2, 1e-1])
        y = np.maximum(y, 0)
        y /= y.sum()
        assert _tsallis_objective(y, s, alpha) <= f0 + 1e-12
    for _ in range(500):
        y = RNG.dirichlet(np.ones(9))
        assert _tsallis_objective(y, s, alpha) <= f0 + 1e-12


def test_alpha_to_one_is_softmax():
    from scipy.special import softmax
    s = RNG.normal(size=40) * 2
    p, _ = oracle.entmax(s, 1.0 + 1e-6, method="bisect")
    np.testing.assert_allclose(p, softmax(s), atol=2e-5)
    p1, lse = oracle.entmax(s, 1.0)
    np.testing.assert_allclose(p1, softmax(s), atol=1e-14)
    assert abs(lse - np.log(np.exp(s).sum())) < 1e-12


def test_sparsemax_is_the_simplex_projection():
    """sparsemax(s) is the Euclidean projection of s on the simplex: (s - p).(y - p) <= 0."""
    s = RNG.normal(size=12)
    p, _ = oracle.entmax(s, 2.0)
    for _ in range(1000):
        y = RNG.dirichlet(np.ones(12) * 0.3)
        assert (s - p) @ (y - p) <= 1e-12


def test_support_shrinks_with_gamma():
    s = RNG.normal(size=300)
    for alpha in (1.5, 2.0):
        sizes = [int((oracle.entmax(g * s, alpha)[0] > 0).sum())
                 for g in np.geomspace(0.05, 50, 40)]
        assert all(a >= b for a, b in zip(sizes, sizes[1:])), sizes


# ----------------------------------------------------------------------------- stage 0
def _tiny_kv(B=2, Hkv=3, T=200, D=16, seed=0):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    hc = torch.randn(Hkv, D, generator=g, dtype=torch.float64)
    return K, hc


def test_stage0_zero_query_is_mean_pooling():
    K, hc = _tiny_kv()
    S = oracle.stage0(K, torch.zeros_like(hc), 16)
    ref = K[:, :, :192].reshape(2, 3, 12, 16, 16).mean(3).numpy()
    np.testing.assert_allclose(S, ref, atol=1e-14)


def test_stage0_is_single_query_sdpa():
    import torch.nn.functional as F
    K, hc = _tiny_kv()
    Bc = 16
    S = oracle.stage0(K, hc, Bc)
    Kc = K[:, :, :192].reshape(2, 3, 12, Bc, 16)                  # [B,H,C,Bc,D]
    q = hc.view(1, 3, 1, 1, 16).expand(2, 3, 12, 1, 16)
    ref = F.scaled_dot_product_attention(q, Kc, Kc)                # scale 1/sqrt(D)
    np.testing.assert_allclose(S, ref.squeeze(3).numpy(), atol=1e-13)


def test_stage0_dominant_query_picks_argmax_key():
    K, _ = _tiny_kv(D=8)
    hc = torch.zeros(3, 8, dtype=torch.float64)
    hc[:, 5] = 1e9            # logit gaps of 1e9/sqrt(8) * (key gap): one key wins
    S = oracle.stage0(K, hc, 20)
    Kc = K[:, :, :200].reshape(2, 3, 10, 20, 8)
    idx = Kc[..., 5].argmax(-1)
    ref = torch.gather(Kc, 3, idx[..., None, None].expand(2, 3, 10, 1, 8)).squeeze(3)
    np.testing.assert_allclose(S, ref.numpy(), atol=1e-9)


# ----------------------------------------------------------------------------- stage 1
def test_stage1_single_visible_chunk_has_p_one_and_small_rows_route_nothing():
    q, k, v, hc = make_prefill(CONFIGS["tiny"], seq_len=256)
    S = oracle.stage0(k, hc, 64)
    p, m, tau = oracle.stage1(q, S, 256, 64, 1.5)
    assert (p[:, :, :64] == 0).all() and np.isnan(tau[:, :, :64]).all()
    np.testing.assert_allclose(p[:, :, 64:128, 0], 1.0, atol=1e-15)
    assert (p[:, :, 64:128, 1:] == 0).all()
    np.testing.assert_allclose(p[:, :, 128:].sum(-1), 1.0, atol=1e-12)


def test_stage1_gqa_mean_query_equals_mean_scores():
    """GQA: the G heads' scores averaged = scores of the mean query; alpha = 1 exposes the
    scores as log p + lse."""
    q, k, v, hc = make_prefill(CONFIGS["tiny"], seq_len=320)
    q = q.double()
    qg = q.view(1, 2, 2, 320, 64)                       # 4 query heads, 2 KV heads, G = 2
    S = oracle.stage0(k[:, :2], hc[:2], 64)
    p, m, lse = oracle.stage1(q, S, 320, 64, 1.0)
    scores = torch.einsum("bghtd,bgcd->bghtc", qg, torch.from_numpy(S)) / 8.0
    mean_sc = scores.mean(2).numpy()                    # [B,Hkv,T,Cf]
    for t in range(64, 320):
        ct = t // 64
        np.testing.assert_allclose(np.log(p[0, :, t, :ct]) + lse[0, :, t, None],
                                   mean_sc[0, :, t, :ct], atol=1e-12)


@pytest.mark.parametrize("gamma", [0.2329096645116806, 3.0])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_stage1_gamma_scales_the_scores_before_entmax(alpha, gamma):
    """gist.science summary, "Stufe 1": the routing weights are alpha-entmax(gamma z).  The
    scores z are computed here independently of the oracle (mean query of the KV group,
    einsum against the summaries, 1/sqrt(D)); oracle.stage1 with gamma must give, row by
    row, the tau and p of oracle.entmax(gamma z) (pinned on its own) and the margins
    m = (alpha-1) gamma z - tau.  The first gamma is the one the 128K workload runs at."""
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=1024 + 37)
    T, D, Bc = q.shape[2], q.shape[3], 64
    S = oracle.stage0(k, hc, Bc)
    qbar = q.double().view(1, 2, 16, T, D).mean(2)                    # [B,Hkv,T,D]
    z = torch.einsum("bgtd,bgcd->bgtc", qbar, torch.from_numpy(S)).numpy() / math.sqrt(D)
    rows = np.array([64, 65, 127, 128, 300, 640, 1000, T - 1])
    p, m, tau = oracle.stage1(q, S, T, Bc, alpha, gamma=gamma, rows=rows)
    for g in range(2):
        for i, t in enumerate(rows):
            ct = t // Bc
            pr, tr = oracle.entmax(gamma * z[0, g, t, :ct], alpha)
            np.testing.assert_allclose(p[0, g, i, :ct], pr, atol=1e-12)
            assert (p[0, g, i, ct:] == 0).all()
            assert abs(tau[0, g, i] - tr) < 1e-12
            np.testing.assert_allclose(m[0, g, i, :ct], (alpha - 1) * gamma * z[0, g, t, :ct] - tr,
                                       atol=1e-12)
    # The pin bites: the gamma = 1 routing differs from the gamma routing on these rows.
    p1, _, _ = oracle.stage1(q, S, T, Bc, alpha, gamma=1.0, rows=rows)
    assert np.abs(p1 - p).max() > 1e-3


def test_stage1_margin_sign_is_the_support():
    cfg = CONFIGS["gqa32k"]
    q, k, v, hc = make_prefill(cfg, seq_len=2048 + 37)
    S = oracle.stage0(k, hc, 64)
    p, m, tau = oracle.stage1(q, S, q.shape[2], 64, 1.5)
    T = q.shape[2]
    ct = np.arange(T) // 64
    vis = np.arange(p.shape[-1])[None, :] < ct[:, None]
    assert ((m[0] > 0) == (p[0] > 0))[:, vis].all()
    assert (p[0][:, ~vis] == 0).all()
    rows = ct >= 1
    np.testing.assert_allclose(p[0][:, rows].sum(-1), 1.0, atol=1e-12)


# ----------------------------------------------------------------------------- stage 2
@pytest.mark.parametrize("case", json.load(open(GOLD))["attention"], ids=lambda c: str(c["p"]))
def test_stage2_hand_examples(case):
    Q = torch.ones(1, 1, 3, 1, dtype=torch.float64)
    K = torch.zeros(1, 1, 3, 1, dtype=torch.float64)
    V = torch.tensor([8.0, 0.0, 2.0], dtype=torch.float64).view(1, 1, 3, 1)
    p = np.zeros((1, 1, 1, 3))
    p[0, 0, 0, :2] = case["p"]
    O = oracle.stage2(Q, K, V, p, chunk_size=1, rows=[2])
    assert abs(O[0, 0, 0, 0] - case["O"]) < 1e-14


def _small_qkv(B=1, Hq=4, Hkv=2, T=150, D=16, seed=3):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, T, D, generator=g, dtype=torch.float64)
    K = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    V = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    hc = torch.randn(Hkv, D, generator=g, dtype=torch.float64)
    return Q, K, V, hc


def test_stage2_dense_is_causal_sdpa():
    import torch.nn.functional as F
    Q, K, V, hc = _small_qkv()
    O = oracle.stage2(Q, K, V, None, chunk_size=16, dense=True)
    ref = F.scaled_dot_product_attention(Q, K.repeat_interleave(2, 1), V.repeat_interleave(2, 1),
                                         is_causal=True)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-13)


def test_stage2_rows_in_first_chunk_are_local_causal_attention():
    import torch.nn.functional as F
    Q, K, V, hc = _small_qkv()
    Bc = 32
    S = oracle.stage0(K, hc, Bc)
    p, m, tau = oracle.stage1(Q, S, 150, Bc, 1.5, rows=range(Bc))
    O = oracle.stage2(Q, K, V, p, Bc, rows=range(Bc))
    ref = F.scaled_dot_product_attention(Q[:, :, :Bc], K[:, :, :Bc].repeat_interleave(2, 1),
                                         V[:, :, :Bc].repeat_interleave(2, 1), is_causal=True)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-13)


def test_stage2_masked_chunks_contribute_exactly_nothing():
    """With the routing p fixed, rewriting K and V inside a row's zero-probability chunks
    leaves that row's output unchanged to the bit (dynamic masking, g = 0 where w = 0)."""
    Q, K, V, hc = _small_qkv(T=256)
    Bc = 16
    S = oracle.stage0(K, hc, Bc)
    p, m, tau = oracle.stage1(Q, S, 256, Bc, 2.0)       # sparsemax: many exact zeros
    checked = 0
    for t in (40, 97, 150, 200, 255):
        for g in range(2):
            ct = t // Bc
            dead = [c for c in range(ct) if p[0, g, t, c] == 0]
            if not dead:
                continue
            K2, V2 = K.clone(), V.clone()
            for c in dead:
                K2[0, g, c * Bc:(c + 1) * Bc] = 1e3
                V2[0, g, c * Bc:(c + 1) * Bc] = -7e5
            O = oracle.stage2(Q, K, V, p[:, :, t:t + 1], Bc, rows=[t])
            O2 = oracle.stage2(Q, K2, V2, p[:, :, t:t + 1], Bc, rows=[t])
            for h in (2 * g, 2 * g + 1):
                assert np.array_equal(O[0, h], O2[0, h])
                checked += 1
    assert checked >= 12


@pytest.mark.parametrize("sigma", [1.0, 0.5, 2.0, 0.0])
def test_stage2_prior_softmax_is_the_variational_optimum(sigma):
    """w = argmax_{w in simplex} z.w - KL(w || g) with the prior g proportional to p^sigma on
    the routed keys (1 on the diagonal keys; sigma is the prior strength): optimal value
    log sum_j g_j e^{z_j}, masked keys get exactly zero weight, and no feasible perturbation
    does better."""
    T, Bc, D = 40, 8, 40
    g_ = torch.Generator().manual_seed(9)
    Q = torch.randn(1, 1, T, D, generator=g_, dtype=torch.float64)
    K = torch.randn(1, 1, T, D, generator=g_, dtype=torch.float64)
    V = torch.eye(T, D, dtype=torch.float64).view(1, 1, T, D)   # O row = attention weights
    hc = torch.randn(1, D, generator=g_, dtype=torch.float64)
    S = oracle.stage0(K, hc, Bc)
    p, m, tau = oracle.stage1(Q, S, T, Bc, 1.5)
    W = oracle.stage2(Q, K, V, p, Bc, sigma=sigma)[0, 0]          # [T, T]
    rng = np.random.default_rng(0)
    for t in range(Bc, T):
        ct = t // Bc
        z = (K[0, 0, :t + 1] @ Q[0, 0, t]).numpy() / math.sqrt(D)
        prior = np.array([1.0 if j // Bc == ct else p[0, 0, t, j // Bc] for j in range(t + 1)])
        w = W[t, :t + 1]
        assert (w[prior == 0] == 0).all() and (W[t, t + 1:] == 0).all()
        sup = prior > 0
        g = np.where(sup, np.where(sup, prior, 1.0) ** sigma, 0.0)
        g = g / g.sum()

        def F(u):
            us = u[sup]
            nz = us > 0
            return u @ z - (us[nz] * np.log(us[nz] / g[sup][nz])).sum()
        best = math.log((g[sup] * np.exp(z[sup])).sum())
        assert abs(F(w) - best) < 1e-12
        for _ in range(200):
            u = np.zeros(t + 1)
            u[sup] = np.maximum(w[sup] + rng.normal(size=sup.sum()) * 1e-2, 0)
            u /= u.sum()
            assert F(u) <= best + 1e-12


# ----------------------------------------------------------------------------- decode
def test_decode_equals_prefill_row():
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=700)
    T = 700
    full = oracle.prefill(q, k, v, hc, 64, 1.5, rows=[699, 640, 511])
    for i, t in enumerate([699, 640, 511]):
        L = t + 1
        dec = oracle.decode(q[:, :, t], k[:, :, :L], v[:, :, :L], hc, [L], 64, 1.5)
        np.testing.assert_allclose(dec["O"], full["O"][:, :, i], atol=1e-13)
        C = (L + 63) // 64
        np.testing.assert_allclose(dec["p"][:, :, :C], full["p"][:, :, i, :C], atol=1e-14)
    assert T == 700


def test_decode_route_from_cached_summaries_equals_decode_and_prefill_rows():
    """Routing a decode step from summaries computed once over the whole cache (frozen
    chunks, later chunks present but not routable) gives decode's routing, which recomputes
    the summaries of the complete chunks, and Stage 1's routing of the same prefill row;
    L = 640 and 641 straddle the completion of chunk 9."""
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=900)
    S = oracle.stage0(k, hc, 64)                                 # 14 complete chunks
    lens = [640, 641, 700, 129]
    qs = torch.stack([q[0, :, L - 1] for L in lens])                    # [4, Hq, D]
    kk = k.expand(4, -1, -1, -1)
    vv = v.expand(4, -1, -1, -1)
    r = oracle.decode_route(qs, np.repeat(S, 4, axis=0), lens, 900, 64, 1.5)
    d = oracle.decode(qs, kk, vv, hc, lens, 64, 1.5)
    np.testing.assert_array_equal(r["p"], d["p"])
    np.testing.assert_array_equal(r["tau"], d["tau"])
    np.testing.assert_array_equal(np.isnan(r["m"]), np.isnan(d["m"]))
    np.testing.assert_array_equal(np.nan_to_num(r["m"]), np.nan_to_num(d["m"]))
    rows = [L - 1 for L in lens]
    p1, m1, tau1 = oracle.stage1(q, S, 900, 64, 1.5, rows=rows)
    for i, L in enumerate(lens):
        np.testing.assert_allclose(r["p"][i], p1[0, :, i], atol=1e-15)
        np.testing.assert_allclose(r["tau"][i], tau1[0, :, i], atol=1e-15)
    assert (r["p"][1, :, 9] >= 0).all() and (r["p"][0, :, 9] == 0).all()   # chunk 9 routable at 641 only


# ----------------------------------------------------------------------------- estimate_diagonal
@pytest.mark.parametrize("alpha", [1.0, 1.5, 2.0])
def test_estimate_diagonal_routes_the_visible_part_of_the_diagonal_chunk(alpha):
    """Reading of estimate_diagonal (aiexpert.news interface paragraph: the diagonal correction
    of the alpha-entmax normalisation; gist.science "Stufe 2": chunks near the diagonal may have
    no summary): the diagonal chunk joins the entmax as one more candidate, its summary
    estimated as Stage 0 does for a complete chunk but over the keys the row can see.  Written
    out here independently: the estimated summary is torch's single-query SDPA (float64) of
    head_cls over keys c_t Bc .. t, the scores an einsum; the routing must be oracle.entmax of
    [routed scores, diagonal score].  Rows t < Bc route to their diagonal chunk alone."""
    import torch.nn.functional as F
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=700)
    T, D, Bc = 700, 128, 64
    S = oracle.stage0(k, hc, Bc)
    rows = np.array([0, 5, 63, 64, 100, 127, 128, 383, 640, 699])
    p, m, tau = oracle.stage1(q, S, T, Bc, alpha, rows=rows, estimate_diagonal=True, K=k,
                              head_cls=hc)
    qbar = q.double().view(1, 2, 16, T, D).mean(2)
    kd = k.double()
    for g in range(2):
        for i, t in enumerate(rows):
            ct = t // Bc
            keys = kd[0, g, ct * Bc:t + 1]                                  # visible diagonal keys
            dsum = F.scaled_dot_product_attention(hc.double()[g].view(1, 1, D), keys[None], keys[None])[0, 0]
            if t == ct * Bc + Bc - 1 and ct < S.shape[2]:                    # a whole chunk: Stage 0's summary
                np.testing.assert_allclose(dsum.numpy(), S[0, g, ct], atol=1e-13)
            z = torch.cat([torch.from_numpy(S[0, g, :ct]) @ qbar[0, g, t], (dsum @ qbar[0, g, t])[None]])
            z = (z / math.sqrt(D)).numpy()
            pr, tr = oracle.entmax(z, alpha)
            np.testing.assert_allclose(p[0, g, i, :ct + 1], pr, atol=1e-12)
            assert (p[0, g, i, ct + 1:] == 0).all()
            assert abs(tau[0, g, i] - tr) < 1e-12
            assert abs(p[0, g, i].sum() - 1.0) < 1e-12
            if ct == 0:
                assert abs(p[0, g, i, 0] - 1.0) < 1e-12
    # Without the flag the routed chunks hold all the mass; with it they hold 1 - p[c_t].
    p0, _, _ = oracle.stage1(q, S, T, Bc, alpha, rows=rows)
    ct = rows // Bc
    routed = rows >= Bc
    assert (np.abs(p0[0][:, routed].sum(-1) - 1) < 1e-12).all()
    pdiag = p[0][:, np.arange(rows.size), ct]                                # [Hkv, nrows]
    routed_mass = p[0].sum(-1) - pdiag
    np.testing.assert_allclose(routed_mass[:, routed], 1 - pdiag[:, routed], atol=1e-12)
    if alpha < 2:
        assert (pdiag[:, routed] > 0).any()


def test_estimate_diagonal_decode_equals_prefill_row():
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=700)
    rows = [699, 640, 639, 511]
    full = oracle.prefill(q, k, v, hc, 64, 1.5, rows=rows, estimate_diagonal=True)
    S = oracle.stage0(k, hc, 64)
    for i, t in enumerate(rows):
        L = t + 1
        dec = oracle.decode(q[:, :, t], k[:, :, :L], v[:, :, :L], hc, [L], 64, 1.5,
                            estimate_diagonal=True)
        np.testing.assert_allclose(dec["O"], full["O"][:, :, i], atol=1e-13)
        C = (L + 63) // 64
        np.testing.assert_allclose(dec["p"][:, :, :C], full["p"][:, :, i, :C], atol=1e-14)
        r = oracle.decode_route(q[:, :, t], S, [L], 700, 64, 1.5, estimate_diagonal=True,
                                K_cache=k, head_cls=hc)
        np.testing.assert_allclose(r["p"][:, :, :C], full["p"][:, :, i, :C], atol=1e-14)


# ----------------------------------------------------------------------------- top-k routing
@pytest.mark.parametrize("n,k", [(1, 4), (7, 3), (50, 16), (2047, 64), (12, 12)])
def test_topk_selects_the_k_highest_scores_with_lower_index_on_ties(n, k):
    """Top-k routing (the fixed-k block selection of the hierarchical baselines the pages
    compare against, liuzhao09.github.io sections 1-2): against numpy's stable sort on the
    negated scores (which keeps the lower index first among equal scores)."""
    s = np.round(RNG.normal(size=n) * 2, 1)          # rounding makes ties likely
    p, theta = oracle.topk(s, k)
    order = np.argsort(-s, kind="stable")
    ke = min(k, n)
    want = np.zeros(n)
    want[order[:ke]] = 1.0 / ke
    np.testing.assert_array_equal(p, want)
    assert theta == s[order[ke - 1]]
    assert abs(p.sum() - 1) < 1e-12


def test_topk_prefill_attends_the_selection_with_a_uniform_prior():
    """With top-k routing Stage 2 is plain softmax over the selected chunks' keys and the
    diagonal chunk (no bias): the oracle's prefill equals its dense attention with every
    unselected routed chunk's keys masked, written out with torch SDPA (float64)."""
    import torch.nn.functional as F
    q, k, v, hc = make_prefill(CONFIGS["gqa32k"], seq_len=600)
    T, D, Bc, K = 600, 128, 64, 3
    r = oracle.prefill(q, k, v, hc, Bc, 1.5, topk=K)
    ct = np.arange(T) // Bc
    sel = r["p"] > 0                                                   # [1,Hkv,T,C]
    assert (sel.sum(-1)[0][:, ct >= 1] == np.minimum(K, ct[ct >= 1])).all()
    keep = np.zeros((2, T, T), bool)
    j = np.arange(T)
    for g in range(2):
        for t in range(T):
            c = j // Bc
            keep[g, t] = (j <= t) & ((c == ct[t]) | ((c < ct[t]) & sel[0, g, t, np.minimum(c, sel.shape[-1] - 1)]))
    mask = torch.from_numpy(np.repeat(keep, 16, axis=0))[None]        # [1,Hq,T,T]
    ref = F.scaled_dot_product_attention(q.double(), k.double().repeat_interleave(16, 1),
                                         v.double().repeat_interleave(16, 1), attn_mask=mask)
    np.testing.assert_allclose(r["O"], ref.numpy(), atol=1e-12)


# ----------------------------------------------------------------------------- backward
def _tiny_problem(seed, B=1, Hq=4, Hkv=2, T=40, D=8, Bc=8):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, T, D, generator=g, dtype=torch.float64)
    K = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    V = torch.randn(B, Hkv, T, D, generator=g, dtype=torch.float64)
    hc = torch.randn(Hkv, D, generator=g, dtype=torch.float64)
    dO = torch.randn(B, Hq, T, D, generator=g, dtype=torch.float64)
    return Q, K, V, hc, dO


def _loss(Q, K, V, hc, dO, Bc, alpha, sigma):
    return float((oracle.prefill(Q, K, V, hc, Bc, alpha, sigma=sigma)["O"] * dO.numpy()).sum())


@pytest.mark.parametrize("alpha,sigma", [(1.5, 1.0), (2.0, 0.5), (1.0, 1.0), (1.25, 2.0)])
def test_backward_matches_central_finite_differences(alpha, sigma):
    """The oracle's gradients of sum(O * dO) through Stages 2, 1 and 0 against central finite
    differences of its own forward, for sampled entries of every input (the entmax supports
    are fixed under the perturbation: every margin lies well away from zero)."""
    Bc = 8
    for seed in range(40):                       # a problem whose routing margins are not tiny
        Q, K, V, hc, dO = _tiny_problem(seed)
        r = oracle.prefill(Q, K, V, hc, Bc, alpha, sigma=sigma)
        m = r["m"][np.isfinite(r["m"])]
        if alpha == 1.0 or np.abs(m).min() > 1e-3:
            break
    else:
        pytest.skip("no problem with clear margins")
    gr = oracle.backward(Q, K, V, hc, dO, Bc, alpha, sigma=sigma)
    rng = np.random.default_rng(seed)
    eps = 1e-6
    for name, X, dX in (("Q", Q, gr["dQ"]), ("K", K, gr["dK"]), ("V", V, gr["dV"]), ("hc", hc, gr["dhc"])):
        flat = X.view(-1)
        for idx in rng.choice(flat.numel(), 12, replace=False):
            old = float(flat[idx])
            flat[idx] = old + eps
            lp = _loss(Q, K, V, hc, dO, Bc, alpha, sigma)
            flat[idx] = old - eps
            lm = _loss(Q, K, V, hc, dO, Bc, alpha, sigma)
            flat[idx] = old
            fd = (lp - lm) / (2 * eps)
            an = dX.reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, an)
    # the routing gradient reaches head_cls (Stage 0): not identically zero
    assert np.abs(gr["dhc"]).max() > 1e-6


def test_backward_without_the_prior_is_masked_attention_backward():
    """sigma = 0 removes the routing from the gradient (the bias is zero on every attended key),
    so dQ, dK, dV are the gradients of plain softmax attention restricted to the routed chunks
    and the diagonal -- torch autograd through scaled_dot_product_attention in float64 with
    that mask -- and head_cls gets no gradient."""
    import torch.nn.functional as F
    Q, K, V, hc, dO = _tiny_problem(3, T=48)
    Bc, T = 8, 48
    r = oracle.prefill(Q, K, V, hc, Bc, 1.5, sigma=0.0)
    gr = oracle.backward(Q, K, V, hc, dO, Bc, 1.5, sigma=0.0)
    ct = np.arange(T) // Bc
    keep = np.zeros((2, T, T), bool)
    for g in range(2):
        for t in range(T):
            for j in range(t + 1):
                c = j // Bc
                keep[g, t, j] = c == ct[t] or r["p"][0, g, t, c] > 0
    mask = torch.from_numpy(np.repeat(keep, 2, axis=0))[None]
    q, k, v = (x.clone().requires_grad_(True) for x in (Q, K, V))
    O = F.scaled_dot_product_attention(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1),
                                       attn_mask=mask)
    (O * dO).sum().backward()
    np.testing.assert_allclose(gr["dQ"], q.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(gr["dK"], k.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(gr["dV"], v.grad.numpy(), atol=1e-12)
    assert np.abs(gr["dhc"]).max() == 0.0
