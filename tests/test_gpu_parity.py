"""GPU parity of every stage against the fp64 oracle, through the C ABI (via the binding),
at sizes the oracle finishes in seconds that still span several tiles and a ragged tail."""
import ctypes
import numpy as np
import pytest
import torch

import oracle
from dash_inputs import CONFIGS, PrefillConfig, make_prefill
from parity_util import check_output, check_routing, unpack_mask

pytestmark = pytest.mark.gpu

dev = "cuda"


@pytest.fixture(scope="module")
def dash():
    import sparse_hierarchical_attention_stage0_b200 as d
    return d


def _cfg(B, Hq, Hkv, T, D, Bc, alpha, planted=True, n_max=8, seed=0, gamma=1.0):
    return PrefillConfig("t", B, Hq, Hkv, T, D, Bc, alpha, gamma=gamma, planted=planted,
                         n_max=n_max, seed=seed)


def _to(*ts):
    return [t.to(dev) for t in ts]


# ------------------------------------------------------------------------------ stage 0
@pytest.mark.parametrize("D,Bc,T", [(64, 64, 1000), (128, 64, 777), (128, 128, 1300),
                                    (64, 128, 256), (128, 64, 50)])
def test_stage0_matches_oracle(dash, D, Bc, T):
    q, k, v, hc = make_prefill(_cfg(2, 4, 2, T, D, Bc, 1.5, planted=False, seed=D + T))
    S = dash.stage0(k.to(dev), hc.to(dev), Bc)
    torch.cuda.synchronize()
    ref = oracle.stage0(k, hc, Bc)
    assert S.shape == ref.shape
    if ref.size:
        rel = np.abs(S.cpu().double().numpy() - ref).max() / np.abs(ref).max()
        assert rel <= 1e-5, rel


def test_update_chunk_cache_is_bit_identical_to_stage0(dash):
    B, Hkv, cap, D, Bc = 3, 2, 1024 + 64, 128, 64
    g = torch.Generator().manual_seed(5)
    k = torch.randn(B, Hkv, cap, D, generator=g).to(torch.bfloat16).to(dev)
    hc = torch.randn(Hkv, D, generator=g).to(dev)
    full = dash.stage0(k, hc, Bc)                           # every complete chunk
    cache = torch.full_like(full, float("nan"))
    seq = torch.tensor([64, 700, 1088], dtype=torch.int32, device=dev)
    dash.update_chunk_cache(k, hc, seq, cache, heads_q=2 * Hkv, chunk_size=Bc, n_recent=cap // Bc)
    torch.cuda.synchronize()
    for b, L in enumerate([64, 700, 1088]):
        n = L // Bc
        assert torch.equal(cache[b, :, :n], full[b, :, :n])
        assert torch.isnan(cache[b, :, n:]).all()           # chunks not yet complete: untouched


def test_update_chunk_cache_reports_bad_seq_len(dash):
    B, Hkv, cap, D = 2, 2, 512, 64
    k = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    hc = torch.zeros(Hkv, D, device=dev)
    cache = torch.zeros(B, Hkv, cap // 64, D, device=dev)
    ws = dash.workspace(256, dev)
    seq = torch.tensor([cap + 1, 64], dtype=torch.int32, device=dev)
    dash.update_chunk_cache(k, hc, seq, cache, heads_q=2, chunk_size=64, ws=ws)
    assert dash.read_device_status(ws) == 1                 # DASH_ERR_INVALID_ARGUMENT
    assert dash.read_device_status(ws) == 0                 # read clears it


# ------------------------------------------------------------------------------ stage 1
@pytest.mark.parametrize("alpha", [1.0, 1.25, 1.5, 2.0])
@pytest.mark.parametrize("G,D,Bc,T", [(16, 128, 64, 2048 + 37), (4, 128, 128, 3000),
                                      (4, 128, 64, 2500 + 11), (1, 64, 64, 1500), (2, 64, 128, 1100)])
def test_route_matches_oracle(dash, alpha, G, D, Bc, T):
    Hkv = 2
    cfg = _cfg(1, G * Hkv, Hkv, T, D, Bc, alpha, seed=int(alpha * 10) + G)
    q, k, v, hc = make_prefill(cfg)
    qd, kd, hcd = _to(q, k, hc)
    S = dash.stage0(kd, hcd, Bc)
    r = dash.route(qd, S, Hkv, Bc, alpha)
    torch.cuda.synchronize()
    # Oracle Stage 1 on the GPU's own summaries isolates the routing arithmetic.
    p_or, m_or, tau_or = oracle.stage1(q, S.cpu(), T, Bc, alpha)
    C = p_or.shape[-1]
    bits = unpack_mask(r["active_blocks"], C)
    n_ex = check_routing(bits, r["p"].cpu().double().numpy(), p_or, m_or, np.arange(T), Bc,
                         alpha, tag=f"a={alpha} G={G}")
    assert n_ex <= 3
    tau = r["tau"].cpu().double().numpy()
    routed = np.arange(T) >= Bc
    np.testing.assert_allclose(tau[..., routed], tau_or[..., routed], atol=2e-5)
    assert np.isnan(tau[..., ~routed]).all()


# ------------------------------------------------------------------------------ prefill
@pytest.mark.parametrize("alpha", [1.0, 1.25, 1.5, 2.0])
@pytest.mark.parametrize("G,D,Bc,T", [(16, 128, 64, 1024 + 100), (4, 128, 128, 1500),
                                      (4, 128, 64, 1300 + 9), (1, 64, 64, 777), (8, 64, 64, 640), (32, 128, 64, 700),
                                      (8, 128, 128, 1500 + 3), (16, 128, 128, 1100)])
def test_prefill_matches_oracle(dash, alpha, G, D, Bc, T):
    Hkv = 2 if G <= 16 else 1
    cfg = _cfg(1, G * Hkv, Hkv, T, D, Bc, alpha, seed=7 + G)
    q, k, v, hc = make_prefill(cfg)
    res = dash.prefill(*_to(q, k, v, hc), chunk_size=Bc, alpha=alpha, enable_gqa=True,
                       return_p=True, return_active_blocks=True, return_summary=True)
    torch.cuda.synchronize()
    ref = oracle.prefill(q, k, v, hc, Bc, alpha)
    C = ref["p"].shape[-1]
    check_routing(unpack_mask(res["active_blocks"], C), res["p"].cpu().double().numpy(),
                  ref["p"], ref["m"], np.arange(T), Bc, alpha, tag="prefill")
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag=f"G={G} a={alpha}")
    assert dash.read_device_status(res["ws"]) == 0


@pytest.mark.parametrize("alpha,sigma", [(1.5, 0.5), (2.0, 2.0), (1.0, 0.25)])
def test_prefill_prior_strength_sigma(dash, alpha, sigma):
    """sigma scales the log-prior bias of the routed chunks (the prior strength the pages
    name for Stage 2; reading C10)."""
    q, k, v, hc = make_prefill(_cfg(1, 32, 2, 1100, 128, 64, alpha, seed=50))
    res = dash.prefill(*_to(q, k, v, hc), chunk_size=64, alpha=alpha, sigma=sigma,
                       enable_gqa=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    ref = oracle.prefill(q, k, v, hc, 64, alpha, sigma=sigma)
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag=f"a={alpha} sigma={sigma}")


def test_tiny_config_every_row(dash):
    """The tiny workload as configured (B=1, 4 query heads on 4 KV heads without GQA, D=64,
    T=1024, chunk 64, alpha 1.5, i.i.d. inputs): mask, p and O on every row."""
    cfg = CONFIGS["tiny"]
    q, k, v, hc = make_prefill(cfg)
    res = dash.prefill(*_to(q, k, v, hc), chunk_size=cfg.chunk_size, alpha=cfg.alpha,
                       enable_gqa=False, return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    ref = oracle.prefill(q, k, v, hc, cfg.chunk_size, cfg.alpha)
    C = ref["p"].shape[-1]
    check_routing(unpack_mask(res["active_blocks"], C), res["p"].cpu().double().numpy(),
                  ref["p"], ref["m"], np.arange(cfg.seq_len), cfg.chunk_size, cfg.alpha, tag="tiny")
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag="tiny")


@pytest.mark.parametrize("G,Bc,T", [(16, 64, 2100 + 37), (8, 128, 1500 + 3)])
def test_attend_without_vt_scratch_takes_the_tile_kernel(dash, G, Bc, T):
    """dash_attend with only the 256-byte status word cannot hold V^T, so Stage 2 runs on the
    64-key-block tile kernel; with dash_attend_workspace_size bytes it runs the 128-key-block
    kernel.  Both match the oracle, across several routing-bias batches (T > 32 chunks)."""
    Hkv = 2
    cfg = _cfg(1, G * Hkv, Hkv, T, 128, Bc, 1.5, seed=23 + G)
    q, k, v, hc = make_prefill(cfg)
    qd, kd, vd, hcd = _to(q, k, v, hc)
    res = dash.prefill(qd, kd, vd, hcd, chunk_size=Bc, alpha=1.5, enable_gqa=True,
                       return_active_blocks=True, return_summary=True)
    torch.cuda.synchronize()
    # tau is re-derived by Stage 1 alone (bit-identical to the prefill's)
    summ = res["summary"]
    r = dash.route(qd, summ, Hkv, Bc, 1.5, return_p=False)
    tau, mask = r["tau"], r["active_blocks"]
    assert torch.equal(mask, res["active_blocks"])
    prm = dash.make_params(1, G * Hkv, Hkv, T, 128, Bc, 1.5, 1.0, 1.0, True)
    assert dash.attend_workspace_size(prm) > 256
    small = dash.workspace(256, qd.device)
    o_tile = dash.attend(qd, kd, vd, summ, tau, mask, Bc, 1.5, ws=small)
    o_fast = dash.attend(qd, kd, vd, summ, tau, mask, Bc, 1.5)
    torch.cuda.synchronize()
    assert dash.read_device_status(small) == 0
    ref = oracle.prefill(q, k, v, hc, Bc, 1.5)
    check_output(o_tile.cpu().float().numpy(), ref["O"], tag="tile kernel")
    check_output(o_fast.cpu().float().numpy(), ref["O"], tag="128-key kernel")
    assert torch.equal(o_fast, res["out"])


def test_prefill_single_partial_chunk(dash):
    """T < chunk_size: every row is local causal attention inside chunk 0."""
    q, k, v, hc = make_prefill(_cfg(2, 8, 2, 40, 64, 64, 1.5, planted=False, seed=3))
    out = dash.prefill(*_to(q, k, v, hc), chunk_size=64, alpha=1.5, enable_gqa=True)
    torch.cuda.synchronize()
    ref = oracle.stage2(q, k, v, None, 64, dense=True)
    check_output(out.cpu().float().numpy(), ref)


def test_dense_equals_force_all_active_and_causal_attention(dash):
    cfg = _cfg(1, 32, 2, 1200, 128, 64, 1.5, seed=11)
    q, k, v, hc = make_prefill(cfg)
    qd, kd, vd, hcd = _to(q, k, v, hc)
    o_dense = dash.prefill(qd, kd, vd, None, 64, enable_gqa=True, dense=True)
    o_force = dash.prefill(qd, kd, vd, hcd, 64, enable_gqa=True, force_all_active=True)
    torch.cuda.synchronize()
    assert torch.equal(o_dense, o_force)
    ref = oracle.stage2(q, k, v, None, 64, dense=True)
    check_output(o_dense.cpu().float().numpy(), ref, tag="dense")


@pytest.mark.parametrize("B,G,Bc,T", [(2, 16, 64, 993), (1, 8, 64, 1505), (1, 32, 128, 1027),
                                      (2, 8, 128, 700), (2, 4, 64, 777), (1, 2, 128, 1100 + 9)])
def test_dense_on_sm_pairs_matches_causal_attention(dash, B, G, Bc, T):
    """Dense mode runs on pairs of SMs, two tiles per pair.  Odd tile counts leave the last
    pair's second tile past the end of the sequence; batch 2 covers several (b, g) planes."""
    cfg = _cfg(B, 2 * G, 2, T, 128, Bc, 1.5, planted=False, seed=20 + G + B)
    q, k, v, hc = make_prefill(cfg)
    qd, kd, vd = _to(q, k, v)
    prm = dash.make_params(B, 2 * G, 2, T, 128, Bc, enable_gqa=True)
    ws = dash.workspace(dash.prefill_workspace_size(prm), qd.device)
    out = dash.prefill(qd, kd, vd, None, Bc, enable_gqa=True, dense=True, ws=ws)
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0
    ref = oracle.stage2(q, k, v, None, Bc, dense=True)
    check_output(out.cpu().float().numpy(), ref, tag=f"dense pairs B={B} G={G} Bc={Bc}")


def test_prefill_batch2_matches_oracle(dash):
    """Routed prefill over four (b, g) planes (the Stage 2 grid walks them one after another)."""
    cfg = _cfg(2, 32, 2, 700, 128, 64, 1.5, seed=31)
    q, k, v, hc = make_prefill(cfg)
    res = dash.prefill(*_to(q, k, v, hc), chunk_size=64, alpha=1.5, enable_gqa=True,
                       return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    ref = oracle.prefill(q, k, v, hc, 64, 1.5)
    C = ref["p"].shape[-1]
    check_routing(unpack_mask(res["active_blocks"], C), res["p"].cpu().double().numpy(),
                  ref["p"], ref["m"], np.arange(700), 64, 1.5, tag="prefill B=2")
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag="prefill B=2")
    assert dash.read_device_status(res["ws"]) == 0


@pytest.mark.parametrize("G,D,Bc,T,dense,n", [(16, 128, 64, 1100, False, 4), (8, 128, 128, 1505, True, 3),
                                              (8, 64, 64, 640, False, 4), (32, 128, 64, 700, False, 64)])
def test_prefill_host_equals_prefill(dash, G, D, Bc, T, dense, n):
    """The sliced prefill from host memory gives dash_prefill's output bit for bit (row slices
    of 128-row multiples; D = 64 runs as one slice; more slices asked than 128-row blocks).
    K, V and q arrive slice by slice, each slice summarising and transposing only its own rows:
    the device buffers and the workspace start as NaN bytes, so a row that no slice covered
    shows up in the output."""
    Hkv = 2 if G <= 16 else 1
    q, k, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, D, Bc, 1.5, seed=40 + G))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    ref = dash.prefill(qd, kd, vd, None if dense else hcd, Bc, 1.5, enable_gqa=True, dense=dense)
    torch.cuda.synchronize()
    hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    bq, bk, bv, bhc, bo = (torch.empty_like(x) for x in (qd, kd, vd, hcd, qd))
    for x in (bq, bk, bv, bo):
        x.view(torch.int16).fill_(-1)                   # 0xFFFF: a bf16 NaN
    prm = dash.make_params(1, G * Hkv, Hkv, T, D, Bc, 1.5, enable_gqa=True, flags=1 if dense else 0)
    ws = dash.workspace(dash.prefill_workspace_size(prm), qd.device)
    ws.fill_(255)
    ws[:256].zero_()
    dash.prefill_host(hq, hk, hv, None if dense else hhc, ho, bq, bk, bv, None if dense else bhc, bo,
                      Bc, 1.5, enable_gqa=True, dense=dense, n_slices=n, ws=ws)
    torch.cuda.current_stream().synchronize()
    assert dash.read_device_status(ws) == 0
    assert torch.equal(ho, ref.cpu())
    assert torch.equal(bo, ref)


def test_inactive_chunks_do_not_touch_the_output(dash):
    """Rewriting V inside chunks that none of the last query chunk's 64 tokens routes to
    leaves those tokens' outputs identical to the bit."""
    cfg = _cfg(1, 32, 2, 2048, 128, 64, 2.0, seed=12, n_max=2)
    q, k, v, hc = make_prefill(cfg)
    qd, kd, vd, hcd = _to(q, k, v, hc)
    res = dash.prefill(qd, kd, vd, hcd, 64, alpha=2.0, enable_gqa=True, return_active_blocks=True)
    torch.cuda.synchronize()
    bits = unpack_mask(res["active_blocks"], 32)[0, :, -64:]     # [Hkv, 64 rows, C]
    used = bits.any(axis=1)                                       # [Hkv, C]
    v2 = vd.clone()
    n_dead = 0
    for g in range(2):
        for c in range(31):
            if not used[g, c]:
                v2[0, g, c * 64:(c + 1) * 64] = 1e4
                n_dead += 1
    assert n_dead > 0
    out2 = dash.prefill(qd, kd, v2, hcd, 64, alpha=2.0, enable_gqa=True)
    torch.cuda.synchronize()
    assert torch.equal(res["out"][:, :, -64:], out2[:, :, -64:])


# ------------------------------------------------------------------------------ decode
def _decode_setup(dash, B, Hq, Hkv, L, D, Bc, seed):
    cfg = _cfg(B, Hq, Hkv, L, D, Bc, 1.5, seed=seed)
    q, k, v, hc = make_prefill(cfg)
    return cfg, q, k, v, hc


@pytest.mark.parametrize("G,D,Bc", [(16, 128, 64), (4, 64, 128), (1, 64, 64)])
def test_decode_matches_oracle_and_prefill_rows(dash, G, D, Bc):
    B, Hkv, L = 3, 2, 1500
    cfg, q, k, v, hc = _decode_setup(dash, B, G * Hkv, Hkv, L, D, Bc, seed=20 + G)
    qd, kd, vd, hcd = _to(q, k, v, hc)
    pre = dash.prefill(qd, kd, vd, hcd, Bc, enable_gqa=True, return_p=True,
                       return_active_blocks=True)
    cap = L + 37
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    kc[:, :, :L] = kd
    vc[:, :, :L] = vd
    cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
    lens = [L, L - 1, Bc * 3]                                 # rows t = L-1, L-2, 3Bc-1
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    dash.update_chunk_cache(kc, hcd, seq, cache, heads_q=G * Hkv, chunk_size=Bc, n_recent=cap // Bc)
    qs = torch.stack([qd[b, :, lens[b] - 1] for b in range(B)])        # [B,Hq,D]
    ws = dash.workspace(256, dev)
    dec = dash.decode(qs, kc, vc, seq, cache, Bc, enable_gqa=True, return_p=True,
                      return_active_blocks=True, ws=ws)
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0
    C = (L + Bc - 1) // Bc
    for b in range(B):
        t = lens[b] - 1
        # decode row == prefill row: routing bit-identical, output within bf16 rounding
        assert torch.equal(dec["p"][b, :, :C], pre["p"][b, :, t])
        assert torch.equal(dec["active_blocks"][b, :, :(C + 63) // 64], pre["active_blocks"][b, :, t])
        d = (dec["out"][b].float() - pre["out"][b, :, t].float()).abs().max().item()
        assert d <= 2e-2, d
    ref = oracle.decode(qs.cpu(), kc.cpu(), vc.cpu(), hc, lens, Bc, 1.5)
    check_output(dec["out"].cpu().float().numpy(), ref["O"], tag="decode")
    bits = unpack_mask(dec["active_blocks"], ref["p"].shape[-1])
    for b in range(B):
        t = lens[b] - 1
        check_routing(bits[b][:, None], dec["p"][b][:, None].cpu().double().numpy(),
                      ref["p"][b][:, None], ref["m"][b][:, None], [t], Bc, 1.5, tag="decode")


def test_newton_cap_hook_reports_device_timeout(dash):
    """Fault injection without a GPU fault: the test flag caps the entmax Newton solve at one
    iteration.  With i.i.d. inputs every row's scaled scores lie within 1 of their maximum, so
    rows need a second step and report DASH_ERR_DEVICE_TIMEOUT through the status word; the
    same call without the flag then succeeds (the context stays usable)."""
    T, D, Bc, Hkv, Hq = 1100, 128, 64, 2, 32
    q, k, v, hc = make_prefill(_cfg(1, Hq, Hkv, T, D, Bc, 1.5, planted=False, seed=60))
    qd, kd, hcd = _to(q, k, hc)
    summ = dash.stage0(kd, hcd, Bc)
    C = (T + Bc - 1) // Bc
    tau = torch.empty(1, Hkv, T, device=dev)
    mask = torch.empty(1, Hkv, T, (C + 63) // 64, dtype=torch.int64, device=dev)
    ws = dash.workspace(256, qd.device)
    for flags, want in ((dash.FLAG_TEST_NEWTON_CAP, 5), (0, 0)):
        prm = dash.make_params(1, Hq, Hkv, T, D, Bc, 1.5, enable_gqa=True, flags=flags)
        rc = dash.lib.dash_route(ctypes.byref(prm), dash._ptr(qd), dash._ptr(summ), dash._ptr(tau),
                                 None, dash._ptr(mask), dash._ptr(ws), 256, dash._stream(qd.device))
        assert rc == 0
        assert dash.read_device_status(ws) == want, (flags, dash.read_device_status(ws))


def test_stall_hook_times_out_and_leaves_the_context_usable(dash):
    """Fault injection without a GPU fault: the test flag makes Stage 0's bounded copy wait
    run out (no copy is issued, so nothing arrives on its barrier).  The kernel reports
    DASH_ERR_DEVICE_TIMEOUT after its 2 s limit and returns with nothing in flight; the next
    call on the same context succeeds and matches the oracle."""
    T, D, Bc = 256, 128, 64                          # 4 chunks: one CTA waits its 2 s
    q, k, v, hc = make_prefill(_cfg(1, 2, 2, T, D, Bc, 1.5, planted=False, seed=61))
    kd, hcd = _to(k, hc)
    summ = torch.empty(1, 2, T // Bc, D, device=dev)
    ws = dash.workspace(256, kd.device)
    for flags, want in ((dash.FLAG_TEST_STALL_WAIT, 5), (0, 0)):
        prm = dash.make_params(1, 2, 2, T, D, Bc, flags=flags)
        rc = dash.lib.dash_stage0(ctypes.byref(prm), dash._ptr(kd), dash._ptr(hcd), dash._ptr(summ),
                                  dash._ptr(ws), 256, dash._stream(kd.device))
        assert rc == 0
        assert dash.read_device_status(ws) == want, flags
    ref = oracle.stage0(k, hc, Bc)
    rel = np.abs(summ.cpu().double().numpy() - ref).max() / np.abs(ref).max()
    assert rel <= 1e-5, rel


def test_decode_reports_bad_seq_len(dash):
    B, Hkv, cap, D = 2, 2, 256, 128
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    cache = torch.zeros(B, Hkv, cap // 64, D, device=dev)
    q = torch.zeros(B, 32, D, dtype=torch.bfloat16, device=dev)
    seq = torch.tensor([cap + 5, 10], dtype=torch.int32, device=dev)
    ws = dash.workspace(256, dev)
    dash.decode(q, kc, kc, seq, cache, 64, enable_gqa=True, ws=ws)
    assert dash.read_device_status(ws) == 1


# ------------------------------------------------------------------------------ estimate_diagonal
@pytest.mark.parametrize("alpha", [1.0, 1.5, 2.0])
@pytest.mark.parametrize("G,D,Bc,T", [(16, 128, 64, 1100 + 5), (4, 128, 128, 1300), (1, 64, 64, 777)])
def test_prefill_estimate_diagonal_matches_oracle(dash, alpha, G, D, Bc, T):
    """estimate_diagonal: the diagonal chunk joins the entmax with its summary estimated over
    the keys each row can see; p[.., c_t] is its probability, the routed chunks share the rest,
    Stage 2 attends the diagonal with bias 0 as before."""
    Hkv = 2
    q, k, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, D, Bc, alpha, seed=70 + G))
    res = dash.prefill(*_to(q, k, v, hc), chunk_size=Bc, alpha=alpha, enable_gqa=True,
                       estimate_diagonal=True, return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    ref = oracle.prefill(q, k, v, hc, Bc, alpha, estimate_diagonal=True)
    C = ref["p"].shape[-1]
    p = res["p"].cpu().double().numpy()
    check_routing(unpack_mask(res["active_blocks"], C), p, ref["p"], ref["m"], np.arange(T), Bc,
                  alpha, tag=f"estimate_diagonal G={G} a={alpha}")
    ct = np.arange(T) // Bc
    pdiag = p[0][:, np.arange(T), ct]
    assert np.abs(p[0].sum(-1) - 1).max() < 1e-4          # the diagonal is part of the simplex
    if alpha < 2:
        assert (pdiag > 0).any()
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag=f"estimate_diagonal G={G}")


def test_decode_estimate_diagonal_matches_oracle(dash):
    B, Hkv, G, L, D, Bc = 3, 2, 16, 1500, 128, 64
    q, k, v, hc = make_prefill(_cfg(B, G * Hkv, Hkv, L, D, Bc, 1.5, seed=71))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    cap = L + 37
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    kc[:, :, :L] = kd
    vc[:, :, :L] = vd
    cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
    lens = [L, Bc * 3 + 1, 40]                                # the last row routes to chunk 0 alone
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    dash.update_chunk_cache(kc, hcd, seq, cache, heads_q=G * Hkv, chunk_size=Bc, n_recent=cap // Bc)
    qs = torch.stack([qd[b, :, lens[b] - 1] for b in range(B)])
    ws = dash.workspace(256, dev)
    dec = dash.decode(qs, kc, vc, seq, cache, Bc, enable_gqa=True, return_p=True,
                      return_active_blocks=True, ws=ws, estimate_diagonal=True, head_cls=hcd)
    pre = dash.prefill(qd, kd, vd, hcd, Bc, enable_gqa=True, estimate_diagonal=True, return_p=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0
    ref = oracle.decode(qs.cpu(), kc.cpu(), vc.cpu(), hc, lens, Bc, 1.5, estimate_diagonal=True)
    check_output(dec["out"].cpu().float().numpy(), ref["O"], tag="decode estimate_diagonal")
    bits = unpack_mask(dec["active_blocks"], ref["p"].shape[-1])
    for b in range(B):
        t = lens[b] - 1
        check_routing(bits[b][:, None], dec["p"][b][:, None].cpu().double().numpy(),
                      ref["p"][b][:, None], ref["m"][b][:, None], [t], Bc, 1.5, tag="decode est")
        C = (L + Bc - 1) // Bc
        assert torch.equal(dec["p"][b, :, :C], pre["p"][b, :, t])        # same routing as prefill
    assert torch.allclose(dec["p"][2, :, 0], torch.ones(Hkv, device=dev))


# ------------------------------------------------------------------------------ top-k routing
@pytest.mark.parametrize("G,D,Bc,T,k", [(16, 128, 64, 1100 + 5, 4), (4, 128, 128, 1500, 3),
                                        (1, 64, 64, 777, 2), (8, 128, 128, 1300, 64)])
def test_prefill_topk_matches_oracle(dash, G, D, Bc, T, k):
    """Top-k routing: the k highest-scoring chunks plus the diagonal, a uniform prior in Stage 2
    (the fixed-k selection of the hierarchical baselines); k = 64 exceeds every row's c_t here,
    so all visible chunks are selected."""
    from parity_util import check_topk
    Hkv = 2
    q, k_, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, D, Bc, 1.5, seed=80 + G))
    res = dash.prefill(*_to(q, k_, v, hc), chunk_size=Bc, enable_gqa=True, topk=k,
                       return_p=True, return_active_blocks=True)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    ref = oracle.prefill(q, k_, v, hc, Bc, 1.5, topk=k)
    C = ref["p"].shape[-1]
    same = check_topk(unpack_mask(res["active_blocks"], C)[0], res["p"].cpu().double().numpy()[0],
                      ref["p"][0], ref["m"][0], np.arange(T), Bc, k, tag=f"topk G={G}")
    assert same.mean() >= 0.999, same.mean()
    rows = np.nonzero(same.all(0))[0]                      # rows whose selection is the oracle's
    check_output(res["out"].cpu().float().numpy()[:, :, rows], ref["O"][:, :, rows], tag="topk")


def test_decode_topk_equals_prefill_row(dash):
    B, Hkv, G, L, D, Bc, K = 3, 2, 16, 1500, 128, 64, 5
    q, k, v, hc = make_prefill(_cfg(B, G * Hkv, Hkv, L, D, Bc, 1.5, seed=81))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    pre = dash.prefill(qd, kd, vd, hcd, Bc, enable_gqa=True, topk=K, return_p=True,
                       return_active_blocks=True)
    cap = L + 37
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    kc[:, :, :L] = kd
    vc[:, :, :L] = vd
    cache = torch.zeros(B, Hkv, cap // Bc, D, device=dev)
    lens = [L, Bc * 4 + 3, 100]
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    dash.update_chunk_cache(kc, hcd, seq, cache, heads_q=G * Hkv, chunk_size=Bc, n_recent=cap // Bc)
    qs = torch.stack([qd[b, :, lens[b] - 1] for b in range(B)])
    ws = dash.workspace(256, dev)
    dec = dash.decode(qs, kc, vc, seq, cache, Bc, enable_gqa=True, topk=K, return_p=True,
                      return_active_blocks=True, ws=ws)
    torch.cuda.synchronize()
    assert dash.read_device_status(ws) == 0
    C = (L + Bc - 1) // Bc
    for b in range(B):
        t = lens[b] - 1
        assert torch.equal(dec["p"][b, :, :C], pre["p"][b, :, t])
        assert torch.equal(dec["active_blocks"][b, :, :(C + 63) // 64], pre["active_blocks"][b, :, t])
    ref = oracle.decode(qs.cpu(), kc.cpu(), vc.cpu(), hc, lens, Bc, 1.5, topk=K)
    check_output(dec["out"].cpu().float().numpy(), ref["O"], tag="decode topk")


# ------------------------------------------------------------------------------ paged KV cache
def test_paged_decode_equals_contiguous_decode(dash):
    """A paged cache (pages of one chunk, a per-sequence block table with the pages scattered
    through the pools) gives the contiguous cache's summaries, routing and output bit for bit,
    and the oracle's output on the gathered cache; a page index outside the pools is reported
    through the status word."""
    B, Hkv, G, D, Bc = 3, 2, 16, 128, 64
    max_blocks = 24
    cap = max_blocks * Bc
    q, k, v, hc = make_prefill(_cfg(B, G * Hkv, Hkv, cap, D, Bc, 1.5, seed=85))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    lens = [cap, Bc * 7 + 5, 64]
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    n_pages = B * max_blocks + 5
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(3))[:B * max_blocks]
    table = perm.view(B, max_blocks).to(torch.int32).to(dev)
    k_pool = torch.zeros(n_pages, Hkv, Bc, D, dtype=torch.bfloat16, device=dev)
    v_pool = torch.zeros_like(k_pool)
    for b in range(B):
        for c in range(max_blocks):
            k_pool[table[b, c]] = kd[b, :, c * Bc:(c + 1) * Bc]
            v_pool[table[b, c]] = vd[b, :, c * Bc:(c + 1) * Bc]
    s_pool = torch.zeros(n_pages, Hkv, D, device=dev)
    dash.update_chunk_cache_paged(k_pool, hcd, table, seq, s_pool, G * Hkv, Bc, n_recent=max_blocks)
    cache = torch.zeros(B, Hkv, max_blocks, D, device=dev)
    dash.update_chunk_cache(kd, hcd, seq, cache, heads_q=G * Hkv, chunk_size=Bc, n_recent=max_blocks)
    qs = torch.stack([qd[b, :, lens[b] - 1] for b in range(B)])
    ws = dash.workspace(256, dev)
    for kw in (dict(), dict(topk=3), dict(estimate_diagonal=True, head_cls=hcd)):
        pg = dash.decode_paged(qs, k_pool, v_pool, table, seq, s_pool, Bc, return_p=True,
                               return_active_blocks=True, ws=ws, **kw)
        ct = dash.decode(qs, kd, vd, seq, cache, Bc, return_p=True, return_active_blocks=True, **kw)
        torch.cuda.synchronize()
        assert dash.read_device_status(ws) == 0
        for key in ("out", "p", "active_blocks"):
            assert torch.equal(pg[key], ct[key]), (kw, key)
    for b in range(B):
        for c in range(lens[b] // Bc):
            assert torch.equal(s_pool[table[b, c]], cache[b, :, c])
    ref = oracle.decode(qs.cpu(), k, v, hc, lens, Bc, 1.5)
    out = dash.decode_paged(qs, k_pool, v_pool, table, seq, s_pool, Bc, ws=ws)
    torch.cuda.synchronize()
    check_output(out.cpu().float().numpy(), ref["O"], tag="paged decode")
    bad = table.clone()
    bad[1, 2] = n_pages + 7
    dash.decode_paged(qs, k_pool, v_pool, bad, seq, s_pool, Bc, ws=ws)
    assert dash.read_device_status(ws) == 1


# ------------------------------------------------------------------------------ fused route-and-attend
@pytest.mark.parametrize("alpha", [1.0, 1.5, 2.0, 1.25])
@pytest.mark.parametrize("G,Bc,T", [(16, 64, 2100 + 37), (8, 128, 1500 + 3), (32, 64, 1300),
                                    (4, 64, 1500 + 3), (2, 128, 900)])
def test_fused_route_and_attend_equals_the_separate_stages(dash, alpha, G, Bc, T):
    """dash_prefill with DASH_FLAG_FUSE_ROUTE runs Stage 1 inside the 128-key-block Stage 2
    kernel (each tile routes its own tokens with Stage 1's arithmetic).  Its mask, p and output
    equal those of the separate Stage 1 and Stage 2 launches bit for bit, and the oracle's;
    the sliced prefill from host memory with the same flag gives the same output."""
    Hkv = 2 if G <= 16 else 1
    q, k, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, 128, Bc, alpha, seed=95 + G))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    prm = dash.make_params(1, G * Hkv, Hkv, T, 128, Bc, alpha, enable_gqa=True, flags=dash.FLAG_FUSE_ROUTE)
    # With G < 8 the full-range call chooses its Stage 2 kernel at run time and is not fused;
    # the sliced prefill from host memory below still routes inside the kernel.
    if G >= 8:
        assert dash.prefill_kernel_count(prm, dash.prefill_workspace_size(prm)) == 3   # no Stage 1 launch
    res = dash.prefill(qd, kd, vd, hcd, Bc, alpha, enable_gqa=True, return_p=True,
                       return_active_blocks=True, return_summary=True, fuse_route=True)
    r = dash.route(qd, res["summary"], Hkv, Bc, alpha)
    o = dash.attend(qd, kd, vd, res["summary"], r["tau"], r["active_blocks"], Bc, alpha)
    torch.cuda.synchronize()
    assert dash.read_device_status(res["ws"]) == 0
    assert torch.equal(res["active_blocks"], r["active_blocks"])
    assert torch.equal(res["p"], r["p"])
    assert torch.equal(res["out"], o)
    ref = oracle.prefill(q, k, v, hc, Bc, alpha)
    C = ref["p"].shape[-1]
    check_routing(unpack_mask(res["active_blocks"], C), res["p"].cpu().double().numpy(),
                  ref["p"], ref["m"], np.arange(T), Bc, alpha, tag="fused")
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag="fused")
    hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    dash.prefill_host(hq, hk, hv, hhc, ho, qd.clone(), kd.clone(), vd.clone(), hcd.clone(),
                      torch.empty_like(qd), Bc, alpha, enable_gqa=True, n_slices=3, fuse_route=True)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(ho, res["out"].cpu())


# ------------------------------------------------------------------------------ backward
def _grad_check(name, got, ref, rel_max=2e-2, rel_mean=2e-3):
    """Gradient parity: errors measured against the largest reference magnitude (the gradients
    sum many terms, each rounded to bf16 on its way into the warp-level MMAs)."""
    got = np.asarray(got, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{name}: non-finite"
    assert err.max() <= rel_max * scale, f"{name}: max err {err.max():.3e} vs scale {scale:.3e}"
    assert err.mean() <= rel_mean * scale, f"{name}: mean err {err.mean():.3e} vs scale {scale:.3e}"
    return err.max() / scale


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.0])
@pytest.mark.parametrize("G,D,Bc,T", [(16, 128, 64, 700), (4, 128, 128, 600 + 7), (1, 64, 64, 333),
                                      (32, 128, 64, 400)])
def test_backward_matches_oracle(dash, alpha, G, D, Bc, T):
    """The gradients of sum(out * dout) w.r.t. q, k, v and head_cls through Stages 2, 1 and 0
    (dash_backward) against the oracle's backward."""
    Hkv = 2 if G <= 16 else 1
    q, k, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, D, Bc, alpha, seed=110 + G))
    g_ = torch.Generator().manual_seed(7)
    dout = torch.randn(q.shape, generator=g_).to(torch.bfloat16)
    qd, kd, vd, hcd, dd = _to(q, k, v, hc, dout)
    out = dash.prefill(qd, kd, vd, hcd, Bc, alpha, enable_gqa=True)
    gr = dash.backward(qd, kd, vd, hcd, out, dd, Bc, alpha)
    torch.cuda.synchronize()
    assert dash.read_device_status(gr["ws"]) == 0
    ref = oracle.backward(q, k, v, hc, dout, Bc, alpha)
    for name, key in (("dq", "dQ"), ("dk", "dK"), ("dv", "dV"), ("dhc", "dhc")):
        _grad_check(f"{name} G={G} a={alpha}", gr[name].cpu().numpy(), ref[key])


# ------------------------------------------------------------------------------ run-time choice
@pytest.mark.parametrize("alpha,Bc,T", [(1.25, 64, 1500), (2.0, 64, 1500), (1.25, 128, 1400 + 7),
                                        (2.0, 128, 2100)])
def test_stage2_choice_at_run_time(dash, alpha, Bc, T):
    """G = 4 routed prefill: a cost kernel picks the 128-key-block or the warp-MMA Stage 2 from
    the mask.  The output matches the oracle and equals, bit for bit, the chosen kernel run on
    its own: the warp kernel through dash_attend without V^T room, the 128-key-block kernel
    through the sliced host prefill (row slices always take it)."""
    G, Hkv, D = 4, 2, 128
    q, k, v, hc = make_prefill(_cfg(1, G * Hkv, Hkv, T, D, Bc, alpha, n_max=12, seed=130 + T))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    prm = dash.make_params(1, G * Hkv, Hkv, T, D, Bc, alpha, enable_gqa=True)
    assert dash.attend_kernel_name(prm, dash.prefill_workspace_size(prm)) == "k_attend_fa|k_attend"
    res = dash.prefill(qd, kd, vd, hcd, Bc, alpha, enable_gqa=True, return_active_blocks=True)
    ran = dash.stage2_kernel_ran(res["ws"])
    assert ran in ("k_attend_fa", "k_attend")
    assert dash.read_device_status(res["ws"]) == 0
    ref = oracle.prefill(q, k, v, hc, Bc, alpha)
    check_output(res["out"].cpu().float().numpy(), ref["O"], tag=f"run-time choice {ran}")
    if ran == "k_attend":
        S = dash.stage0(kd, hcd, Bc)
        r = dash.route(qd, S, Hkv, Bc, alpha)
        o = dash.attend(qd, kd, vd, S, r["tau"], r["active_blocks"], Bc, alpha, ws=dash.workspace(256, dev))
        assert dash.attend_kernel_name(prm, 256) == "k_attend"
    else:
        hq, hk, hv, hhc = (x.contiguous().pin_memory() for x in (q, k, v, hc))
        ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        dash.prefill_host(hq, hk, hv, hhc, ho, qd.clone(), kd.clone(), vd.clone(), hcd.clone(),
                          torch.empty_like(qd), Bc, alpha, enable_gqa=True, n_slices=3)
        torch.cuda.current_stream().synchronize()
        o = ho
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), res["out"].cpu())


# ------------------------------------------------------------------------------ decode step
@pytest.mark.parametrize("kw", [dict(), dict(estimate_diagonal=True), dict(topk=4)])
def test_decode_step_equals_append_update_and_decode(dash, kw):
    """dash_decode_step (append the new K/V, route, attend, summarise a completed chunk,
    increment seq_lens, one launch) over 70 steps of three ragged sequences, each crossing
    chunk boundaries, equals bit for bit the separate path (K/V rows written by the host,
    dash_update_chunk_cache, dash_decode): outputs and routing every step, caches, summaries
    and lengths at the end; the paged step equals the contiguous one."""
    B, Hkv, G, D, Bc = 3, 2, 16, 128, 64
    max_blocks = 24
    cap = max_blocks * Bc
    steps = 70
    q, k, v, hc = make_prefill(_cfg(B, G * Hkv, Hkv, cap, D, Bc, 1.5, seed=87))
    qd, kd, vd, hcd = _to(q, k, v, hc)
    L0 = [Bc * 11 + 3, Bc * 5 - 1, 17]
    # separate path (A), fused step (Bc), fused step on pages (Bp)
    kA, vA = torch.zeros_like(kd), torch.zeros_like(vd)
    for b in range(B):
        kA[b, :, :L0[b]] = kd[b, :, :L0[b]]
        vA[b, :, :L0[b]] = vd[b, :, :L0[b]]
    kB, vB = kA.clone(), vA.clone()
    seqA = torch.tensor(L0, dtype=torch.int32, device=dev)
    seqB, seqP = seqA.clone(), seqA.clone()
    cA = torch.zeros(B, Hkv, max_blocks, D, device=dev)
    dash.update_chunk_cache(kA, hcd, seqA, cA, heads_q=G * Hkv, chunk_size=Bc, n_recent=max_blocks)
    cB = cA.clone()
    n_pages = B * max_blocks + 3
    table = torch.randperm(n_pages, generator=torch.Generator().manual_seed(5))[:B * max_blocks]
    table = table.view(B, max_blocks).to(torch.int32).to(dev)
    kP = torch.zeros(n_pages, Hkv, Bc, D, dtype=torch.bfloat16, device=dev)
    vP = torch.zeros_like(kP)
    sP = torch.zeros(n_pages, Hkv, D, device=dev)
    for b in range(B):
        for c in range(max_blocks):
            kP[table[b, c]] = kA[b, :, c * Bc:(c + 1) * Bc]
            vP[table[b, c]] = vA[b, :, c * Bc:(c + 1) * Bc]
            sP[table[b, c]] = cA[b, :, c]
    wsA, wsU = (dash.workspace(4096, dev) for _ in range(2))
    wsB, wsP = (torch.zeros(4096, dtype=torch.uint8, device=dev) for _ in range(2))   # step: zeroed once
    hk = hcd if kw.get("estimate_diagonal") else None
    for s in range(steps):
        pos = [L0[b] + s for b in range(B)]
        qs = torch.stack([qd[b, :, pos[b]] for b in range(B)])
        kn = torch.stack([kd[b, :, pos[b]] for b in range(B)])
        vn = torch.stack([vd[b, :, pos[b]] for b in range(B)])
        for b in range(B):
            kA[b, :, pos[b]] = kn[b]
            vA[b, :, pos[b]] = vn[b]
        seqA += 1
        dash.update_chunk_cache(kA, hcd, seqA, cA, heads_q=G * Hkv, chunk_size=Bc, n_recent=1, ws=wsU)
        ra = dash.decode(qs, kA, vA, seqA, cA, Bc, return_p=True, return_active_blocks=True, ws=wsA,
                         head_cls=hk, **kw)
        rb = dash.decode_step(qs, kn, vn, kB, vB, seqB, cB, hcd, Bc, return_p=True,
                              return_active_blocks=True, ws=wsB, **kw)
        rp = dash.decode_step(qs, kn, vn, kP, vP, seqP, sP, hcd, Bc, return_p=True,
                              return_active_blocks=True, ws=wsP, block_table=table, **kw)
        for key in ("out", "p", "active_blocks"):
            assert torch.equal(ra[key], rb[key]), (s, key)
            assert torch.equal(rb[key], rp[key]), (s, key, "paged")
    torch.cuda.synchronize()
    for ws in (wsA, wsB, wsP, wsU):
        assert dash.read_device_status(ws) == 0
    for ws in (wsB, wsP):                     # every step left its arrival counters at zero
        assert not ws[32:32 + 4 * B].any()
    assert torch.equal(seqA, seqB) and torch.equal(seqA, seqP)
    assert torch.equal(kA, kB) and torch.equal(vA, vB) and torch.equal(cA, cB)
    for b in range(B):
        for c in range(int(seqA[b]) // Bc):
            assert torch.equal(sP[table[b, c]], cA[b, :, c])
            assert torch.equal(kP[table[b, c]], kA[b, :, c * Bc:(c + 1) * Bc])
    # a step past the capacity is refused on the device and leaves the sequence unchanged
    full = torch.tensor([cap, 5, 5], dtype=torch.int32, device=dev)
    dash.decode_step(qs, kn, vn, kB, vB, full, cB, hcd, Bc, ws=wsB)
    # the status word is not cleared by a step: the error stays through a clean step after it
    dash.decode_step(qs, kn, vn, kB, vB, torch.tensor([5, 5, 5], dtype=torch.int32, device=dev),
                     cB, hcd, Bc, ws=wsB)
    assert dash.read_device_status(wsB) == 1
    assert dash.read_device_status(wsB) == 0
    assert full[0].item() == cap and full[1].item() == 6
    assert not wsB[32:32 + 4 * B].any()
