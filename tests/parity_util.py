"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (fixed by the library's specification):
  * active-block mask: bit-exact, except a routed chunk whose oracle margin
    m = (alpha-1) s - tau satisfies |m| <= (1e-6)^(alpha-1), i.e. whose would-be probability
    |m|^(1/(alpha-1)) is within 1e-6 of zero on either side of the threshold; the diagonal
    bit and the bits above it are never excused;
  * routing probabilities p: <= 1e-4 absolute;
  * bf16 output O: <= 2e-2 max absolute and <= 5e-3 mean absolute error.
"""
import numpy as np
import torch

P_TOL = 1e-4
O_MAX_TOL = 2e-2
O_MEAN_TOL = 5e-3


def unpack_mask(words: torch.Tensor, C: int) -> np.ndarray:
    """int64 words [..., W] (bit c%64 of word c//64, LSB first) -> bool [..., C]."""
    w = np.ascontiguousarray(words.detach().cpu().numpy()).view(np.uint64)
    bits = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")
    return bits[..., :C].astype(bool)


def check_routing(mask_bits, p_gpu, p_or, m_or, rows, chunk_size, alpha, tag=""):
    """mask_bits, p_gpu, p_or, m_or: [..., nrows, C] arrays for the given rows.  Returns the
    number of excused mismatches; raises AssertionError on any other discrepancy."""
    rows = np.asarray(rows)
    C = p_or.shape[-1]
    ct = rows // chunk_size                                   # [nrows]
    col = np.arange(C)
    routed = col[None, :] < ct[:, None]                       # [nrows, C]
    diag = col[None, :] == ct[:, None]
    above = col[None, :] > ct[:, None]
    want = (p_or > 0) & routed
    assert mask_bits[..., diag].all(), f"{tag}: diagonal bit missing"
    assert not mask_bits[..., above].any(), f"{tag}: bit above the diagonal set"
    bad = (mask_bits != want) & routed
    n_excused = 0
    if bad.any():
        if alpha == 1.0:
            raise AssertionError(f"{tag}: {int(bad.sum())} mask mismatches with softmax routing")
        band = (1e-6) ** (alpha - 1.0)
        unexcused = bad & ~(np.abs(m_or) <= band)
        if unexcused.any():
            idx = np.argwhere(unexcused)[:5]
            raise AssertionError(f"{tag}: {int(unexcused.sum())} unexcused mask mismatches, "
                                 f"e.g. {idx.tolist()} margins {m_or[unexcused][:5]}")
        n_excused = int(bad.sum())
    if p_gpu is not None:
        err = np.abs(p_gpu - p_or)
        assert err.max() <= P_TOL, f"{tag}: p max abs err {err.max():.3e}"
    return n_excused


def check_output(o_gpu, o_or, tag=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_or)
    assert np.isfinite(o_gpu).all(), f"{tag}: non-finite output"
    assert err.max() <= O_MAX_TOL, f"{tag}: O max abs err {err.max():.3e}"
    assert err.mean() <= O_MEAN_TOL, f"{tag}: O mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_topk(mask_bits, p_gpu, p_or, m_or, rows, chunk_size, k, tol=1e-4, tag=""):
    """Top-k routing: every row selects min(k, c_t) routed chunks plus its diagonal; the
    selection is a valid top-k of the oracle's scores up to `tol` (a selected chunk's oracle
    margin s - theta >= -tol, an unselected one's <= tol: near-ties may fall either way under
    fp32 rounding), and p is uniform over it.  Returns the boolean per-row mask of rows whose
    selection equals the oracle's exactly."""
    rows = np.asarray(rows)
    C = p_or.shape[-1]
    ct = rows // chunk_size
    col = np.arange(C)
    routed = col[None, :] < ct[:, None]
    diag = col[None, :] == ct[:, None]
    above = col[None, :] > ct[:, None]
    assert mask_bits[..., diag].all(), f"{tag}: diagonal bit missing"
    assert not mask_bits[..., above].any(), f"{tag}: bit above the diagonal set"
    sel = mask_bits & routed
    ke = np.minimum(k, ct)
    assert (sel.sum(-1) == ke).all(), f"{tag}: selection sizes differ from min(k, c_t)"
    m = np.where(routed, m_or, 0.0)
    assert (m[sel] >= -tol).all(), f"{tag}: a selected chunk lies below the k-th score"
    assert (m[routed & ~sel] <= tol).all(), f"{tag}: an unselected chunk lies above the k-th score"
    want = np.where(sel, 1.0 / np.maximum(ke, 1)[:, None], 0.0)
    if p_gpu is not None:
        assert np.abs(p_gpu - want).max() <= 1e-6, f"{tag}: p is not uniform over the selection"
    return (sel == ((p_or > 0) & routed)).all(-1)
