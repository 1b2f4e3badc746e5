"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the scoring path's stated bar): support masks, valid rows,
support sizes and status bits bit-exact; logprobs within 1e-4 absolute;
entropies and L1 within 1e-4 relative (exact zeros exactly zero); gradients
within 2e-3 relative, per row in the 2-norm and per element against the
row's largest magnitude.

Top-p and min-p decide set membership from floating-point sums.  Rows whose
oracle crossing lies within 1e-6 of top_p (or whose min-p ratio lies within
1e-6 relative of min_p) are counted as boundary rows: for them the GPU's
support must still be a prefix of the oracle's total order whose mass is
within the band, and its scores must equal the oracle's scores of that
support.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

LP_ATOL = 1e-4
H_RTOL = 1e-4
G_RTOL = 2e-3
BAND = 1e-6

# oracle status bit -> library status bit
STATUS_MAP = {
    oracle.TARGET_OUT_OF_RANGE: 1 << 0,
    oracle.TARGET_NOT_IN_SUPPORT: 1 << 1,
    oracle.BAD_SUPPORT_ID: 1 << 2,
    oracle.DUP_SUPPORT_ID: 1 << 3,
    oracle.NONFINITE_INPUT: 1 << 4,
}


def map_status(s):
    out = np.zeros_like(s, dtype=np.int64)
    for ob, lb in STATUS_MAP.items():
        out |= np.where(s & ob, lb, 0)
    return out


def to_device(a: np.ndarray, dev="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def unpack_mask(words: torch.Tensor, vocab: int) -> np.ndarray:
    w = words.cpu().numpy().astype(np.int32).view(np.uint32)
    bits = np.unpackbits(w.view(np.uint8), bitorder="little").reshape(w.shape[0], -1)
    return bits[:, :vocab].astype(np.uint8)


def _z(logits: np.ndarray, vocab: int, temperature) -> np.ndarray:
    """Tempered logits in fp64 (for ordering checks of boundary rows)."""
    x = logits[:, :vocab]
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << 16).view(np.float32)
    t = np.broadcast_to(np.asarray(temperature, dtype=np.float64), (x.shape[0],))
    return x.astype(np.float64) / t[:, None]


def assert_close_rel(got, want, rtol, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    zero = want == 0.0
    assert np.all(got[zero] == 0.0), f"{what}: exact zeros not exactly zero"
    nz = ~zero
    rel = np.abs(got[nz] - want[nz]) / np.abs(want[nz])
    assert rel.size == 0 or rel.max() <= rtol, f"{what}: max rel {rel.max():.3g}"


def compare_scores(out, ref, logits, vocab, temperature, targets, top_k, top_p, min_p,
                   check_full=True, check_entropy=True):
    """Compare a vs_score_fwd result with the oracle; returns the number of
    boundary rows."""
    rows = len(ref["lp_full"])
    band = (ref["topp_margin"] < BAND) | (ref["minp_margin"] < BAND)
    gsize = out["support_size"].cpu().numpy()
    assert np.array_equal(out["valid"].cpu().numpy(), ref["valid"]), "valid"
    status = out["status"].cpu().numpy().astype(np.int64)
    assert np.all((status & (1 << 5)) == 0), "device wait timed out"
    lps = out["lp_support"].cpu().numpy().astype(np.float64)
    hs = out["h_support"].cpu().numpy() if check_entropy else None
    if check_full:
        lpf = out["lp_full"].cpu().numpy().astype(np.float64)
        fin = np.isfinite(ref["lp_full"])
        assert np.array_equal(np.isfinite(lpf), fin), "lp_full finiteness"
        assert np.abs(lpf[fin] - ref["lp_full"][fin]).max(initial=0) <= LP_ATOL, "lp_full"
        if check_entropy:
            hf = out["h_full"].cpu().numpy()
            ok = np.isfinite(ref["h_full"])
            assert np.array_equal(np.isfinite(hf), ok)
            assert_close_rel(hf[ok], ref["h_full"][ok], H_RTOL, "h_full")
    mask = unpack_mask(out["mask"], vocab) if "mask" in out else None
    sure = ~band
    assert np.array_equal(gsize[sure], ref["support_size"][sure]), "support_size"
    assert np.array_equal(status[sure], map_status(ref["status"][sure])), "status"
    if mask is not None:
        assert np.array_equal(mask[sure], ref["mask"][sure]), "support mask"
    fin = np.isfinite(ref["lp_support"]) & sure
    assert np.array_equal(np.isfinite(lps[sure]), np.isfinite(ref["lp_support"][sure])), "lp_S finiteness"
    assert np.all((lps[sure] == -np.inf) == (ref["lp_support"][sure] == -np.inf))
    assert np.abs(lps[fin] - ref["lp_support"][fin]).max(initial=0) <= LP_ATOL, "lp_support"
    if check_entropy:
        ok = np.isfinite(ref["h_support"]) & sure
        assert_close_rel(hs[ok], ref["h_support"][ok], H_RTOL, "h_support")
    # boundary rows: the GPU support is a valid prefix of the total order
    if band.any():
        assert mask is not None, "boundary rows need the mask to be checked"
        z = _z(logits, vocab, temperature)
        for i in np.nonzero(band)[0]:
            order = np.lexsort((np.arange(vocab), -z[i]))
            n = int(gsize[i])
            assert mask[i].sum() == n
            assert np.all(mask[i][order[:n]] == 1), "boundary row support is not a prefix"
            assert abs(n - ref["support_size"][i]) <= max(4, ref["support_size"][i] // 100)
            ids = np.nonzero(mask[i])[0].astype(np.int32)[None, :]
            t_i = float(np.broadcast_to(np.asarray(temperature, np.float64), (rows,))[i])
            r2 = oracle.score(logits[i:i + 1], targets[i:i + 1], temperature=t_i, support=ids,
                              vocab=vocab)
            if np.isfinite(r2["lp_support"][0]):
                assert abs(lps[i] - r2["lp_support"][0]) <= LP_ATOL
            if check_entropy:
                assert_close_rel(hs[i:i + 1], r2["h_support"], H_RTOL, "h_support (boundary)")
    return int(band.sum())


def compare_grad(g_gpu, g_ref, exclude=None, rtol=G_RTOL, what="grad"):
    g = np.asarray(g_gpu, np.float64)
    r = np.asarray(g_ref, np.float64)
    if exclude is not None:
        g = np.where(exclude, 0.0, g)
        r = np.where(exclude, 0.0, r)
    nr = np.linalg.norm(r, axis=1)
    diff = np.linalg.norm(g - r, axis=1)
    zero_rows = nr == 0
    assert np.all(diff[zero_rows] == 0.0), f"{what}: rows with zero gradient are not zero"
    nz = ~zero_rows
    if nz.any():
        rel = diff[nz] / nr[nz]
        assert rel.max() <= rtol, f"{what}: max row rel {rel.max():.3g}"
        amax = np.abs(r[nz]).max(axis=1, keepdims=True)
        el = np.abs(g[nz] - r[nz]) / amax
        assert el.max() <= rtol, f"{what}: max elementwise rel {el.max():.3g}"
