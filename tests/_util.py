"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the scoring path's stated bar): support masks, valid rows,
support sizes and status bits bit-exact; logprobs within 1e-4 absolute;
entropies and L1 within 1e-4 relative (exact zeros exactly zero); gradients
within 2e-3 relative, per row in the 2-norm and per element against the
row's largest magnitude.

Top-p and min-p decide set membership from floating-point sums.  Rows whose
oracle crossing lies within 1e-6 of top_p (or whose min-p ratio lies within
1e-6 relative of min_p) are counted as boundary rows.  For them the GPU's
support size n must name a prefix of the oracle's total order that the rules
allow within that band (boundary_prefix_ok: the first n - 1 entries hold
less than top_p + 1e-6 of the top-k mass; the n-th entry passes min-p within
the band; the prefix stops because it reached top_p - 1e-6, min-p drops the
next entry within the band, or it is the whole top-k set), the support mask
(when requested) must be exactly that prefix, and the scores and status must
equal the oracle's scores of that prefix.
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


def boundary_prefix_ok(n, facts, top_p, min_p, band=BAND):
    """True when a support of the first n entries of the total order is one
    the top-k / top-p / min-p rules allow with the top-p mass and the min-p
    ratio each known only to within `band` (facts: oracle.prefix of n)."""
    nk = int(facts["nk"])
    if n < 1 or n > nk:
        return False
    use_p, use_m = top_p < 1.0, min_p > 0.0
    if use_p and not facts["mass_prev"] < top_p + band:
        return False
    if use_m and not facts["ratio_n"] >= min_p * (1.0 - band):
        return False
    return bool(n == nk or (use_p and facts["mass_n"] >= top_p - band)
                or (use_m and facts["ratio_next"] < min_p * (1.0 + band)))


def _per_row(v, rows, dt):
    return np.broadcast_to(np.asarray(v, dt), (rows,))


def compare_scores(out, ref, logits, vocab, temperature, targets, top_k, top_p, min_p,
                   check_full=True, check_entropy=True):
    """Compare a vs_score_fwd result with the oracle, every row: exactly off
    the boundary band, by the prefix rule on it.  Returns (boundary rows,
    boundary rows whose support size differs from the oracle's)."""
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
    # boundary rows: the GPU support is a prefix the rules allow within the band
    idx = np.nonzero(band)[0]
    if idx.size == 0:
        return 0, 0
    t_all = _per_row(temperature, rows, np.float64)
    k_all = _per_row(top_k, rows, np.int32)
    p_all = _per_row(np.asarray(top_p, np.float32).astype(np.float64), rows, np.float64)
    m_all = _per_row(np.asarray(min_p, np.float32).astype(np.float64), rows, np.float64)
    facts = oracle.prefix(logits[idx], gsize[idx], temperature=np.ascontiguousarray(t_all[idx]),
                          top_k=np.ascontiguousarray(k_all[idx]), vocab=vocab, want_ids=True)
    differ = 0
    for a, i in enumerate(idx):
        n = int(gsize[i])
        f = {k: v[a] for k, v in facts.items() if k != "ids"}
        assert boundary_prefix_ok(n, f, p_all[i], m_all[i]), (
            f"row {i}: support size {n} is not a prefix the rules allow (oracle "
            f"{ref['support_size'][i]}, mass {f['mass_prev']:.9f}..{f['mass_n']:.9f}, "
            f"top_p {p_all[i]}, min_p {m_all[i]})")
        differ += int(n != ref["support_size"][i])
        ids = facts["ids"][a]
        if mask is not None:
            assert mask[i].sum() == n and np.all(mask[i][ids] == 1), \
                "boundary row mask is not the prefix"
        r2 = oracle.score(logits[i:i + 1], targets[i:i + 1], temperature=float(t_all[i]),
                          support=ids[None, :], vocab=vocab)
        assert status[i] == map_status(r2["status"])[0], f"row {i}: status (boundary)"
        if np.isfinite(r2["lp_support"][0]):
            assert abs(lps[i] - r2["lp_support"][0]) <= LP_ATOL, f"row {i}: lp_S (boundary)"
        else:
            assert lps[i] == r2["lp_support"][0], f"row {i}: lp_S (boundary)"
        if check_entropy:
            assert_close_rel(hs[i:i + 1], r2["h_support"], H_RTOL, "h_support (boundary)")
    return int(idx.size), differ


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
