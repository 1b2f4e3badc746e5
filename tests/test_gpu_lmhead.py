"""GPU parity of vs_fused_lmhead_score (tcgen05 projection + fused scoring)
against the fp64 oracle: the oracle materialises z = (H W^T) / T in fp64 for
the checked rows and runs the scoring program on it (top-k, then inclusive
top-p on the top-k mass, then min-p).

The GPU accumulates the K-long dot products in fp32, so its logits differ
from the fp64 ones by ~1e-6; top-k orders whose k-th and (k+1)-th logits lie
within 1e-4, and top-p / min-p decisions within 1e-5 of their thresholds, are
boundary rows: counted, and checked for validity instead of equality."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import LP_ATOL, assert_close_rel, to_device

pytestmark = pytest.mark.gpu

GAP = 1e-4
BAND = 1e-5


def _case(rows, vocab, hidden, seed, sh=1.0, sw=0.02):
    h = workloads.to_bf16_bits(workloads.normal((rows, hidden), sh, seed, stream=1))
    w = workloads.to_bf16_bits(workloads.normal((vocab, hidden), sw, seed, stream=2))
    y = workloads.integers(rows, 0, vocab, seed, 3).astype(np.int32)
    return h, w, y


def _check(h, w, y, T, k, p, mp, rows_checked=None):
    rows, hidden = h.shape
    vocab = w.shape[0]
    out = vsb.fused_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(), T, k,
                                 float(np.float32(p)), float(np.float32(mp)))
    torch.cuda.synchronize()
    sel = np.arange(rows) if rows_checked is None else np.asarray(rows_checked)
    z = oracle.lmhead_logits(h, w, sel.astype(np.int32), float(np.float32(T)))
    yy = y[sel]
    # a target inside the top-k for half of the rows, so lp_S is finite there
    ref = oracle.score(z, yy, top_k=k, top_p=float(np.float32(p)), min_p=float(np.float32(mp)),
                       want_mask=True)
    get = {kk: v.cpu().numpy() for kk, v in out.items()}
    assert np.all((get["status"][sel] & (1 << 5)) == 0), "device wait timed out"
    # full-vocabulary values never depend on decisions
    assert np.abs(get["lp_full"][sel] - ref["lp_full"]).max() <= LP_ATOL
    assert_close_rel(get["h_full"][sel], ref["h_full"], 1e-4, "h_full")
    # top-k ids in the total order
    order = np.argsort(-z, axis=1, kind="stable")[:, :k]
    amb = (ref["topk_gap"] < GAP) | (ref["topp_margin"] < BAND) | (ref["minp_margin"] < BAND)
    # near-ties anywhere inside the top-k also make the order ambiguous
    zs = np.take_along_axis(z, order, axis=1)
    inner = (np.diff(-zs, axis=1) < GAP).any(axis=1) if k > 1 else np.zeros(len(sel), bool)
    amb_ids = amb | inner
    ids = get["topk_ids"][sel]
    sure = ~amb_ids
    assert np.array_equal(ids[sure], order[sure]), "top-k ids"
    # top-k logprobs (full vocabulary) for every row
    lse = ref["lse_full"][:, None]
    want_lp = np.take_along_axis(z, np.clip(ids, 0, None), axis=1) - lse
    assert np.abs(get["topk_logprob"][sel] - want_lp).max() <= LP_ATOL
    s_ok = ~amb
    assert np.array_equal(get["support_size"][sel][s_ok], ref["support_size"][s_ok])
    assert np.array_equal(get["valid"][sel], ref["valid"])
    lps = get["lp_support"][sel].astype(np.float64)
    fin = np.isfinite(ref["lp_support"]) & s_ok
    assert np.array_equal(np.isfinite(lps[s_ok]), np.isfinite(ref["lp_support"][s_ok]))
    assert np.abs(lps[fin] - ref["lp_support"][fin]).max(initial=0) <= LP_ATOL
    assert_close_rel(get["h_support"][sel][s_ok], ref["h_support"][s_ok], 1e-4, "h_support")
    return int(amb.sum()), len(sel)


def test_fused_head_small_ragged():
    # rows not a multiple of 128, vocab not a multiple of 256
    h, w, y = _case(200, 5000, 256, seed=1)
    # targets drawn from each row's top-5 half of the time, by the oracle's own logits
    z = oracle.lmhead_logits(h, w, np.arange(200, dtype=np.int32), 0.8)
    top = np.argsort(-z, axis=1, kind="stable")
    y[::2] = top[::2, 2]
    nb, n = _check(h, w, y, 0.8, 20, 0.95, 0.02)
    print(f"fused head small: {nb} boundary rows of {n}")


@pytest.mark.parametrize("k,p,mp", [(1, 1.0, 0.0), (8, 0.5, 0.0), (64, 0.99, 0.1), (20, 1.0, 0.3)])
def test_fused_head_filters(k, p, mp):
    h, w, y = _case(130, 3000, 128, seed=2 + k, sh=2.0, sw=0.05)
    _check(h, w, y, 1.1, k, p, mp)


def test_fused_head_per_row_temperature_single_row():
    h, w, y = _case(1, 700, 64, seed=9)
    out = vsb.fused_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(),
                                 torch.tensor([0.7], device="cuda"), 5, 0.9, 0.0)
    torch.cuda.synchronize()
    z = oracle.lmhead_logits(h, w, np.array([0], np.int32), float(np.float32(0.7)))
    ref = oracle.score(z, y, top_k=5, top_p=float(np.float32(0.9)))
    assert abs(out["lp_full"].item() - ref["lp_full"][0]) <= LP_ATOL


@pytest.mark.slow
def test_lmhead_workload_full_size_sampled_rows():
    wl = workloads.lmhead()
    rows = wl["rows"]
    # one row in every 256-row unit (the pair-mode row block), at a seeded
    # offset, and the last row
    off = np.random.default_rng(0).integers(0, 256, rows // 256)
    sel = np.unique(np.concatenate([np.arange(rows // 256) * 256 + off, [rows - 1]]))
    nb, n = _check(wl["hidden_states"], wl["weight"], wl["targets"], wl["temperature"],
                   wl["top_k"], wl["top_p"], wl["min_p"], rows_checked=sel)
    print(f"lmhead full size: {nb} boundary rows of {n} checked")


# ids of two groups of duplicated weight rows.  Group A holds a block of 24
# consecutive ids inside one tile, so a top-k list fills with A entries tied
# at its minimum; group B (the larger logit) follows in the same tile and
# must evict the A entry with the largest id.  Both groups also straddle tile
# and split boundaries.
_TIE_A = list(range(1030, 1054)) + [2000, 2990]
_TIE_B = [1250, 2500, 2999]


@pytest.mark.parametrize("rows,vocab,k", [(130, 3000, 8), (130, 3000, 2), (2048, 4096, 20)])
def test_fused_head_exact_ties(rows, vocab, k):
    """Exactly tied logits (duplicated weight rows) come out in the total
    order, value descending then id ascending, across in-list evictions and
    the merge of vocabulary splits."""
    hidden = 64
    h, w, y = _case(rows, vocab, hidden, seed=31)
    h[:, 0] = 0x4080  # 4.0: the duplicated rows' logits stand far above the rest
    rest = w[7].copy()
    for ids, lead in ((_TIE_A, 0x3F80), (_TIE_B, 0x3FA0)):  # 1.0, 1.25
        w[ids] = rest
        w[ids, 0] = lead
    want = np.array(_TIE_B + _TIE_A, dtype=np.int32)
    n = min(k, len(want))
    out = vsb.fused_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(), 1.0, k,
                                 1.0, 0.0)
    torch.cuda.synchronize()
    ids = out["topk_ids"].cpu().numpy()
    lp = out["topk_logprob"].cpu().numpy()
    assert np.array_equal(ids[:, :n], np.broadcast_to(want[:n], (rows, n)))
    # a tie group shares one logprob bit for bit
    nb = min(n, len(_TIE_B))
    assert np.all(lp[:, :nb] == lp[:, :1])
    if n > nb:
        assert np.all(lp[:, nb:n] == lp[:, nb:nb + 1])
    sel = np.linspace(0, rows - 1, 16).astype(np.int64)
    _check(h, w, y, 1.0, k, 1.0, 0.0, rows_checked=sel)
