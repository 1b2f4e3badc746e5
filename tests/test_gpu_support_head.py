"""GPU parity of vs_support_lmhead_score (support-only fused projection)
against the fp64 oracle: the oracle materialises z = (H W^T) / T in fp64 for
the checked rows and scores the recorded support on it.  The projection
path has no full-vocabulary fallback, so rows with no kept id are checked
against their own rule (lp_S NaN, entropy 0, valid 0, ROW_EMPTY_SUPPORT)."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import LP_ATOL, assert_close_rel, map_status, to_device

pytestmark = pytest.mark.gpu


def _case(rows, vocab, hidden, width, seed, sh=1.0, sw=0.05):
    h = workloads.to_bf16_bits(workloads.normal((rows, hidden), sh, seed, stream=1))
    w = workloads.to_bf16_bits(workloads.normal((vocab, hidden), sw, seed, stream=2))
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, vocab, (rows, width)).astype(np.int32)
    widths = rng.integers(0, width + 1, rows)
    for i in range(rows):
        ids[i, widths[i]:] = -1
    y = workloads.integers(rows, 0, vocab, seed, 3).astype(np.int32)
    # half of the targets inside their support
    for i in range(0, rows, 2):
        if widths[i] > 0:
            y[i] = ids[i, rng.integers(0, widths[i])]
    return h, w, ids, y


def _check(h, w, ids, y, T, rows_checked=None):
    rows, hidden = h.shape
    vocab, width = w.shape[0], ids.shape[1]
    t_dev = torch.from_numpy(np.asarray(T, np.float32)).cuda() if np.ndim(T) else float(T)
    out = vsb.support_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(), t_dev,
                                   torch.from_numpy(ids).cuda(), want_logits=True)
    torch.cuda.synchronize()
    get = {k: v.cpu().numpy() for k, v in out.items()}
    sel = np.arange(rows) if rows_checked is None else np.asarray(rows_checked)
    t64 = np.broadcast_to(np.asarray(T, np.float32).astype(np.float64), (rows,))[sel]
    z = oracle.lmhead_logits(h, w, sel.astype(np.int32), 1.0) / t64[:, None]
    ref = oracle.score(z, y[sel], support=ids[sel])
    empty = ref["support_size"] == 0
    st = get["status"][sel].astype(np.int64)
    assert np.all((st & vsb.ROW_DEVICE_TIMEOUT) == 0)
    # support logits: z at kept slots, -inf elsewhere
    lg = get["support_logits"][sel].astype(np.float64)
    for r, i in enumerate(sel):
        seen = set()
        for s in range(width):
            sid = int(ids[i, s])
            if 0 <= sid < vocab and sid not in seen:
                seen.add(sid)
                assert abs(lg[r, s] - z[r, sid]) <= 1e-5 * max(1.0, abs(z[r, sid])), (i, s)
            else:
                assert lg[r, s] == -np.inf, (i, s)
    # rows with a kept id: the recorded-support definitions
    ne = ~empty
    assert np.array_equal(get["valid"][sel][ne], ref["valid"][ne])
    assert np.array_equal(get["support_size"][sel], ref["support_size"])
    assert np.array_equal(st[ne], map_status(ref["status"][ne]))
    lps = get["lp_support"][sel].astype(np.float64)
    want = ref["lp_support"]
    assert np.array_equal(lps[ne] == -np.inf, want[ne] == -np.inf)
    fin = ne & np.isfinite(want)
    assert np.abs(lps[fin] - want[fin]).max(initial=0) <= LP_ATOL
    hs = get["h_support"][sel]
    assert_close_rel(hs[ne], ref["h_support"][ne], 1e-4, "h_support")
    assert np.all(hs[ne & (ref["support_size"] == 1)] == 0.0)  # singletons: exactly zero
    # rows with no kept id
    assert np.all(np.isnan(lps[empty]))
    assert np.all(hs[empty] == 0.0)
    assert np.all(get["valid"][sel][empty] == 0)
    assert np.all((st[empty] & vsb.ROW_EMPTY_SUPPORT) != 0)
    assert np.array_equal(st[empty] & ~vsb.ROW_EMPTY_SUPPORT,
                          map_status(ref["status"][empty]) & ~vsb.ROW_EMPTY_SUPPORT)
    assert np.all((st[ne] & vsb.ROW_EMPTY_SUPPORT) == 0)
    return int(empty.sum())


def test_support_head_small_ragged():
    # hidden a multiple of 8 but not of 256 (tail of the dot-product loop)
    h, w, ids, y = _case(130, 3000, 200, 16, seed=1)
    ids[3, :] = -1                      # empty row
    ids[5, :] = [7] + [-1] * 15         # singleton
    y[5] = 7
    ids[6, :4] = [9, 9, 11, 9]          # repeated ids
    ids[8, :3] = [-5, 3000, 12]         # bad ids
    ids[10, 2] = -1                     # pad in the middle
    y[12] = -1                          # target out of range
    y[14] = 3000
    _check(h, w, ids, y, 0.8)


@pytest.mark.parametrize("width", [1, 64, 300])
def test_support_head_widths_and_row_temperatures(width):
    rows = 40
    h, w, ids, y = _case(rows, 5000, 512, width, seed=10 + width, sh=2.0, sw=0.03)
    T = workloads.uniform(rows, 0.5, 1.5, 10 + width, 4).astype(np.float32)
    _check(h, w, ids, y, T)


def test_support_head_duplicated_weight_rows_tie_exactly():
    """Equal weight rows give bitwise-equal support logits; a support of k
    such ids has entropy log k and logprob -log k."""
    h, w, ids, y = _case(8, 600, 64, 8, seed=5)
    w[[20, 21, 22, 23]] = w[20]
    ids[:] = -1
    ids[:, :4] = [20, 21, 22, 23]
    y[:] = 22
    out = vsb.support_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(), 1.0,
                                   torch.from_numpy(ids).cuda(), want_logits=True)
    torch.cuda.synchronize()
    lg = out["support_logits"].cpu().numpy()
    assert np.all(lg[:, :4] == lg[:, :1])
    assert np.allclose(out["lp_support"].cpu().numpy(), -np.log(4.0), atol=1e-6)
    assert np.allclose(out["h_support"].cpu().numpy(), np.log(4.0), rtol=1e-6)


def test_support_head_zero_width_and_zero_rows():
    h, w, ids, y = _case(4, 100, 64, 1, seed=3)
    out = vsb.support_lmhead_score(to_device(h), to_device(w), torch.from_numpy(y).cuda(), 1.0,
                                   torch.from_numpy(np.zeros((4, 0), np.int32)).cuda())
    torch.cuda.synchronize()
    assert np.all(np.isnan(out["lp_support"].cpu().numpy()))
    assert np.all((out["status"].cpu().numpy() & vsb.ROW_EMPTY_SUPPORT) != 0)
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    vsb.support_lmhead_score(e, to_device(w), torch.empty(0, dtype=torch.int32, device="cuda"), 1.0,
                             torch.empty((0, 8), dtype=torch.int32, device="cuda"))


@pytest.mark.slow
def test_support_head_workload_full_size_sampled_rows():
    """The support-only projection workload (8,192 rows, hidden 4,096, V =
    151,936, replay-recipe supports): sampled rows against the oracle."""
    wl = workloads.lmhead()
    sup = workloads.support_lists()
    sel = np.sort(np.random.default_rng(1).choice(wl["rows"], 12, replace=False))
    sel[0] = int(np.nonzero(sup["widths"] == 0)[0][0])  # one empty row
    sel[1] = int(np.nonzero(sup["widths"] == 1)[0][0])  # one singleton
    _check(wl["hidden_states"], wl["weight"], sup["support"], sup["targets"], wl["temperature"],
           rows_checked=np.sort(sel))
