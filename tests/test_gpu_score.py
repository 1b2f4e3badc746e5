"""GPU parity of vs_score_fwd / vs_score_bwd against the fp64 oracle, through
the C ABI, on seeded inputs: several tiles per row with ragged tails, bf16
and fp32, per-row parameters, edge cases, and the full-size workloads."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import LP_ATOL, compare_grad, compare_scores, map_status, to_device, unpack_mask

pytestmark = pytest.mark.gpu

F32 = np.float32


def _run(logits, targets, temperature, top_k=0, top_p=1.0, min_p=0.0, vocab=None,
         want_grad=False):
    """GPU forward (mask + entropy) and the oracle on the same inputs."""
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    dev = "cuda"
    t_np = np.asarray(temperature, F32)
    lg = to_device(logits)
    tg = torch.from_numpy(np.asarray(targets, np.int32)).to(dev)
    t_arg = torch.from_numpy(t_np).to(dev) if t_np.ndim else float(t_np)
    def dev_param(v, dt):
        return torch.from_numpy(np.asarray(v, dt)).to(dev) if np.ndim(v) else v
    out = vsb.score_fwd(lg, tg, temperature=t_arg, top_k=dev_param(top_k, np.int32),
                        top_p=dev_param(top_p, F32), min_p=dev_param(min_p, F32),
                        want_mask=True, want_grad=want_grad, vocab=vocab)
    torch.cuda.synchronize()
    t64 = t_np.astype(np.float64)
    ref = oracle.score(logits, targets, temperature=t64 if t64.ndim else float(t64),
                       top_k=top_k if np.ndim(top_k) == 0 else np.asarray(top_k, np.int32),
                       top_p=np.asarray(top_p, F32).astype(np.float64) if np.ndim(top_p)
                       else float(F32(top_p)),
                       min_p=np.asarray(min_p, F32).astype(np.float64) if np.ndim(min_p)
                       else float(F32(min_p)),
                       want_mask=True, vocab=vocab)
    nb = compare_scores(out, ref, logits, vocab, t64 if t64.ndim else np.full(rows, float(t64)),
                        np.asarray(targets, np.int32), top_k, top_p, min_p)
    return out, ref, nb


def test_tiny_workload():
    w = workloads.tiny()
    _run(w["logits"], w["targets"], w["temperature"], w["top_k"], w["top_p"], w["min_p"])


FILTERS = [(0, 1.0, 0.0), (0, 0.95, 0.0), (100, 1.0, 0.0), (0, 1.0, 0.05), (200, 0.9, 0.02),
           (1, 1.0, 0.0), (0, 1e-4, 0.0), (5000, 0.999, 0.0), (37, 0.5, 0.3)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("filt", FILTERS)
def test_ragged_rows_all_filters(dtype, filt):
    rows, vocab = 6, 50_021
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(rows, vocab, 3.0, seed=11, dtype=dtype, ld=ld)
    if dtype == "f32":
        logits[:, :vocab] = np.round(logits[:, :vocab] * 4) / 4  # plenty of exact ties
    temp = workloads.uniform(rows, 0.6, 1.2, 11, 7).astype(F32)
    targets = workloads.integers(rows, 0, vocab, 11, 8).astype(np.int32)
    _run(logits, targets, temp, *filt, vocab=vocab)


def test_per_row_filter_arrays():
    rows, vocab = 12, 30_000
    logits = workloads.random_logits(rows, vocab, 2.5, seed=5)
    temp = workloads.uniform(rows, 0.5, 1.5, 5, 1).astype(F32)
    k = np.array([0, 1, 10, 29_999, 30_000, -3, 50, 0, 7, 400, 0, 2], np.int32)
    p = np.array([1.0, 0.9, 0.5, 0.99, 1.0, 0.8, 1.0, 0.3, 0.95, 0.7, 1.0, 1.0], F32)
    m = np.array([0.0, 0.0, 0.1, 0.0, 0.2, 0.0, 0.05, 0.0, 0.0, 0.01, 0.5, 0.0], F32)
    targets = workloads.integers(rows, 0, vocab, 5, 2).astype(np.int32)
    _run(logits, targets, temp, k, p, m)


@pytest.mark.parametrize("vocab", [1, 2, 7, 31, 33, 1000, 4097])
def test_small_and_odd_vocab(vocab):
    rows = 3
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(rows, vocab, 2.0, seed=vocab, dtype="bf16", ld=ld)
    targets = np.array([0, vocab - 1, vocab // 2], np.int32)
    for filt in [(0, 1.0, 0.0), (2, 0.8, 0.1), (0, 0.5, 0.0)]:
        _run(logits, targets, np.full(rows, 0.9, F32), *filt, vocab=vocab)


def test_edge_rows_nonfinite_targets_ties_singletons():
    rows, vocab = 8, 4096
    x = workloads.normal((rows, vocab), 2.0, seed=3, stream=1)
    x[0, 17] = np.nan
    x[1, 5] = np.inf
    x[2, 9] = -np.inf
    x[3, :] = 1.25                       # all equal: ties everywhere
    x[4, 100] = 40.0                     # dominant token -> singleton support
    logits = workloads.to_bf16_bits(x)
    targets = np.array([3, 3, 3, 4000, 100, -1, vocab, 12], np.int32)
    out, ref, _ = _run(logits, targets, np.ones(rows, F32), 7, 0.9, 0.0)
    st = out["status"].cpu().numpy()
    assert st[0] & vsb.ROW_NONFINITE_INPUT and st[1] & vsb.ROW_NONFINITE_INPUT
    assert st[5] & vsb.ROW_TARGET_OUT_OF_RANGE and st[6] & vsb.ROW_TARGET_OUT_OF_RANGE
    mask = unpack_mask(out["mask"], vocab)
    assert mask[3].nonzero()[0].tolist() == list(range(7))  # first k ids among equal values
    # singleton: exact zeros
    assert out["h_support"][4].item() == 0.0 and out["lp_support"][4].item() == 0.0


@pytest.mark.parametrize("filt", [(100, 1.0, 0.0), (0, 0.5, 0.0), (50, 0.9, 0.01)])
def test_crossing_below_the_key_window(filt):
    # one logit tens of binades above the rest: with a huge temperature the
    # selection crossing lies deep below the maximum's key, outside the
    # exact-key window, so the general radix descent decides
    rows, vocab = 4, 20_000
    x = workloads.normal((rows, vocab), 1.0, seed=8, stream=1)
    x[:, 3] = 3e9
    logits = workloads.to_bf16_bits(x)
    _run(logits, np.arange(rows, dtype=np.int32), np.full(rows, 1e9, F32), *filt)


@pytest.mark.parametrize("scale,shift", [(0.01, 0.0), (1.0, 2e30), (3.0, 0.004)])
def test_window_crossing_zero_and_huge_values(scale, shift):
    # tiny logits: the top-p window reaches across zero into negative keys;
    # huge logits: positive-only raw-bit binning is not used
    rows, vocab = 4, 9000
    x = workloads.normal((rows, vocab), scale, seed=17, stream=1) + np.float32(shift)
    logits = workloads.to_bf16_bits(x)
    temp = np.full(rows, 1.0 if shift < 1e3 else 2e29, F32)
    for filt in [(0, 0.5, 0.0), (0, 0.999, 0.0), (300, 1.0, 0.0), (0, 1.0, 0.3)]:
        _run(logits, np.arange(rows, dtype=np.int32), temp, *filt)


@pytest.mark.parametrize("spike", [8.0, 1000.0])
def test_row_max_after_the_first_stage(spike):
    # the exact-key window is fixed from the first streamed stage's maximum;
    # a row maximum far above it (1000) lies outside the window and the row
    # falls back to the radix descent, a near one (8) lands in the keys kept
    # above that maximum
    rows, vocab = 4, 100_000
    x = workloads.normal((rows, vocab), 1.0, seed=31, stream=1)
    x[:, 90_000] = spike
    x[1, 99_999] = spike / 2
    logits = workloads.to_bf16_bits(x)
    t = np.full(rows, 0.8 if spike < 100 else 300.0, F32)
    for filt in [(0, 0.9, 0.0), (20, 0.95, 0.0), (0, 1.0, 0.05), (0, 0.7, 0.02)]:
        _run(logits, np.array([90_000, 3, 99_999, 17], np.int32), t, *filt)
        _run_nomask(logits, np.array([90_000, 3, 99_999, 17], np.int32), t, *filt)


@pytest.mark.parametrize("filt", FILTERS)
def test_ragged_rows_all_filters_without_mask(filt):
    rows, vocab = 6, 50_021
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(rows, vocab, 3.0, seed=13, dtype="bf16", ld=ld)
    temp = workloads.uniform(rows, 0.6, 1.2, 13, 7).astype(F32)
    targets = workloads.integers(rows, 0, vocab, 13, 8).astype(np.int32)
    _run_nomask(logits, targets, temp, *filt, vocab=vocab)


def test_all_negative_rows():
    rows, vocab = 5, 30_000
    x = workloads.normal((rows, vocab), 3.0, seed=12, stream=1) - 60.0
    logits = workloads.to_bf16_bits(x)
    for filt in [(0, 0.95, 0.0), (64, 0.8, 0.0), (0, 1.0, 0.1)]:
        _run(logits, np.arange(rows, dtype=np.int32), np.full(rows, 0.9, F32), *filt)


def test_singletons_are_exact_zeros():
    rows, vocab = 16, 20_000
    logits = workloads.random_logits(rows, vocab, 3.0, seed=21)
    lf = workloads.bf16_bits_to_f32(logits)
    targets = np.argmax(lf, axis=1).astype(np.int32)  # first max id
    out, ref, _ = _run(logits, targets, np.ones(rows, F32), top_k=1)
    assert np.all(out["h_support"].cpu().numpy() == 0.0)
    assert np.all(out["lp_support"].cpu().numpy() == 0.0)
    assert np.all(out["support_size"].cpu().numpy() == 1)


def test_large_vocab():
    # well beyond a shared-memory-resident row; rows are streamed
    vocab = 1_000_003
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(2, vocab, 3.0, seed=9, ld=ld)
    _run(logits, np.array([0, vocab - 1], np.int32), np.array([0.7, 1.1], F32), 0, 0.9, 0.0,
         vocab=vocab)
    _run(logits, np.array([5, 17], np.int32), np.array([1.0, 1.0], F32), 1000, 0.99, 0.0,
         vocab=vocab)


def test_zero_rows():
    lg = torch.empty((0, 1024), dtype=torch.bfloat16, device="cuda")
    tg = torch.empty(0, dtype=torch.int32, device="cuda")
    vsb.score_fwd(lg, tg)


@pytest.mark.slow
def test_fullvocab_workload_full_size():
    w = workloads.fullvocab()
    out, ref, (nb, nd) = _run(w["logits"], w["targets"], w["temperature"], w["top_k"], w["top_p"],
                              w["min_p"])
    print(f"fullvocab: {nb} of {w['rows']} rows within 1e-6 of the top-p boundary, "
          f"{nd} of them with a support size other than the oracle's")


def test_entropy_sum_and_valid_count():
    rows, vocab = 10, 5000
    logits = workloads.random_logits(rows, vocab, 3.0, seed=2)
    lg = to_device(logits)
    tg = torch.zeros(rows, dtype=torch.int32, device="cuda")
    out = vsb.score_fwd(lg, tg, top_p=0.9, want_reduce=True)
    torch.cuda.synchronize()
    h = out["h_support"].cpu().numpy().astype(np.float64)
    assert abs(out["entropy_sum"].item() - h.sum()) <= 1e-9 * max(1.0, abs(h.sum()))
    assert out["valid_count"].item() == rows


# ---------------------------------------------------------------------------
# recorded support


def _recorded_case(rows, vocab, width, seed):
    rng = np.random.default_rng(seed)
    logits = workloads.random_logits(rows, vocab, 3.0, seed=seed)
    sup = np.full((rows, width), -1, np.int32)
    targets = rng.integers(0, vocab, rows).astype(np.int32)
    for i in range(rows):
        kind = i % 8
        w = int(rng.integers(1, width + 1))
        ids = rng.choice(vocab, size=w, replace=False).astype(np.int32)
        if kind == 0:
            ids = ids[:0]                      # empty
        elif kind == 1:
            ids = ids[:1]                      # singleton
        sup[i, : len(ids)] = ids
        if kind == 2 and len(ids) > 2:         # pads in the middle, a duplicate
            sup[i, 1] = -1
            sup[i, min(width - 1, len(ids))] = ids[0]
        if kind == 3 and len(ids) > 0:
            sup[i, 0] = vocab + 5              # bad id
        if kind in (1, 4) and len(ids) > 0:
            targets[i] = ids[-1]               # target in the support
        if kind == 5 and len(ids) > 1:
            targets[i] = ids[0]
    rng.shuffle(sup, axis=1)
    return logits, sup, targets


@pytest.mark.parametrize("want_full", [True, False])
def test_recorded_support_cases(want_full):
    rows, vocab, width = 64, 5000, 16
    logits, sup, targets = _recorded_case(rows, vocab, width, 4)
    temp = workloads.uniform(rows, 0.7, 1.3, 4, 9).astype(F32)
    out = vsb.score_fwd(to_device(logits), torch.from_numpy(targets).cuda(),
                        temperature=torch.from_numpy(temp).cuda(),
                        support_ids=torch.from_numpy(sup).cuda(), want_mask=True,
                        want_full=want_full)
    torch.cuda.synchronize()
    ref = oracle.score(logits, targets, temperature=temp.astype(np.float64), support=sup,
                       want_mask=True)
    assert np.array_equal(unpack_mask(out["mask"], vocab), ref["mask"])
    assert np.array_equal(out["valid"].cpu().numpy(), ref["valid"])
    assert np.array_equal(out["support_size"].cpu().numpy(), ref["support_size"])
    assert np.array_equal(out["status"].cpu().numpy(), map_status(ref["status"]))
    lps = out["lp_support"].cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref["lp_support"])
    assert np.array_equal(np.isfinite(lps), fin)
    assert np.abs(lps[fin] - ref["lp_support"][fin]).max() <= LP_ATOL
    hs = out["h_support"].cpu().numpy()
    from _util import assert_close_rel
    assert_close_rel(hs, ref["h_support"], 1e-4, "h_support")
    if want_full:
        assert np.abs(out["lp_full"].cpu().numpy() - ref["lp_full"]).max() <= LP_ATOL
        assert_close_rel(out["h_full"].cpu().numpy(), ref["h_full"], 1e-4, "h_full")


@pytest.mark.slow
def test_replay_workload_full_size_sampled_rows():
    w = workloads.replay()
    rows, vocab = w["rows"], w["vocab"]
    lg = to_device(w["logits"])
    out = vsb.score_fwd(lg, torch.from_numpy(w["targets"]).cuda(),
                        support_ids=torch.from_numpy(w["support"]).cuda(), want_full=False,
                        want_grad=True, want_reduce=True)
    torch.cuda.synchronize()
    widths = w["widths"]
    # every empty and singleton row, plus a seeded sample of the rest
    rng = np.random.default_rng(0)
    special = np.nonzero(widths <= 1)[0]
    others = rng.choice(np.nonzero(widths > 1)[0], size=256, replace=False)
    sel = np.sort(np.concatenate([special, others]))
    ref = oracle.score(w["logits"][sel], w["targets"][sel], support=w["support"][sel])
    lps = out["lp_support"].cpu().numpy()[sel].astype(np.float64)
    assert np.abs(lps - ref["lp_support"]).max() <= LP_ATOL
    from _util import assert_close_rel
    assert_close_rel(out["h_support"].cpu().numpy()[sel], ref["h_support"], 1e-4, "h_support")
    assert np.array_equal(out["valid"].cpu().numpy()[sel], ref["valid"])
    assert np.array_equal(out["support_size"].cpu().numpy(), np.maximum(widths, 0))
    # properties at full size: singleton rows have exact zero entropy; empty rows invalid
    hs = out["h_support"].cpu().numpy()
    assert np.all(hs[widths == 1] == 0.0)
    assert np.all(out["valid"].cpu().numpy()[widths == 0] == 0)
    assert out["valid_count"].item() == int((widths > 0).sum())


# ---------------------------------------------------------------------------
# backward


def _grads(rows):
    rng = np.random.default_rng(rows)
    return [rng.normal(size=rows).astype(F32) for _ in range(4)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("filt", [(0, 1.0, 0.0), (200, 0.9, 0.02), (0, 0.95, 0.0), (3, 1.0, 0.0)])
def test_backward_computed_support(dtype, filt):
    rows, vocab = 6, 20_011
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(rows, vocab, 2.0, seed=13, dtype=dtype, ld=ld)
    temp = workloads.uniform(rows, 0.6, 1.2, 13, 2).astype(F32)
    fw = oracle.score(logits, np.zeros(rows, np.int32), temperature=temp.astype(np.float64),
                      top_k=filt[0], top_p=float(F32(filt[1])), min_p=float(F32(filt[2])),
                      want_mask=True, vocab=vocab)
    # targets: inside the support for some rows, outside for others
    targets = np.array([np.nonzero(fw["mask"][i])[0][-1] if i % 2 == 0 else (i * 997) % vocab
                        for i in range(rows)], np.int32)
    out, ref, (nb, _) = _run(logits, targets, temp, *filt, vocab=vocab, want_grad=True)
    assert nb == 0
    g = _grads(rows)
    gt = [torch.from_numpy(x).cuda() for x in g]
    dl = vsb.score_bwd(to_device(logits), torch.from_numpy(targets).cuda(), out["ctx"], *gt,
                       temperature=torch.from_numpy(temp).cuda(), top_k=filt[0],
                       top_p=float(F32(filt[1])), min_p=float(F32(filt[2])), vocab=vocab)
    torch.cuda.synchronize()
    gref = oracle.score_grad(logits, targets, *[x.astype(np.float64) for x in g],
                             temperature=temp.astype(np.float64), top_k=filt[0],
                             top_p=float(F32(filt[1])), min_p=float(F32(filt[2])), vocab=vocab)
    compare_grad(dl.cpu().numpy()[:, :vocab], gref)


def test_backward_bf16_output_and_accumulate():
    rows, vocab = 4, 12_000
    logits = workloads.random_logits(rows, vocab, 2.0, seed=17)
    temp = np.full(rows, 0.8, F32)
    targets = np.arange(rows, dtype=np.int32)
    out, ref, _ = _run(logits, targets, temp, 0, 0.9, 0.0, want_grad=True)
    g = [torch.ones(rows, device="cuda") for _ in range(4)]
    kw = dict(temperature=torch.from_numpy(temp).cuda(), top_p=float(F32(0.9)))
    lg, tg = to_device(logits), torch.from_numpy(targets).cuda()
    d32 = vsb.score_bwd(lg, tg, out["ctx"], *g, **kw)
    d16 = vsb.score_bwd(lg, tg, out["ctx"], *g, grad_dtype=torch.bfloat16, **kw)
    base = torch.randn((rows, vocab), device="cuda", dtype=torch.float32)
    acc = base.clone()
    vsb.score_bwd(lg, tg, out["ctx"], *g, mode=vsb.VS_GRAD_ACCUMULATE, out=acc, **kw)
    torch.cuda.synchronize()
    gref = oracle.score_grad(logits, targets, *[np.ones(rows)] * 4,
                             temperature=temp.astype(np.float64), top_p=float(F32(0.9)))
    compare_grad(d32.cpu().numpy(), gref)
    # bf16 output: the fp32 result rounded to nearest even
    want16 = d32.to(torch.bfloat16)
    assert torch.equal(d16, want16)
    assert torch.allclose(acc, base + d32, rtol=0, atol=1e-6)


@pytest.mark.parametrize("mode", ["dense", "sparse"])
def test_backward_recorded_support(mode):
    rows, vocab, width = 48, 6000, 12
    logits, sup, targets = _recorded_case(rows, vocab, width, 8)
    temp = np.full(rows, 1.1, F32)
    lg, tg = to_device(logits), torch.from_numpy(targets).cuda()
    st = torch.from_numpy(sup).cuda()
    kw = dict(temperature=float(temp[0]), support_ids=st)
    out = vsb.score_fwd(lg, tg, want_grad=True, want_full=False, **kw)
    rng = np.random.default_rng(1)
    g_lps = rng.normal(size=rows).astype(F32)
    g_hs = rng.normal(size=rows).astype(F32)
    if mode == "sparse":
        empty = ((sup >= 0) & (sup < vocab)).sum(1) == 0
        g_lps[empty] = 0.0  # empty rows' lp_S gradient is dense (full vocabulary)
    gref = oracle.score_grad(logits, targets, None, g_lps.astype(np.float64), None,
                             g_hs.astype(np.float64), temperature=float(temp[0]), support=sup)
    if mode == "dense":
        dl = vsb.score_bwd(lg, tg, out["ctx"], None, torch.from_numpy(g_lps).cuda(), None,
                           torch.from_numpy(g_hs).cuda(), **kw)
        torch.cuda.synchronize()
        compare_grad(dl.cpu().numpy()[:, :vocab], gref)
    else:
        sp = vsb.score_bwd(lg, tg, out["ctx"], None, torch.from_numpy(g_lps).cuda(), None,
                           torch.from_numpy(g_hs).cuda(), mode=vsb.VS_GRAD_SPARSE, **kw)
        torch.cuda.synchronize()
        sp = sp.cpu().numpy()
        dense = np.zeros((rows, vocab))
        for i in range(rows):
            seen = set()
            for wpos in range(width):
                j = sup[i, wpos]
                if 0 <= j < vocab and j not in seen:
                    seen.add(j)
                    dense[i, j] = sp[i, wpos]
                else:
                    assert sp[i, wpos] == 0.0
        compare_grad(dense, gref)


@pytest.mark.slow
def test_replay_backward_full_size_sampled_rows():
    w = workloads.replay()
    rows, vocab = w["rows"], w["vocab"]
    lg = to_device(w["logits"])
    tg = torch.from_numpy(w["targets"]).cuda()
    st = torch.from_numpy(w["support"]).cuda()
    out = vsb.score_fwd(lg, tg, support_ids=st, want_full=False, want_grad=True)
    g_lps = torch.ones(rows, device="cuda")
    g_hs = torch.full((rows,), 0.01, device="cuda")
    dl = vsb.score_bwd(lg, tg, out["ctx"], None, g_lps, None, g_hs, support_ids=st,
                       grad_dtype=torch.float32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    widths = w["widths"]
    sel = np.sort(np.concatenate([np.nonzero(widths == 0)[0][:16], np.nonzero(widths == 1)[0][:16],
                                  rng.choice(rows, 64, replace=False)]))
    gref = oracle.score_grad(w["logits"][sel], w["targets"][sel], None, np.ones(len(sel)), None,
                             np.full(len(sel), 0.01), support=w["support"][sel])
    compare_grad(dl[torch.from_numpy(sel).cuda()].cpu().numpy()[:, :vocab], gref)


def _run_nomask(logits, targets, temperature, top_k, top_p, min_p, vocab=None):
    """GPU forward as a caller with no support mask and no saved state asks
    for it (the tie cut at the threshold is then resolved for the target
    alone), against the oracle on every row: logprobs and entropies over the
    full vocabulary and over the support; boundary rows by the prefix rule
    (the support rebuilt from the GPU's support size)."""
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    t_np = np.asarray(temperature, F32)
    k_arg = torch.from_numpy(np.asarray(top_k, np.int32)).cuda() if np.ndim(top_k) else top_k
    out = vsb.score_fwd(to_device(logits), torch.from_numpy(np.asarray(targets, np.int32)).cuda(),
                        temperature=torch.from_numpy(t_np).cuda() if t_np.ndim else float(t_np),
                        top_k=k_arg, top_p=float(F32(top_p)), min_p=float(F32(min_p)),
                        want_entropy=True, vocab=vocab)
    torch.cuda.synchronize()
    t64 = t_np.astype(np.float64)
    ref = oracle.score(logits, targets, temperature=t64 if t64.ndim else float(t64),
                       top_k=np.asarray(top_k, np.int32) if np.ndim(top_k) else top_k,
                       top_p=float(F32(top_p)), min_p=float(F32(min_p)), vocab=vocab)
    nb, nd = compare_scores(out, ref, logits, vocab, t64 if t64.ndim else np.full(rows, float(t64)),
                            np.asarray(targets, np.int32), top_k, top_p, min_p)
    sure = ~((ref["topp_margin"] < 1e-6) | (ref["minp_margin"] < 1e-6))
    return ref, sure, nb, nd


def test_target_in_threshold_tie_group_without_mask():
    """The target inside the threshold's tie group with part of the group
    kept (the lowest ids first): membership is decided by the ties before
    it, counted on either side of the target."""
    rows, vocab, G, H = 8, 40_000, 400, 50
    x = np.minimum(workloads.normal((rows, vocab), 1.0, 23, stream=1), 3.5)
    rng = np.random.default_rng(23)
    top_k = np.zeros(rows, np.int32)
    targets = np.zeros(rows, np.int32)
    for i in range(rows):
        lo = 0 if i < 4 else vocab // 2 + 1  # rows 4-7: the whole group after the middle
        ids = rng.choice(np.arange(lo, vocab), G + H, replace=False)
        grp, hi = np.sort(ids[:G]), ids[G:]
        x[i, grp] = 5.0
        x[i, hi] = 6.0
        c = G // 2 if i < 4 else G - 2
        top_k[i] = H + c
        targets[i] = [grp[c - 1], grp[c], grp[-1], grp[0], grp[c - 1], grp[c], grp[-1], hi[0]][i]
    logits = workloads.to_bf16_bits(x)
    ref, sure, _, _ = _run_nomask(logits, targets, 1.0, top_k, 1.0, 0.0)
    assert sure.all()
    kept = np.isfinite(ref["lp_support"])
    assert kept.tolist() == [True, False, False, True, True, False, False, True]


@pytest.mark.slow
def test_fullvocab_workload_full_size_without_mask():
    """The fullvocab workload (128 x 151,936 bf16, top-p 0.95) exactly as the
    benchmark calls it: no support mask, no saved state."""
    w = workloads.fullvocab()
    ref, sure, nb, nd = _run_nomask(w["logits"], w["targets"], w["temperature"], w["top_k"],
                                    w["top_p"], w["min_p"])
    print(f"fullvocab without mask: {nb} boundary rows checked by the prefix rule, "
          f"{nd} of them with a support size other than the oracle's")
