"""GPU parity of the vocabulary-parallel fused head: the weight split into
uneven vocabulary shards, each shard's partial record block computed by
vs_fused_lmhead_partial (here all on one device, one block after another,
exactly what an all-gather over the shards' ranks assembles), then
vs_fused_lmhead_merge.  The merged outputs are compared with the
single-shard vs_fused_lmhead_score and with the fp64 oracle on the
materialised logits."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import LP_ATOL, assert_close_rel, to_device

pytestmark = pytest.mark.gpu


def _shards(vocab, cuts):
    edges = [0] + list(cuts) + [vocab]
    return [(edges[i], edges[i + 1] - edges[i]) for i in range(len(edges) - 1)]


@pytest.mark.parametrize("rows,vocab,hidden,k,p,mp,cuts", [
    (200, 5003, 128, 20, 0.9, 0.02, [1700, 3333]),
    (64, 2000, 64, 8, 1.0, 0.0, [1000]),
    (33, 4096, 192, 64, 0.95, 0.0, [256, 512, 3000]),
])
def test_tp_merge_matches_single_shard_and_oracle(rows, vocab, hidden, k, p, mp, cuts):
    h = workloads.to_bf16_bits(workloads.normal((rows, hidden), 1.0, rows, stream=1))
    w = workloads.to_bf16_bits(workloads.normal((vocab, hidden), 0.05, rows, stream=2))
    y = workloads.integers(rows, 0, vocab, rows, 3).astype(np.int32)
    y[-1] = vocab  # out of range: flagged, NaN logprobs
    dh, dw = to_device(h), to_device(w)
    ty = torch.from_numpy(y).cuda()
    T = 0.9
    pf, mf = float(np.float32(p)), float(np.float32(mp))
    blocks = [vsb.fused_lmhead_partial(dh, dw[b:b + n], b, vocab, ty, T, k)
              for b, n in _shards(vocab, cuts)]
    merged = vsb.fused_lmhead_merge(torch.stack(blocks), rows, vocab, ty, T, k, pf, mf)
    full = vsb.fused_lmhead_score(dh, dw, ty, T, k, pf, mf)
    torch.cuda.synchronize()
    m = {kk: v.cpu().numpy() for kk, v in merged.items()}
    f = {kk: v.cpu().numpy() for kk, v in full.items()}
    # the same candidates in the same order; statistics merged in another
    # order, so values agree to rounding
    assert np.array_equal(m["topk_ids"], f["topk_ids"])
    assert np.array_equal(m["status"], f["status"]) and np.array_equal(m["valid"], f["valid"])
    ok = np.isfinite(f["lp_full"])
    assert np.array_equal(np.isfinite(m["lp_full"]), ok)
    assert np.abs(m["lp_full"][ok] - f["lp_full"][ok]).max() <= 1e-5
    assert_close_rel(m["h_full"], f["h_full"], 1e-5, "h_full (merged vs single)")
    # against the oracle on the fp64 logits of the rows
    z = oracle.lmhead_logits(h, w, np.arange(rows, dtype=np.int32), float(np.float32(T)))
    ref = oracle.score(z, y, top_k=k, top_p=pf, min_p=mf)
    assert np.abs(m["lp_full"][ok] - ref["lp_full"][ok]).max() <= LP_ATOL
    assert_close_rel(m["h_full"], ref["h_full"], 1e-4, "h_full")
    sure = (ref["topk_gap"] >= 1e-4) & (ref["topp_margin"] >= 1e-5) & (ref["minp_margin"] >= 1e-5)
    assert np.array_equal(m["support_size"][sure], ref["support_size"][sure])
    fin = np.isfinite(ref["lp_support"]) & sure
    assert np.abs(m["lp_support"][fin] - ref["lp_support"][fin]).max(initial=0) <= LP_ATOL
    assert (m["status"][-1] & vsb.ROW_TARGET_OUT_OF_RANGE) and np.isnan(m["lp_full"][-1])
