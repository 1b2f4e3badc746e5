"""GPU parity of vs_fused_lmhead_bwd (the fused head's VJP: logits recomputed
on the tensor cores, the logit gradient formed in the GEMM epilogue, then
d_hidden = dx W and d_weight = dx^T H) against the oracle's fp64 chain
(projection -> scoring -> score_grad -> the two products).

The support is the one the GPU forward chose (its top-k ids, first
support_size of them), passed to the oracle as a recorded support, so the
check is of the gradient and not of the (separately tested) support
decision.

Tolerance: the logit gradient is rounded to bf16 before the two products
(they run on bf16 tensor cores), 2^-9 relative per element at most and
about a third of that in the root mean square; the products accumulate
many such terms with independent rounding, so each output row is checked at
5e-3 relative in the 2-norm and each element within 5e-3 of its row's
largest magnitude."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import to_device

pytestmark = pytest.mark.gpu

RTOL = 5e-3


def _rows_close(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    nr = np.linalg.norm(want, axis=1)
    diff = np.linalg.norm(got - want, axis=1)
    zero = nr == 0
    assert np.all(diff[zero] == 0.0), f"{what}: rows with zero gradient are not zero"
    if (~zero).any():
        rel = diff[~zero] / nr[~zero]
        assert rel.max() <= RTOL, f"{what}: max row rel {rel.max():.3g}"
        amax = np.abs(want[~zero]).max(axis=1, keepdims=True)
        el = np.abs(got[~zero] - want[~zero]) / amax
        assert el.max() <= RTOL, f"{what}: max elementwise rel {el.max():.3g}"


def _case(rows, vocab, hidden, seed, T, k, p, mp, targets_in_support=True):
    h = workloads.to_bf16_bits(workloads.normal((rows, hidden), 1.0, seed, stream=1))
    w = workloads.to_bf16_bits(workloads.normal((vocab, hidden), 0.05, seed, stream=2))
    y = workloads.integers(rows, 0, vocab, seed, 3).astype(np.int32)
    dh, dw = to_device(h), to_device(w)
    if targets_in_support:
        # half of the rows take their top token as target (lp_S finite there)
        f0 = vsb.fused_lmhead_score(dh, dw, torch.from_numpy(y).cuda(), T, k, p, mp)
        torch.cuda.synchronize()
        top = f0["topk_ids"][:, 0].cpu().numpy()
        y[::2] = top[::2]
    ty = torch.from_numpy(y).cuda()
    fwd = vsb.fused_lmhead_score(dh, dw, ty, T, k, float(np.float32(p)), float(np.float32(mp)),
                                 want_grad=True)
    rng = np.random.default_rng(seed)
    g = [rng.normal(size=rows).astype(np.float32) for _ in range(4)]
    gt = [torch.from_numpy(x).cuda() for x in g]
    out = vsb.fused_lmhead_bwd(dh, dw, ty, k, fwd, *gt)
    torch.cuda.synchronize()
    n = fwd["support_size"].cpu().numpy()
    ids = fwd["topk_ids"].cpu().numpy()
    sup = np.full((rows, k), -1, np.int32)
    for i in range(rows):
        sup[i, :n[i]] = ids[i, :n[i]]
    rH, rW = oracle.lmhead_grad(h, w, y, float(np.float32(T)), *[x.astype(np.float64) for x in g],
                                support=sup)
    return out, rH, rW, n


@pytest.mark.parametrize("rows,vocab,hidden,k,p,mp", [
    (300, 3001, 256, 20, 0.9, 0.02),   # ragged rows and vocabulary, all three filters
    (77, 1000, 128, 1, 1.0, 0.0),      # singleton supports: no support-entropy gradient
    (130, 2048, 192, 64, 1.0, 0.0),    # top-k only, the largest k
])
def test_fused_head_backward_matches_oracle(rows, vocab, hidden, k, p, mp):
    out, rH, rW, n = _case(rows, vocab, hidden, 7 + rows, 0.8, k, p, mp)
    _rows_close(out["d_hidden"].cpu().numpy(), rH, "d_hidden")
    _rows_close(out["d_weight"].cpu().numpy(), rW, "d_weight")
    if k == 1:
        assert np.all(n == 1)


def test_fused_head_backward_several_vocabulary_chunks():
    # more columns than one backward chunk (32,768): the gradient is formed
    # and consumed chunk by chunk, d_hidden accumulating over the chunks
    out, rH, rW, _ = _case(64, 70_001, 128, 11, 1.1, 16, 0.95, 0.0)
    _rows_close(out["d_hidden"].cpu().numpy(), rH, "d_hidden")
    _rows_close(out["d_weight"].cpu().numpy(), rW, "d_weight")


def test_fused_head_backward_zero_upstream_and_one_output():
    rows, vocab, hidden, k = 40, 900, 64, 8
    h = workloads.to_bf16_bits(workloads.normal((rows, hidden), 1.0, 3, stream=1))
    w = workloads.to_bf16_bits(workloads.normal((vocab, hidden), 0.05, 3, stream=2))
    ty = torch.from_numpy(workloads.integers(rows, 0, vocab, 3, 3).astype(np.int32)).cuda()
    dh, dw = to_device(h), to_device(w)
    fwd = vsb.fused_lmhead_score(dh, dw, ty, 1.0, k, 0.9, 0.0, want_grad=True)
    z = vsb.fused_lmhead_bwd(dh, dw, ty, k, fwd)  # every upstream gradient NULL
    only_h = vsb.fused_lmhead_bwd(dh, dw, ty, k, fwd, g_h_full=torch.ones(rows, device="cuda"),
                                  want_weight=False)
    torch.cuda.synchronize()
    assert torch.all(z["d_hidden"] == 0) and torch.all(z["d_weight"] == 0)
    assert "d_weight" not in only_h and torch.isfinite(only_h["d_hidden"]).all()
    rH, _ = oracle.lmhead_grad(h, w, ty.cpu().numpy(), 1.0, None, None, np.ones(rows), None,
                               top_k=k, top_p=float(np.float32(0.9)))
    _rows_close(only_h["d_hidden"].cpu().numpy(), rH, "d_hidden (entropy only)")
