"""GPU parity of vs_l1_distance against the fp64 oracle (DSpark distance,
accept rate, weighted loss and draft gradient), through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import assert_close_rel, compare_grad, to_device

pytestmark = pytest.mark.gpu


def _pad(a, ld):
    """Rows padded to a 16-byte stride with NaN (never read by the kernels)."""
    vocab = a.shape[1]
    if ld == vocab:
        return a
    fill = 0x7FC0 if a.dtype == np.uint16 else np.nan
    return np.pad(a, ((0, 0), (0, ld - vocab)), constant_values=fill)


def _check(draft, target, weight, grad_dtype=torch.float32, sample=None):
    rows, vocab = draft.shape
    ld = (vocab + 7) // 8 * 8
    d, t = to_device(_pad(draft, ld)), to_device(_pad(target, ld))
    w = None if weight is None else torch.from_numpy(weight).cuda()
    out = vsb.l1_distance(d, t, w, want_loss=True, want_grad=True, grad_dtype=grad_dtype,
                          vocab=vocab)
    torch.cuda.synchronize()
    w64 = None if weight is None else weight.astype(np.float64)
    ref = oracle.l1(draft, target, weight=w64)
    assert_close_rel(out["l1"].cpu().numpy(), ref["l1"], 1e-4, "l1")
    acc = out["accept"].cpu().numpy().astype(np.float64)
    assert np.abs(acc - ref["accept"]).max() <= 1e-4
    loss = out["loss"].cpu().numpy().astype(np.float64)
    assert_close_rel(loss[:1], [ref["loss_num"]], 1e-4, "loss numerator")
    assert_close_rel(loss[1:2], [ref["loss_den"]], 1e-6, "loss denominator")
    assert_close_rel(loss[2:], [ref["loss"]], 1e-4, "loss")
    sel = np.arange(rows) if sample is None else sample
    # gradient rows: oracle on the selected rows, normalised by the full weight sum
    ws = np.ones(rows) if weight is None else weight.astype(np.float64)
    gref = oracle.l1(draft[sel], target[sel], weight=ws[sel], want_grad=True,
                     global_wsum=float(ws.sum()))
    gref_g = gref["grad"]
    near = np.abs(_probs(draft[sel]) - _probs(target[sel])) < 1e-6
    g = out["grad"][torch.from_numpy(sel).cuda()].float().cpu().numpy()[:, :vocab]
    compare_grad(g, gref_g, exclude=near,
                 rtol=2e-3 if grad_dtype == torch.float32 else 6e-3)
    return out


def _probs(bits):
    x = bits.astype(np.float64) if bits.dtype != np.uint16 else workloads.bf16_bits_to_f32(bits).astype(np.float64)
    x = np.exp(x - x.max(1, keepdims=True))
    return x / x.sum(1, keepdims=True)


@pytest.mark.parametrize("vocab", [20_011, 1000, 33, 1])
def test_l1_ragged_bf16(vocab):
    w = workloads.distance(rows=16, vocab=vocab, seed=5)
    _check(w["draft"], w["target"], w["weight"])


def test_l1_row_stride_beyond_vocab():
    vocab, ld = 10_001, 10_008
    w = workloads.distance(rows=4, vocab=vocab, seed=6)
    pad = lambda a: np.pad(a, ((0, 0), (0, ld - vocab)), constant_values=0x7FC0)  # NaN pads
    d, t = to_device(pad(w["draft"])), to_device(pad(w["target"]))
    out = vsb.l1_distance(d, t, torch.from_numpy(w["weight"]).cuda(), want_grad=True, vocab=vocab)
    torch.cuda.synchronize()
    ref = oracle.l1(w["draft"], w["target"], weight=w["weight"].astype(np.float64), want_grad=True)
    assert_close_rel(out["l1"].cpu().numpy(), ref["l1"], 1e-4, "l1")
    compare_grad(out["grad"].cpu().numpy()[:, :vocab], ref["grad"])


def test_l1_f32_and_bf16_grad():
    rng = np.random.default_rng(3)
    d = (rng.normal(size=(8, 4096)) * 2).astype(np.float32)
    t = (d + rng.normal(size=d.shape) * 0.7).astype(np.float32)
    wt = rng.uniform(size=8).astype(np.float32)
    _check(d, t, wt)
    _check(workloads.to_bf16_bits(d), workloads.to_bf16_bits(t), wt, grad_dtype=torch.bfloat16)


def test_l1_identical_rows_exact():
    w = workloads.distance(rows=6, vocab=30_000, seed=9)
    d = to_device(w["draft"])
    out = vsb.l1_distance(d, d.clone(), torch.from_numpy(w["weight"]).cuda(), want_grad=True)
    torch.cuda.synchronize()
    assert torch.all(out["l1"] == 0) and torch.all(out["accept"] == 1)
    assert torch.all(out["grad"] == 0)
    assert out["loss"][0].item() == 0.0 and out["loss"][2].item() == 0.0


def test_l1_unweighted_and_zero_weights():
    w = workloads.distance(rows=5, vocab=8000, seed=1)
    _check(w["draft"], w["target"], None)
    d, t = to_device(w["draft"]), to_device(w["target"])
    out = vsb.l1_distance(d, t, torch.zeros(5, device="cuda"), want_grad=True)
    torch.cuda.synchronize()
    assert out["loss"][2].item() == 0.0 and torch.all(out["grad"] == 0)


@pytest.mark.slow
def test_distance_workload_full_size():
    w = workloads.distance()
    rng = np.random.default_rng(0)
    sel = np.sort(rng.choice(w["rows"], 160, replace=False))
    out = _check(w["draft"], w["target"], w["weight"], grad_dtype=torch.bfloat16, sample=sel)
    assert out["grad"].dtype == torch.bfloat16


def test_l1_sharded_rows_take_the_global_denominator():
    """A batch split into three uneven row shards, each scored by
    vs_l1_distance_sharded with the weight sum over all shards (each shard's
    vs_l1_weight_sum, added on the device as an all-reduce would): the
    concatenated gradients equal the oracle's on the whole batch, the loss
    contributions add up to its loss, and the numerators and denominators
    to its numerator and denominator."""
    w = workloads.distance(rows=24, vocab=20_011, seed=12)
    rows, vocab = 24, 20_011
    ld = (vocab + 7) // 8 * 8
    d, t = to_device(_pad(w["draft"], ld)), to_device(_pad(w["target"], ld))
    wt = torch.from_numpy(w["weight"]).cuda()
    cuts = [0, 5, 17, 24]
    parts = [vsb.l1_weight_sum(cuts[i + 1] - cuts[i], wt[cuts[i]:cuts[i + 1]]) for i in range(3)]
    wsum = parts[0] + parts[1] + parts[2]
    outs = [vsb.l1_distance(d[cuts[i]:cuts[i + 1]], t[cuts[i]:cuts[i + 1]], wt[cuts[i]:cuts[i + 1]],
                            want_loss=True, want_grad=True, vocab=vocab, global_weight_sum=wsum)
            for i in range(3)]
    torch.cuda.synchronize()
    ref = oracle.l1(w["draft"], w["target"], weight=w["weight"].astype(np.float64), want_grad=True)
    assert abs(wsum.item() - w["weight"].astype(np.float64).sum()) <= 1e-12 * wsum.item()
    g = np.concatenate([o["grad"].cpu().numpy()[:, :vocab] for o in outs])
    near = np.abs(_probs(w["draft"]) - _probs(w["target"])) < 1e-6
    compare_grad(g, ref["grad"], exclude=near)
    loss = np.stack([o["loss"].cpu().numpy().astype(np.float64) for o in outs])
    assert_close_rel([loss[:, 2].sum()], [ref["loss"]], 1e-4, "loss (sum of contributions)")
    assert_close_rel([loss[:, 0].sum()], [ref["loss_num"]], 1e-4, "numerator")
    assert_close_rel([loss[:, 1].sum()], [ref["loss_den"]], 1e-6, "denominator")
    # the unsharded call on the whole batch agrees element by element
    full = vsb.l1_distance(d, t, wt, want_loss=True, want_grad=True, vocab=vocab)
    torch.cuda.synchronize()
    gf = full["grad"].cpu().numpy()[:, :vocab]
    assert np.abs(g - gf).max() <= 1e-6 * np.abs(gf).max()
