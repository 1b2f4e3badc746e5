"""GPU parity of the seeded Gumbel-max sample (vs_score_fwd with
VS_WANT_SAMPLE) against the oracle's sampler: the same generator, the same
fp32 operation sequence, so the sampled token must match exactly.

With the support mask requested, the oracle samples over the support the GPU
returned (a valid support even on rows at the top-p / min-p boundary, where
several supports are correct), so every row is compared.  Without the mask,
the oracle samples over its own support and rows off the boundary band are
compared."""

import numpy as np
import pytest
import torch

import oracle
import sampling_support_b200 as vsb
import workloads
from _util import to_device, unpack_mask

pytestmark = pytest.mark.gpu

F32 = np.float32
FILTERS = [(0, 1.0, 0.0), (0, 0.95, 0.0), (100, 1.0, 0.0), (0, 1.0, 0.05), (200, 0.9, 0.02),
           (1, 1.0, 0.0), (37, 0.5, 0.3)]


def _sample(logits, targets, T, k, p, mp, seed, vocab=None, want_mask=True, support=None):
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    t_arg = torch.from_numpy(np.asarray(T, F32)).cuda() if np.ndim(T) else float(T)
    out = vsb.score_fwd(to_device(logits), torch.from_numpy(np.asarray(targets, np.int32)).cuda(),
                        temperature=t_arg, top_k=k, top_p=float(F32(p)), min_p=float(F32(mp)),
                        want_mask=want_mask, vocab=vocab, sample_seed=seed,
                        support_ids=None if support is None else torch.from_numpy(support).cuda())
    torch.cuda.synchronize()
    return out


def _oracle_mask(logits, targets, T, k, p, mp, vocab=None, support=None):
    t64 = np.asarray(T, F32).astype(np.float64)
    ref = oracle.score(logits, targets, temperature=t64 if t64.ndim else float(t64), top_k=k,
                       top_p=float(F32(p)), min_p=float(F32(mp)), want_mask=True, vocab=vocab,
                       support=support)
    return ref


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("filt", FILTERS)
def test_sample_matches_oracle_over_the_returned_support(dtype, filt):
    rows, vocab = 6, 50_021
    ld = (vocab + 7) // 8 * 8
    logits = workloads.random_logits(rows, vocab, 3.0, seed=21, dtype=dtype, ld=ld)
    if dtype == "f32":
        logits[:, :vocab] = np.round(logits[:, :vocab] * 4) / 4  # exact ties
    T = workloads.uniform(rows, 0.6, 1.2, 21, 7).astype(F32)
    y = workloads.integers(rows, 0, vocab, 21, 8).astype(np.int32)
    for seed in (0, 12345, 2**63 + 7):
        out = _sample(logits, y, T, *filt, seed, vocab=vocab)
        mask = unpack_mask(out["mask"], vocab)
        want = oracle.gumbel_sample(logits, T, mask, seed, vocab=vocab)
        got = out["sampled"].cpu().numpy()
        assert np.array_equal(got, want), (seed, got, want)
        assert np.all(mask[np.arange(rows), got] == 1)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sample_without_mask_matches_oracle(dtype):
    rows, vocab = 6, 30_000
    logits = workloads.random_logits(rows, vocab, 3.0, seed=4, dtype=dtype)
    T = workloads.uniform(rows, 0.6, 1.2, 4, 7).astype(F32)
    y = workloads.integers(rows, 0, vocab, 4, 8).astype(np.int32)
    for k, p, mp in [(0, 0.9, 0.0), (50, 1.0, 0.0), (0, 1.0, 0.0)]:
        out = _sample(logits, y, T, k, p, mp, 99, want_mask=False)
        ref = _oracle_mask(logits, y, T, k, p, mp)
        sure = ~((ref["topp_margin"] < 1e-6) | (ref["minp_margin"] < 1e-6))
        want = oracle.gumbel_sample(logits, T, ref["mask"], 99)
        got = out["sampled"].cpu().numpy()
        assert np.array_equal(got[sure], want[sure])


def test_sample_recorded_support():
    rows, vocab, width = 10, 5000, 12
    logits = workloads.random_logits(rows, vocab, 2.0, seed=8)
    rng = np.random.default_rng(8)
    sup = rng.integers(0, vocab, (rows, width)).astype(np.int32)
    sup[0, :] = -1                     # empty: no sample
    sup[1, 1:] = -1                    # singleton
    sup[2, :4] = [5, 5, 7, 5]          # repeats
    sup[3, :3] = [-4, vocab, 9]        # bad ids
    y = sup[:, -1].copy()
    out = _sample(logits, y, 0.9, 0, 1.0, 0.0, 7, want_mask=True, support=sup)
    ref = _oracle_mask(logits, y, 0.9, 0, 1.0, 0.0, support=sup)
    want = oracle.gumbel_sample(logits, 0.9, ref["mask"], 7)
    got = out["sampled"].cpu().numpy()
    assert np.array_equal(got, want)
    assert got[0] == -1 and got[1] == sup[1, 0]


def test_sample_nonfinite_row_and_row_independence():
    rows, vocab = 4, 4096
    logits = workloads.random_logits(rows, vocab, 1.0, seed=3)
    logits[1] = logits[0]
    logits[2, 17] = 0x7FC0  # NaN (bf16)
    y = np.zeros(rows, np.int32)
    out = _sample(logits, y, 1.0, 0, 1.0, 0.0, 5, want_mask=False)
    got = out["sampled"].cpu().numpy()
    assert got[2] == -1
    ref = _oracle_mask(logits, y, 1.0, 0, 1.0, 0.0)
    want = oracle.gumbel_sample(logits, 1.0, ref["mask"], 5)
    ok = np.array([0, 1, 3])
    assert np.array_equal(got[ok], want[ok])


def test_sample_rows_over_several_launches():
    """More rows than one launch keeps in L2 (the row index keys the noise
    across launches)."""
    rows, vocab = 200, 151_936
    logits = workloads.random_logits(rows, vocab, 3.0, seed=17)
    T = workloads.uniform(rows, 0.6, 1.2, 17, 7).astype(F32)
    y = workloads.integers(rows, 0, vocab, 17, 8).astype(np.int32)
    out = _sample(logits, y, T, 0, 0.95, 0.0, 2024, want_mask=True)
    mask = unpack_mask(out["mask"], vocab)
    want = oracle.gumbel_sample(logits, T, mask, 2024)
    assert np.array_equal(out["sampled"].cpu().numpy(), want)


@pytest.mark.slow
def test_sample_fullvocab_workload():
    w = workloads.fullvocab()
    out = _sample(w["logits"], w["targets"], w["temperature"], w["top_k"], w["top_p"], w["min_p"],
                  31337, want_mask=False)
    ref = _oracle_mask(w["logits"], w["targets"], w["temperature"], w["top_k"], w["top_p"],
                       w["min_p"])
    sure = ~((ref["topp_margin"] < 1e-6) | (ref["minp_margin"] < 1e-6))
    want = oracle.gumbel_sample(w["logits"], w["temperature"], ref["mask"], 31337)
    got = out["sampled"].cpu().numpy()
    assert np.array_equal(got[sure], want[sure])
    print(f"fullvocab sampling: {int(sure.sum())} of {w['rows']} rows compared")
