"""Seeded synthetic inputs for the scoring path.

This module only draws inputs.  It holds none of the scoring arithmetic
(no log-sum-exp, softmax normalisation, entropy, support selection or
distance): both the CUDA path and the oracle consume the arrays it returns,
and the same bit patterns reach both (bf16 values are produced here, on the
host, and copied to the device unchanged).

Random numbers come from numpy's Philox (4x64, 10 rounds) counter-based generator
(Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
one stream per (seed, block) via SeedSequence, so results do not depend on
the number of worker threads.

Distribution notation: N(0, s) means mean 0 and standard deviation s.

The five named workloads follow the problem statement of the scoring path:

* ``tiny``      8 x 1,024 fp32 logits ~ N(0,2), T = 1, targets uniform,
                top_k 50, top_p 0.9, min_p 0.05.
* ``fullvocab`` 128 x 151,936 bf16 logits ~ N(0,3) plus 8 distinct uniformly
                drawn ids per row raised by +8; per-row T ~ U[0.6,1.2];
                top_p 0.95; targets sampled from the tempered distribution
                with the Gumbel-max trick.
* ``distance``  512 x 151,936 bf16 draft ~ N(0,3); target = bf16(draft +
                N(0,0.5)); row weights ~ U[0,1].
* ``replay``    8,192 x 151,936 bf16 logits ~ N(0,3) with 64 distinct
                Zipf(1.1)-ranked ids per row raised by +6 (id = rank - 1);
                recorded support = the first w of them, w = 0 with prob.
                0.02, 1 with prob. 0.10, else U{1..64}; padded with -1 to
                width 64; targets Gumbel-max over the support (uniform when
                it is empty).
* ``lmhead``    hidden [8192, 4096] bf16 ~ N(0,1), weight [151,936, 4096]
                bf16 ~ N(0,0.02), T = 0.8, top_k 20, top_p 0.95,
                min_p 0.02, targets uniform.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

VOCAB = 151_936

_BLOCK = 1 << 22  # elements per independently seeded block


def _gen(seed_seq: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(seed_seq))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(
        np.uint16
    )
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(shape, sigma: float, seed: int, stream: int = 0, dtype=np.float32) -> np.ndarray:
    """N(0, sigma) samples (float32), generated in parallel blocks."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    nblk = (n + _BLOCK - 1) // _BLOCK
    seqs = np.random.SeedSequence([seed, stream, 0x5EED]).spawn(max(nblk, 1))

    def fill(b):
        lo, hi = b * _BLOCK, min(n, (b + 1) * _BLOCK)
        g = _gen(seqs[b])
        g.standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])
        if sigma != 1.0:
            out[lo:hi] *= np.float32(sigma)

    if nblk <= 1:
        if n:
            fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return out.reshape(shape).astype(dtype, copy=False)


def uniform(shape, lo: float, hi: float, seed: int, stream: int) -> np.ndarray:
    g = _gen(np.random.SeedSequence([seed, stream, 0x0F]))
    return g.uniform(lo, hi, size=shape)


def integers(shape, lo: int, hi: int, seed: int, stream: int) -> np.ndarray:
    g = _gen(np.random.SeedSequence([seed, stream, 0x1D]))
    return g.integers(lo, hi, size=shape, dtype=np.int64)


def gumbel_max_targets(logits_f32: np.ndarray, temperature: np.ndarray, seed: int,
                       stream: int) -> np.ndarray:
    """One draw per row from the categorical distribution with weights
    exp(l / T), by the Gumbel-max trick: argmax_j (l_j / T + G_j),
    G_j ~ Gumbel(0, 1).  This is how a sampler draws a target token."""
    rows, vocab = logits_f32.shape
    out = np.empty(rows, dtype=np.int32)
    seqs = np.random.SeedSequence([seed, stream, 0x6B]).spawn(max(rows, 1))

    def draw(i):
        g = _gen(seqs[i])
        gum = g.gumbel(size=vocab)
        out[i] = int(np.argmax(logits_f32[i].astype(np.float64) / float(temperature[i]) + gum))

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(draw, range(rows)))
    return out


def random_logits(rows: int, vocab: int, sigma: float, seed: int, dtype: str = "bf16",
                  ld: int | None = None) -> np.ndarray:
    """[rows, ld] logits ~ N(0, sigma); bf16 as uint16 bits, else float32.
    Columns beyond `vocab` (padding when ld > vocab) are filled with NaN so a
    kernel that reads them is caught."""
    ld = vocab if ld is None else ld
    x = normal((rows, vocab), sigma, seed, stream=1)
    if ld != vocab:
        full = np.full((rows, ld), np.nan, dtype=np.float32)
        full[:, :vocab] = x
        x = full
    return to_bf16_bits(x) if dtype == "bf16" else x


# ----------------------------------------------------------------------------
# the five named workloads


def tiny(seed: int = 0) -> dict:
    rows, vocab = 8, 1024
    logits = normal((rows, vocab), 2.0, seed, stream=1)
    return dict(name="tiny", rows=rows, vocab=vocab, dtype="f32", logits=logits,
                temperature=np.ones(rows, dtype=np.float32),
                targets=integers(rows, 0, vocab, seed, 2).astype(np.int32),
                top_k=50, top_p=0.9, min_p=0.05)


def fullvocab(rows: int = 128, vocab: int = VOCAB, seed: int = 1, spikes: int = 8,
              spike: float = 8.0, with_targets: bool = True) -> dict:
    x = normal((rows, vocab), 3.0, seed, stream=1)
    g = _gen(np.random.SeedSequence([seed, 3, 0x5B]))
    for i in range(rows):
        ids = g.choice(vocab, size=min(spikes, vocab), replace=False)
        x[i, ids] += np.float32(spike)
    logits = to_bf16_bits(x)
    temperature = uniform(rows, 0.6, 1.2, seed, 4).astype(np.float32)
    targets = (gumbel_max_targets(bf16_bits_to_f32(logits), temperature, seed, 5)
               if with_targets else integers(rows, 0, vocab, seed, 5).astype(np.int32))
    return dict(name="fullvocab", rows=rows, vocab=vocab, dtype="bf16", logits=logits,
                temperature=temperature, targets=targets, top_k=0, top_p=0.95, min_p=0.0)


def distance(rows: int = 512, vocab: int = VOCAB, seed: int = 2) -> dict:
    d = normal((rows, vocab), 3.0, seed, stream=1)
    draft = to_bf16_bits(d)
    noise = normal((rows, vocab), 0.5, seed, stream=2)
    target = to_bf16_bits(bf16_bits_to_f32(draft) + noise)
    w = uniform(rows, 0.0, 1.0, seed, 3).astype(np.float32)
    return dict(name="distance", rows=rows, vocab=vocab, dtype="bf16", draft=draft,
                target=target, weight=w)


def _zipf_cdf(vocab: int, s: float) -> np.ndarray:
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    w = ranks ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def _zipf_support_lists(rows: int, vocab: int, seed: int, width: int, zipf_s: float):
    """Per row `width` distinct ids drawn from Zipf(zipf_s) over ranks 1..V
    (id = rank - 1), and a recorded width per row: 0 with probability 0.02, 1
    with 0.10, else U{1..width}; returns (ids [rows, width], widths,
    support [rows, width] -1 padded)."""
    cdf = _zipf_cdf(vocab, zipf_s)
    g = _gen(np.random.SeedSequence([seed, 2, 0x21]))
    boosted = np.empty((rows, width), dtype=np.int32)
    for i in range(rows):
        chosen: list[int] = []
        seen = set()
        while len(chosen) < width:
            draws = np.searchsorted(cdf, g.random(4 * width), side="right")
            for r in draws:
                r = int(min(r, vocab - 1))
                if r not in seen:
                    seen.add(r)
                    chosen.append(r)
                    if len(chosen) == width:
                        break
        boosted[i] = chosen
    u = uniform(rows, 0.0, 1.0, seed, 3)
    widths = integers(rows, 1, width + 1, seed, 4)
    widths = np.where(u < 0.02, 0, np.where(u < 0.12, 1, widths)).astype(np.int32)
    support = np.full((rows, width), -1, dtype=np.int32)
    for i in range(rows):
        support[i, : widths[i]] = boosted[i, : widths[i]]
    return boosted, widths, support


def replay(rows: int = 8192, vocab: int = VOCAB, seed: int = 3, width: int = 64,
           boost: float = 6.0, zipf_s: float = 1.1) -> dict:
    x = normal((rows, vocab), 3.0, seed, stream=1)
    boosted, widths, support = _zipf_support_lists(rows, vocab, seed, width, zipf_s)
    rows_idx = np.repeat(np.arange(rows), width)
    x[rows_idx, boosted.reshape(-1)] += np.float32(boost)
    logits = to_bf16_bits(x)
    # targets: Gumbel-max over the recorded support at T = 1; uniform when empty
    gt = _gen(np.random.SeedSequence([seed, 5, 0x6B]))
    lf = bf16_bits_to_f32(logits)
    targets = np.empty(rows, dtype=np.int32)
    uni = integers(rows, 0, vocab, seed, 6)
    for i in range(rows):
        w = widths[i]
        if w == 0:
            targets[i] = uni[i]
            continue
        ids = support[i, :w]
        targets[i] = ids[int(np.argmax(lf[i, ids].astype(np.float64) + gt.gumbel(size=w)))]
    return dict(name="replay", rows=rows, vocab=vocab, dtype="bf16", logits=logits,
                support=support, widths=widths, targets=targets,
                temperature=np.ones(rows, dtype=np.float32))


def support_lists(rows: int = 8192, vocab: int = VOCAB, seed: int = 3, width: int = 64,
                  zipf_s: float = 1.1) -> dict:
    """Recorded supports of the replay recipe (Zipf ids, width mix) for the
    support-only projection, with targets drawn uniformly from each row's
    support (uniform over the vocabulary for an empty support)."""
    _, widths, support = _zipf_support_lists(rows, vocab, seed, width, zipf_s)
    pick = uniform(rows, 0.0, 1.0, seed, 7)
    uni = integers(rows, 0, vocab, seed, 6)
    targets = np.empty(rows, dtype=np.int32)
    for i in range(rows):
        w = int(widths[i])
        targets[i] = uni[i] if w == 0 else support[i, min(w - 1, int(pick[i] * w))]
    return dict(name="support_lists", rows=rows, vocab=vocab, support=support, widths=widths,
                targets=targets)


def lmhead(rows: int = 8192, vocab: int = VOCAB, hidden: int = 4096, seed: int = 4) -> dict:
    h = to_bf16_bits(normal((rows, hidden), 1.0, seed, stream=1))
    w = to_bf16_bits(normal((vocab, hidden), 0.02, seed, stream=2))
    return dict(name="lmhead", rows=rows, vocab=vocab, hidden=hidden, hidden_states=h,
                weight=w, temperature=0.8, top_k=20, top_p=0.95, min_p=0.02,
                targets=integers(rows, 0, vocab, seed, 3).astype(np.int32))
