"""Pins for the fp64 oracle against what the pages and mathematics fix.

Nothing here compares the oracle with itself: every expected value comes from
a closed form, a hand-derived case (tests/golden), a brute-force enumeration
written independently of the oracle's sort-and-prefix code, a numpy library
routine, an invariance of the definitions, or central finite differences.
"""

import itertools
import json
import math
from pathlib import Path

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = Path(__file__).parent / "golden" / "support_cases.json"


def _eval(expr):
    if expr == "-inf":
        return -math.inf
    return eval(expr, {"log": math.log, "exp": math.exp, "e": math.e, "__builtins__": {}})


def _logits(vals):
    out = []
    for v in vals:
        if isinstance(v, str) and v.startswith("log:"):
            out.append(math.log(float(v[4:])))
        elif isinstance(v, str) and v.startswith("expr:"):
            out.append(_eval(v[5:]))
        else:
            out.append(float(v))
    return np.array(out, dtype=np.float64)


# ---------------------------------------------------------------------------
# hand-derived golden cases


def test_golden_computed_support_cases():
    cases = json.loads(GOLDEN.read_text())["cases"]
    for c in cases:
        l = _logits(c["logits"])
        n = len(l)
        for t_i, y in enumerate(c["targets"]):
            r = oracle.score(l[None, :], [y], temperature=c["temperature"], top_k=c["top_k"],
                             top_p=c["top_p"], min_p=c["min_p"], want_mask=True)
            got = sorted(np.nonzero(r["mask"][0])[0].tolist())
            assert got == c["support"], c["name"]
            assert r["support_size"][0] == len(c["support"])
            exp_lp = _eval(c["lp_support"][t_i])
            if exp_lp == -math.inf:
                assert r["lp_support"][0] == -math.inf, c["name"]
                assert r["status"][0] & oracle.TARGET_NOT_IN_SUPPORT
            else:
                assert abs(r["lp_support"][0] - exp_lp) < 1e-12, c["name"]
            if c["h_support"] is None:
                assert abs(r["h_support"][0] - r["h_full"][0]) < 1e-12
            else:
                assert abs(r["h_support"][0] - _eval(c["h_support"])) < 1e-12, c["name"]
            if c.get("exact_zero"):
                assert r["h_support"][0] == 0.0
                if exp_lp == 0:
                    assert r["lp_support"][0] == 0.0
            assert r["valid"][0] == 1


def test_golden_recorded_support_cases():
    names = {"DUP_SUPPORT_ID": oracle.DUP_SUPPORT_ID,
             "TARGET_NOT_IN_SUPPORT": oracle.TARGET_NOT_IN_SUPPORT}
    for c in json.loads(GOLDEN.read_text())["recorded"]:
        l = _logits(c["logits"])
        sup = np.array([c["support_ids"]], dtype=np.int32)
        for t_i, y in enumerate(c["targets"]):
            r = oracle.score(l[None, :], [y], support=sup, want_mask=True)
            assert sorted(np.nonzero(r["mask"][0])[0].tolist()) == c["support"]
            exp_lp = _eval(c["lp_support"][t_i])
            if exp_lp == -math.inf:
                assert r["lp_support"][0] == -math.inf
            else:
                assert abs(r["lp_support"][0] - exp_lp) < 1e-12
            if "status" in c:
                want = 0
                for part in c["status"][t_i].split("|"):
                    want |= names[part]
                assert r["status"][0] == want
            if "valid" in c:
                assert r["valid"][0] == c["valid"]
                assert r["h_support"][0] == 0.0


# ---------------------------------------------------------------------------
# closed forms


@pytest.mark.parametrize("vocab", [1024, workloads.VOCAB])
def test_uniform_logits_closed_form(vocab):
    l = np.full((2, vocab), 0.75, dtype=np.float32)
    r = oracle.score(l, [0, vocab - 1], temperature=0.9)
    assert np.allclose(r["lp_full"], -math.log(vocab), rtol=0, atol=1e-11)
    assert np.allclose(r["h_full"], math.log(vocab), rtol=1e-12)
    # no filter: the support is the full vocabulary
    assert np.array_equal(r["support_size"], [vocab, vocab])
    assert np.allclose(r["h_support"], math.log(vocab), rtol=1e-12)
    assert np.allclose(r["lp_support"], -math.log(vocab), atol=1e-11)


def test_uniform_over_recorded_support_is_log_size():
    rng = np.random.default_rng(5)
    l = rng.normal(size=(1, 200))
    ids = np.array([[3, 17, 40, 41, 99, -1, -1]], dtype=np.int32)
    l[0, ids[0, :5]] = 2.5  # equal logits on the support
    r = oracle.score(l, [17], support=ids)
    assert abs(r["h_support"][0] - math.log(5)) < 1e-12
    assert abs(r["lp_support"][0] + math.log(5)) < 1e-12


def test_singleton_support_exact_zeros():
    rng = np.random.default_rng(7)
    l = rng.normal(size=(3, 50)) * 3
    ids = np.array([[4, -1, -1], [-1, 9, -1], [-1, -1, 31]], dtype=np.int32)
    y = [4, 9, 31]
    r = oracle.score(l, y, support=ids)
    assert np.all(r["h_support"] == 0.0)
    assert np.all(r["lp_support"] == 0.0)
    assert np.all(r["valid"] == 1)
    g = oracle.score_grad(l, y, g_h_support=np.ones(3), support=ids)
    assert np.all(g == 0.0)  # zero entropy gradient for a singleton
    g = oracle.score_grad(l, y, g_lp_support=np.ones(3), support=ids)
    assert np.all(g == 0.0)  # lp_S is identically 0


def test_bf16_and_fp32_widening():
    # bf16 patterns and their exact values, widened independently of the oracle
    bits = np.array([[0x3F80, 0xC000, 0x4049, 0x0000, 0xBF00, 0x4180]], dtype=np.uint16)
    vals = np.array([[1.0, -2.0, 3.140625, 0.0, -0.5, 16.0]])
    a = oracle.score(bits, [2])
    b = oracle.score(vals, [2])
    for k in ("lp_full", "h_full"):
        assert a[k][0] == b[k][0]
    f = workloads.bf16_bits_to_f32(bits).astype(np.float32)
    c = oracle.score(f, [2])
    assert c["lp_full"][0] == a["lp_full"][0]


def test_lmhead_logits_match_numpy_matmul():
    rng = np.random.default_rng(11)
    h = workloads.to_bf16_bits(rng.normal(size=(6, 96)).astype(np.float32))
    w = workloads.to_bf16_bits((rng.normal(size=(40, 96)) * 0.02).astype(np.float32))
    sel = np.array([5, 0, 3], dtype=np.int32)
    got = oracle.lmhead_logits(h, w, sel, 0.8)
    hf = workloads.bf16_bits_to_f32(h).astype(np.float64)
    wf = workloads.bf16_bits_to_f32(w).astype(np.float64)
    want = hf[sel] @ wf.T / 0.8
    assert np.allclose(got, want, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------------------
# brute force on tiny rows, written without sorting or prefix scans


def _stable_rank(z):
    """rank_j = #{i : z_i > z_j or (z_i == z_j and i < j)} (descending value,
    ascending id)."""
    n = len(z)
    return np.array([sum(1 for i in range(n) if z[i] > z[j] or (z[i] == z[j] and i < j))
                     for j in range(n)])


def _brute_support(z, k, p, min_p):
    n = len(z)
    rank = _stable_rank(z)
    s1 = [j for j in range(n) if (k <= 0 or k >= n) or rank[j] < k]
    w = np.exp(z - z.max())
    mass1 = w[s1].sum()
    if p < 1.0:
        # smallest cardinality of any subset of S1 whose mass reaches p * mass1
        best = None
        for size in range(1, len(s1) + 1):
            for sub in itertools.combinations(s1, size):
                if w[list(sub)].sum() >= p * mass1:
                    best = size
                    break
            if best is not None:
                break
        s2 = [j for j in s1 if rank[j] < best]
    else:
        s2 = s1
    if min_p > 0:
        s2 = [j for j in s2 if w[j] >= min_p * w.max()]
    return sorted(s2)


def test_brute_force_support_with_ties():
    rng = np.random.default_rng(3)
    checked = 0
    for trial in range(300):
        n = int(rng.integers(2, 11))
        # small integer grid so that ties are frequent
        z = rng.integers(-3, 4, size=n).astype(np.float64) * 0.5
        k = int(rng.integers(0, n + 2))
        p = float(rng.choice([1.0, rng.uniform(0.05, 0.999)]))
        min_p = float(rng.choice([0.0, rng.uniform(0.01, 0.9)]))
        r = oracle.score(z[None, :], [0], top_k=k, top_p=p, min_p=min_p, want_mask=True)
        # skip decisions within rounding distance of the boundary
        if r["topp_margin"][0] < 1e-9 or r["minp_margin"][0] < 1e-9:
            continue
        want = _brute_support(z, k, p, min_p)
        got = sorted(np.nonzero(r["mask"][0])[0].tolist())
        assert got == want, (z, k, p, min_p)
        checked += 1
    assert checked > 250


def test_support_size_monotone_in_p_and_k():
    rng = np.random.default_rng(9)
    l = (rng.normal(size=(4, 300)) * 2).astype(np.float32)
    y = [0, 1, 2, 3]
    prev = np.zeros(4, dtype=np.int64)
    for p in [0.1, 0.3, 0.5, 0.7, 0.9, 0.99, 1.0]:
        s = oracle.score(l, y, top_p=p)["support_size"]
        assert np.all(s >= prev)
        prev = s
    prev = np.zeros(4, dtype=np.int64)
    for k in [1, 2, 5, 20, 100, 299, 0]:
        s = oracle.score(l, y, top_k=k, top_p=0.8)["support_size"]
        assert np.all(s >= prev)
        prev = s


def test_topk_keeps_exactly_k_lowest_ids_on_all_equal_row():
    l = np.zeros((1, 64), dtype=np.float32)
    r = oracle.score(l, [0], top_k=7, want_mask=True)
    assert np.nonzero(r["mask"][0])[0].tolist() == list(range(7))


def test_min_p_to_zero_gives_topp_support():
    rng = np.random.default_rng(1)
    l = rng.normal(size=(3, 500)) * 3
    a = oracle.score(l, [0, 0, 0], top_p=0.9, want_mask=True)
    b = oracle.score(l, [0, 0, 0], top_p=0.9, min_p=1e-300, want_mask=True)
    assert np.array_equal(a["mask"], b["mask"])


# ---------------------------------------------------------------------------
# invariances of the definitions


def test_shift_and_temperature_invariance():
    rng = np.random.default_rng(21)
    l = rng.normal(size=(5, 400)) * 2
    y = rng.integers(0, 400, size=5)
    kw = dict(top_k=100, top_p=0.9, min_p=0.01, want_mask=True)
    a = oracle.score(l, y, temperature=0.7, **kw)
    b = oracle.score(l + 3.25, y, temperature=0.7, **kw)   # constant shift
    c = oracle.score(l * 2.0, y, temperature=1.4, **kw)    # (a l) / (a T)
    for o in (b, c):
        assert np.array_equal(a["mask"], o["mask"])
        for k in ("lp_full", "lp_support", "h_full", "h_support"):
            assert np.allclose(a[k], o[k], rtol=1e-12, atol=1e-11)


# ---------------------------------------------------------------------------
# gradients: central finite differences in fp64


def _fd_check(l, y, T, kind, **filt):
    rows, n = l.shape
    h = 1e-6
    g = np.zeros(rows)
    g[:] = 1.0
    kw = {kind: g}
    grad = oracle.score_grad(l, y, temperature=T, **kw, **filt)
    key = {"g_lp_full": "lp_full", "g_lp_support": "lp_support", "g_h_full": "h_full",
           "g_h_support": "h_support"}[kind]
    fd = np.zeros_like(l)
    for j in range(n):
        lp, lm = l.copy(), l.copy()
        lp[:, j] += h
        lm[:, j] -= h
        fp = oracle.score(lp, y, temperature=T, **filt)[key]
        fm = oracle.score(lm, y, temperature=T, **filt)[key]
        fd[:, j] = (fp - fm) / (2 * h)
    scale = np.abs(fd).max()
    assert np.abs(grad - fd).max() <= 1e-6 * max(scale, 1e-3), kind
    return grad


@pytest.mark.parametrize("kind", ["g_lp_full", "g_lp_support", "g_h_full", "g_h_support"])
def test_finite_difference_computed_support(kind):
    rng = np.random.default_rng(31)
    rows, n = 3, 40
    filt = dict(top_k=25, top_p=0.8, min_p=0.02)
    # continuous logits; keep rows whose support decisions are far from a boundary
    while True:
        l = rng.normal(size=(rows, n)) * 1.5
        r = oracle.score(l, np.zeros(rows, np.int32), temperature=0.8, **filt)
        if (r["topp_margin"].min() > 1e-3 and r["minp_margin"].min() > 1e-3
                and r["topk_gap"].min() > 1e-3):
            break
    # targets inside the support
    mask = oracle.score(l, np.zeros(rows, np.int32), temperature=0.8, want_mask=True,
                        **filt)["mask"]
    y = np.array([np.nonzero(mask[i])[0][-1] for i in range(rows)], dtype=np.int32)
    g = _fd_check(l, y, 0.8, kind, **filt)
    # softmax shift invariance: gradients sum to zero over the row
    assert np.allclose(g.sum(axis=1), 0.0, atol=1e-12)


@pytest.mark.parametrize("kind", ["g_lp_support", "g_h_support"])
def test_finite_difference_recorded_support(kind):
    rng = np.random.default_rng(41)
    l = rng.normal(size=(3, 30)) * 2
    ids = np.array([[1, 5, 7, -1], [-1, 2, 2, 29], [-1, -1, -1, -1]], dtype=np.int32)
    y = np.array([5, 29, 11], dtype=np.int32)  # last row: empty support
    _fd_check(l, y, 1.3, kind, support=ids)


def test_empty_support_gradient_is_full_vocab_logprob_gradient():
    rng = np.random.default_rng(43)
    l = rng.normal(size=(2, 25))
    ids = np.full((2, 3), -1, dtype=np.int32)
    y = np.array([3, 7], dtype=np.int32)
    a = oracle.score_grad(l, y, g_lp_support=np.ones(2), support=ids)
    b = oracle.score_grad(l, y, g_lp_full=np.ones(2))
    assert np.array_equal(a, b)
    r = oracle.score(l, y, support=ids)
    assert np.all(r["valid"] == 0) and np.all(r["lp_support"] == r["lp_full"])


# ---------------------------------------------------------------------------
# L1 distance


def test_l1_identical_rows():
    rng = np.random.default_rng(2)
    d = workloads.to_bf16_bits(rng.normal(size=(3, 1000)).astype(np.float32) * 3)
    r = oracle.l1(d, d.copy(), want_grad=True)
    assert np.all(r["l1"] == 0.0) and np.all(r["accept"] == 1.0)
    assert np.all(r["grad"] == 0.0)


def test_l1_two_point_closed_form():
    a = np.array([0.3, -1.2, 2.0, 5.0])
    d = np.stack([a, np.zeros(4)], axis=1)
    t = np.zeros((4, 2))
    r = oracle.l1(d, t, weight=np.array([1.0, 2.0, 0.5, 0.0]))
    sig = 1.0 / (1.0 + np.exp(-a))
    want = 2.0 * np.abs(sig - 0.5)
    assert np.allclose(r["l1"], want, rtol=1e-13)
    assert np.allclose(r["accept"], 1.0 - np.abs(sig - 0.5), rtol=1e-13)


def test_l1_identities_and_bounds():
    rng = np.random.default_rng(4)
    d = rng.normal(size=(6, 300)) * 3
    t = d + rng.normal(size=(6, 300)) * 0.5
    r = oracle.l1(d, t)
    p = np.exp(d - d.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    q = np.exp(t - t.max(1, keepdims=True))
    q /= q.sum(1, keepdims=True)
    # total-variation identity: 1 - L1 / 2 = sum_j min(p_j, q_j)
    assert np.allclose(1.0 - r["l1"] / 2.0, np.minimum(p, q).sum(1), rtol=1e-12)
    assert np.all((r["l1"] >= 0) & (r["l1"] <= 2))


def test_l1_weighted_loss_special_cases():
    rng = np.random.default_rng(6)
    d = rng.normal(size=(5, 200)) * 2
    t = rng.normal(size=(5, 200)) * 2
    base = oracle.l1(d, t)
    one_hot = oracle.l1(d, t, weight=np.array([0, 0, 1.0, 0, 0]))
    assert abs(one_hot["loss"] - base["l1"][2]) < 1e-15
    equal = oracle.l1(d, t, weight=np.full(5, 0.37))
    assert abs(equal["loss"] - base["l1"].mean()) < 1e-14
    unweighted = oracle.l1(d, t)
    assert abs(unweighted["loss"] - base["l1"].mean()) < 1e-14
    zero = oracle.l1(d, t, weight=np.zeros(5), want_grad=True)
    assert zero["loss"] == 0.0 and np.all(zero["grad"] == 0.0)


def test_l1_finite_difference_gradient():
    rng = np.random.default_rng(8)
    d = rng.normal(size=(2, 20)) * 2
    t = d + rng.normal(size=(2, 20))
    w = np.array([0.3, 0.9])
    r = oracle.l1(d, t, weight=w, want_grad=True)
    h = 1e-6
    fd = np.zeros_like(d)
    for i in range(2):
        for j in range(20):
            dp, dm = d.copy(), d.copy()
            dp[i, j] += h
            dm[i, j] -= h
            fd[i, j] = (oracle.l1(dp, t, weight=w)["loss"] - oracle.l1(dm, t, weight=w)["loss"]) / (2 * h)
    assert np.abs(r["grad"] - fd).max() < 1e-7


def test_dominant_token_entropy_closed_form():
    # one logit L above V-1 equal logits at 0: with d = (V-1) e^-L,
    # H = log1p(d) + L d / (1 + d),  lp(max) = -log1p(d)
    V, L = 4096, 40.0
    l = np.zeros((1, V))
    l[0, 7] = L
    r = oracle.score(l, [7])
    d = (V - 1) * math.exp(-L)
    h = math.log1p(d) + L * d / (1.0 + d)
    assert abs(r["h_full"][0] - h) <= 1e-12 * h
    assert abs(r["lp_full"][0] + math.log1p(d)) <= 1e-12 * math.log1p(d)


# ---------------------------------------------------------------------------
# seeded Gumbel-max sampling: the generator, the logarithm and the sampler,
# each pinned to something other than itself


def test_philox4x64_matches_numpy():
    """The oracle's Philox4x64-10 equals numpy's (a library implementation of
    the same published generator); numpy advances its counter before each
    block, so its first block is the oracle's block at counter + 1,
    including the carry into the next counter word."""
    for key in ([0, 0], [0x123456789ABCDEF0, 0x0FEDCBA987654321], [2**64 - 1, 7]):
        for start in ([0, 0, 0, 0], [5, 0, 0, 0], [2**64 - 1, 0, 0, 0], [2**64 - 2, 3, 1, 9]):
            raw = np.random.Philox(key=np.array(key, np.uint64),
                                   counter=np.array(start, np.uint64)).random_raw(8)
            c = list(start)
            for blk in range(2):
                # counter + 1 as a 256-bit little-endian integer
                v = sum(int(w) << (64 * i) for i, w in enumerate(c)) + 1
                c = [(v >> (64 * i)) & (2**64 - 1) for i in range(4)]
                got = oracle.philox4x64_10(c, key)
                assert np.array_equal(got, raw[4 * blk: 4 * blk + 4]), (key, start, blk)


def test_log_f32_within_two_ulp_of_the_exact_log():
    """The fixed-sequence fp32 logarithm stays within 2 ulp of log(x) over
    the range the sampler feeds it (2^-25 .. 20), including values around 1
    and around the sqrt(2) split, where a dropped series term or a wrong
    reduction would show."""
    xs = np.concatenate([
        np.geomspace(2.0**-25, 20.0, 4001),
        1.0 + np.linspace(-0.05, 0.05, 2001),
        math.sqrt(2.0) * (1.0 + np.linspace(-1e-3, 1e-3, 201)),
        np.array([1.0, 2.0, 0.5, 0.75, 3.0, 1e-7, 17.3]),
    ]).astype(np.float32)
    for x in xs:
        got = float(oracle.log_f32(x))
        want = math.log(float(x))
        ulp = float(np.spacing(np.float32(abs(want)))) if want != 0.0 else 2.0**-149
        assert abs(got - want) <= 2 * ulp + 1e-45, (float(x), got, want)
    assert float(oracle.log_f32(np.float32(1.0))) == 0.0


def test_gumbel_noise_moments():
    """G = -log(-log U) has mean the Euler-Mascheroni constant and variance
    pi^2/6; 40,000 draws along one row must agree within 5 standard errors."""
    g = np.array([oracle.gumbel_f32(11, 3, j) for j in range(40_000)], np.float64)
    n = len(g)
    assert abs(g.mean() - 0.5772156649) < 5 * math.sqrt(math.pi**2 / 6 / n)
    # the sample variance of a Gumbel has standard error ~ sqrt((mu4 - s^4) / n), mu4 = 2.4 pi^4 / 15
    s2 = math.pi**2 / 6
    se = math.sqrt((2.4 * math.pi**4 / 15 - s2**2) / n)
    assert abs(g.var() - s2) < 5 * se
    assert len(set(g.tolist())) > 0.99 * n  # distinct draws per token


def test_gumbel_max_frequencies_follow_the_support_softmax():
    """Over many seeds the sampled token of one row has the distribution
    softmax(l / T) restricted to the support (each probability within 5
    binomial standard errors); tokens outside the support never appear."""
    vocab = 12
    l = np.array([0.5, 2.0, -1.0, 1.0, 3.0, 0.0, 2.5, -0.5, 1.5, 0.25, 2.25, -2.0], np.float32)
    mask = np.array([1, 1, 0, 1, 1, 0, 0, 1, 1, 0, 1, 1], np.uint8)
    T = np.float32(0.8)
    n = 6000
    logits = np.tile(l, (n, 1))
    masks = np.tile(mask, (n, 1))
    # one row, many seeds: draw seed s for row 0 by sampling a 1-row batch
    picks = np.array([oracle.gumbel_sample(logits[:1], T, masks[:1], seed=s)[0] for s in range(n)])
    assert np.all(mask[picks] == 1)
    z = l.astype(np.float64) / float(T)
    q = np.where(mask == 1, np.exp(z - z.max()), 0.0)
    q /= q.sum()
    freq = np.bincount(picks, minlength=vocab) / n
    se = np.sqrt(q * (1 - q) / n)
    assert np.all(np.abs(freq - q) <= 5 * se + 1e-12), (freq, q)


def test_gumbel_sample_edge_cases():
    logits = np.array([[1.0, 2.0, 3.0, 4.0]] * 3, np.float32)
    mask = np.array([[0, 0, 0, 0], [0, 0, 1, 0], [1, 1, 1, 1]], np.uint8)
    got = oracle.gumbel_sample(logits, 1.0, mask, seed=5)
    assert got[0] == -1 and got[1] == 2
    # rows are independent streams: the same logits in another row may differ,
    # and re-running is deterministic
    again = oracle.gumbel_sample(logits, 1.0, mask, seed=5)
    assert np.array_equal(got, again)


def test_prefix_facts_closed_forms():
    """The prefix helper used to check boundary rows: masses and ratios of a
    hand-built row (probabilities 4:3:2:1:0.5), renormalised over the top-k
    set when top-k is active, ids in the total order with ties to the lower
    id."""
    l = np.log(np.array([[2.0, 4.0, 3.0, 0.5, 1.0]]))
    r = oracle.prefix(l, [2], want_ids=True)
    assert r["ids"][0].tolist() == [1, 2]
    assert abs(r["mass_n"][0] - 7 / 10.5) < 1e-15
    assert abs(r["mass_prev"][0] - 4 / 10.5) < 1e-15
    assert abs(r["ratio_n"][0] - 0.75) < 1e-15 and abs(r["ratio_next"][0] - 0.5) < 1e-15
    assert r["nk"][0] == 5
    r = oracle.prefix(l, [3], top_k=3)
    assert abs(r["mass_n"][0] - 1.0) < 1e-15 and abs(r["mass_prev"][0] - 7 / 9) < 1e-15
    assert r["nk"][0] == 3
    r = oracle.prefix(l, [0])
    assert r["mass_n"][0] == 0.0 and r["mass_prev"][0] == 0.0 and r["ratio_n"][0] == 1.0
    ties = np.zeros((1, 6))
    r = oracle.prefix(ties, [4], want_ids=True)
    assert r["ids"][0].tolist() == [0, 1, 2, 3]
    assert abs(r["mass_n"][0] - 4 / 6) < 1e-15
    r = oracle.prefix(ties, [6])
    assert r["ratio_next"][0] == 0.0 and abs(r["mass_n"][0] - 1.0) < 1e-15


def test_lmhead_grad_finite_differences():
    """The fused head's backward in the oracle (projection -> scoring -> VJP)
    against central finite differences of the scalar objective through
    oracle.score on fp64 logits z = H W^T / T, for entries of H and of W,
    with top-k / top-p / min-p active (decisions held fixed away from their
    thresholds)."""
    rng = np.random.default_rng(5)
    rows, vocab, hid, T = 3, 40, 6, 0.7
    H = rng.normal(size=(rows, hid))
    W = rng.normal(size=(vocab, hid)) * 0.8
    y = np.array([0, 5, 39], np.int32)
    z0 = H @ W.T / T
    y[0] = int(np.argmax(z0[0]))  # a target inside the support
    g = [np.array([0.7, -0.2, 1.1]), np.array([1.3, 0.4, -0.5]), np.array([0.2, -0.9, 0.3]),
         np.array([-0.6, 0.8, 0.5])]
    kw = dict(top_k=10, top_p=0.8, min_p=0.05)
    dH, dW = oracle.lmhead_grad(H, W, y, T, *g, **kw)

    def objective(Hm, Wm):
        r = oracle.score(Hm @ Wm.T / T, y, **kw)
        lps = np.where(np.isfinite(r["lp_support"]), r["lp_support"], 0.0)
        return float(np.sum(g[0] * r["lp_full"] + g[1] * lps + g[2] * r["h_full"]
                            + g[3] * r["h_support"]))

    h = 1e-6
    for (i, k) in [(0, 0), (1, 3), (2, 5)]:
        Hp, Hm = H.copy(), H.copy()
        Hp[i, k] += h
        Hm[i, k] -= h
        fd = (objective(Hp, W) - objective(Hm, W)) / (2 * h)
        assert abs(fd - dH[i, k]) <= 1e-6 * max(1.0, abs(fd)), (i, k, fd, dH[i, k])
    for (v, k) in [(int(np.argmax(z0[0])), 2), (7, 1), (39, 4)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[v, k] += h
        Wm[v, k] -= h
        fd = (objective(H, Wp) - objective(H, Wm)) / (2 * h)
        assert abs(fd - dW[v, k]) <= 1e-6 * max(1.0, abs(fd)), (v, k, fd, dW[v, k])
