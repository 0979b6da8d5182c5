"""Pins of the oracle's near-tie classifier (oracle.sampler.sampler_step).

The GPU parity tests drop positions (or whole sequences) from bit-exact
comparison when the oracle says a decision sits within 1e-4 (log space) of
flipping.  A classifier that over- or under-flags would silently weaken or
break them, so each flag is pinned here on rows built in closed form so that
the quantity it watches lies just inside or just outside the margin:

  gumbel           the top-2 gap of the Gumbel-perturbed scores z + g
  argmax           the top-2 gap of the raw logits
  commit_boundary  the confidence gap at the top-k cut, or the entropy-bounded
                   cut moving (a prefix sum or a rank swap near the bound)
  renoise          a committed position's confidence near ln 0.05
  stop             the mean entropy near 0.005

Rows are two-outcome wherever possible, whose softmax quantities have closed
forms: with z = (delta, 0), the log confidence of outcome 0 is -softplus(-delta)
and the entropy is that of a Bernoulli(sigmoid(delta)).
"""
import math

import numpy as np

from oracle import sampler as S
from oracle.philox import TAG_GUMBEL, uniform_from_word, vocab_words

MARGIN = 1e-4
INSIDE = (0.5e-4, 0.9e-4)
OUTSIDE = (1.1e-4, 2e-4)
SEED, BLOCK, STEP = 5, 0, 3


def temp():
    return S.temperature(S.SamplerCfg(), STEP)


def softplus(x):
    return math.log1p(math.exp(x))


def softplus_inv(y):
    return math.log(math.expm1(y))


def bern_entropy(delta):
    p = 1.0 / (1.0 + math.exp(-delta))
    return -(p * math.log(p) + (1 - p) * math.log(1 - p))


def delta_for_entropy(h):
    """delta > 0 with bern_entropy(delta) = h (bisection; the entropy falls with delta)."""
    lo, hi = 1e-9, 60.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if bern_entropy(mid) > h:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def step(logits, tok, committed, cfg=S.SamplerCfg(), seed=SEED, prev=None):
    return S.sampler_step(cfg, np.asarray(logits, dtype=np.float64), np.asarray(tok),
                          np.asarray(committed, dtype=bool), prev, STEP, seed, 0, BLOCK)


def test_gumbel_flag_fires_exactly_inside_the_margin():
    V = 8
    gaps = INSIDE + OUTSIDE
    T = temp()
    rows = []
    for pos, gap in enumerate(gaps):
        g = S.gumbel_noise(uniform_from_word(vocab_words(SEED, 0, BLOCK, STEP, pos, TAG_GUMBEL,
                                                         V)))
        score = np.full(V, -3.0)
        score[0], score[1] = 1.0, 1.0 - gap
        rows.append(T * (score - g))  # z + g = the planned scores
    r = step(rows, np.zeros(len(gaps), int), np.ones(len(gaps), bool))
    assert np.array_equal(r.x_hat, np.zeros(len(gaps)))
    assert r.near_tie["gumbel"].tolist() == [True, True, False, False]


def test_argmax_flag_fires_exactly_inside_the_margin():
    V = 8
    gaps = INSIDE + OUTSIDE
    rows = []
    for gap in gaps:
        row = np.zeros(V)
        row[2], row[5] = 1.0, 1.0 - gap
        rows.append(row)
    r = step(rows, np.zeros(len(gaps), int), np.ones(len(gaps), bool))
    assert np.array_equal(r.argmax, np.full(len(gaps), 2))
    assert r.near_tie["argmax"].tolist() == [True, True, False, False]


def two_outcome(deltas):
    T = temp()
    return [T * np.array([d, 0.0]) for d in deltas]


def seed_with_sample_zero(deltas, committed):
    """A sampler seed under which every uncommitted row samples outcome 0, so
    that its log confidence is -softplus(-delta)."""
    for seed in range(100):
        r = step(two_outcome(deltas), np.zeros(len(deltas), int), committed, seed=seed)
        if np.all(r.x_hat[~np.asarray(committed)] == 0):
            return seed
    raise AssertionError("no seed samples outcome 0 everywhere")


def test_topk_commit_boundary_flag():
    """k = 1 over two uncommitted positions whose confidences differ by `gap`."""
    cfg = S.SamplerCfg(commit_k=1)
    d0 = 3.0
    for gap, want in [(g, True) for g in INSIDE] + [(g, False) for g in OUTSIDE]:
        d1 = -softplus_inv(softplus(-d0) + gap)  # lambda_1 = lambda_0 - gap
        committed = np.zeros(2, bool)
        seed = seed_with_sample_zero([d0, d1], committed)
        r = step(two_outcome([d0, d1]), np.zeros(2, int), committed, cfg, seed)
        assert abs((r.logconf[0] - r.logconf[1]) - gap) < 1e-12
        assert r.commit_mask.tolist() == [True, False]
        assert r.near_tie["commit_boundary"].tolist() == [want, want], gap


def entropy_case(entropies):
    cfg = S.SamplerCfg(selection=S.SELECT_ENTROPY, entropy_bound=0.1)
    deltas = [delta_for_entropy(h) for h in entropies]
    n = len(entropies)
    r = step(two_outcome(deltas), np.zeros(n, int), np.zeros(n, bool), cfg)
    np.testing.assert_allclose(r.entropy, entropies, rtol=0, atol=1e-12)
    return r


def test_entropy_cut_prefix_sum_just_above_the_bound():
    # sorted entropies 0.02, 0.03, 0.05 + e: the sum of all three is 0.1 + e
    for e, want in [(x, True) for x in INSIDE] + [(x, False) for x in OUTSIDE]:
        r = entropy_case([0.05 + e, 0.02, 0.03])
        assert r.commit_mask.tolist() == [False, True, True]
        assert r.near_tie["commit_boundary"].tolist() == [want, False, want], e


def test_entropy_cut_everything_selected_just_below_the_bound():
    # the sum of all three is 0.1 - e: all selected, the last would drop out
    # if the sum rose by e
    for e, want in [(x, True) for x in INSIDE] + [(x, False) for x in OUTSIDE]:
        r = entropy_case([0.05 - e, 0.02, 0.03])
        assert r.commit_mask.tolist() == [True, True, True]
        assert r.near_tie["commit_boundary"].tolist() == [want, False, False], e


def test_entropy_cut_rank_swap_at_the_cut():
    # sorted 0.02, 0.06, 0.06 + e: the cut falls between two near-equal entropies
    for e, want in [(x, True) for x in INSIDE] + [(x, False) for x in OUTSIDE]:
        r = entropy_case([0.06 + e, 0.06, 0.02])
        assert r.commit_mask.tolist() == [False, True, True]
        assert r.near_tie["commit_boundary"].tolist() == [want, want, False], e


def test_renoise_flag_fires_exactly_inside_the_margin():
    log_tau = math.log(0.05)
    offsets = [-INSIDE[0], INSIDE[1], -OUTSIDE[0], OUTSIDE[1]]
    deltas = [-softplus_inv(-(log_tau + o)) for o in offsets]  # lambda = ln 0.05 + o
    n = len(deltas)
    r = step(two_outcome(deltas), np.zeros(n, int), np.ones(n, bool))
    np.testing.assert_allclose(r.logconf, [log_tau + o for o in offsets], rtol=0, atol=1e-12)
    assert r.near_tie["renoise"].tolist() == [True, True, False, False]
    assert r.renoise_mask.tolist() == [True, False, True, False]


def test_stop_flag_fires_exactly_inside_the_margin():
    n = 4
    for off, want in [(-INSIDE[0], True), (INSIDE[1], True), (-OUTSIDE[0], False),
                      (OUTSIDE[1], False)]:
        d = delta_for_entropy(0.005 + off)
        r = step(two_outcome([d] * n), np.zeros(n, int), np.ones(n, bool))
        assert abs(float(np.mean(r.entropy)) - (0.005 + off)) < 1e-12
        assert bool(r.near_tie["stop"]) == want, off
