"""Pins of the oracle sampler against the settings the pages fix and against invariants."""
import heapq
import math

import numpy as np
import pytest

from conftest import sampler_settings
from oracle import philox as P
from oracle import sampler as S


def cfg(**kw):
    return S.SamplerCfg(**kw)


def test_defaults_match_the_published_settings():
    ss = sampler_settings()
    c = S.SamplerCfg()
    assert c.max_steps == ss["max_steps"]
    assert c.t_start == ss["t_start"] and c.t_end == ss["t_end"]
    assert c.stop_entropy == ss["stop_entropy"]
    assert ss["commit_min"] <= c.commit_k <= ss["commit_max"]


def test_temperature_schedule_linear_endpoints():
    c = S.SamplerCfg()
    ts = [S.temperature(c, s) for s in range(c.max_steps)]
    assert ts[0] == 0.8
    assert ts[-1] == pytest.approx(0.4, abs=1e-15)
    d = np.diff(ts)
    assert np.allclose(d, d[0], rtol=0, atol=1e-15) and d[0] < 0


def test_gumbel_max_frequencies_follow_softmax():
    # Gumbel-max theorem: P(x_hat = v) = softmax(l / T)_v.
    logits = np.array([[0.0, 1.0, -0.5, 0.3]], dtype=np.float32)
    c = S.SamplerCfg()
    temp = S.temperature(c, 10)
    p = np.exp(logits[0] / temp)
    p /= p.sum()
    n = 6000
    counts = np.zeros(4)
    for pos in range(n):
        st = S.position_stats(logits[0], temp, seed=3, b=0, block=0, step=10, pos=pos)
        counts[st.x_hat] += 1
    chi2 = float(np.sum((counts - n * p) ** 2 / (n * p)))
    assert chi2 < 20  # 3 dof


def test_low_temperature_sample_is_argmax():
    rng = np.random.default_rng(1)
    row = rng.normal(size=64).astype(np.float32)
    row[17] += 5.0
    st = S.position_stats(row, 1e-3, seed=0, b=0, block=0, step=0, pos=0)
    assert st.x_hat == 17 and st.argmax == 17


def test_entropy_closed_forms():
    v = 512
    st = S.position_stats(np.zeros(v, dtype=np.float32), 0.8, 0, 0, 0, 0, 0)
    assert st.entropy == pytest.approx(math.log(v), rel=1e-12)
    row = np.zeros(v, dtype=np.float32)
    row[3] = 50.0
    st = S.position_stats(row, 0.4, 0, 0, 0, 0, 0)
    assert st.entropy < 1e-40 or st.entropy == pytest.approx(0.0, abs=1e-40)
    assert st.x_hat == 3 and st.argmax == 3
    # two-way tie: H = ln 2
    row = np.full(v, -1e4, dtype=np.float32)
    row[[5, 9]] = 0.0
    st = S.position_stats(row, 0.5, 0, 0, 0, 0, 0)
    assert st.entropy == pytest.approx(math.log(2), rel=1e-9)
    assert st.argmax == 5  # ties go to the lower index


def test_commit_count_and_topk_bruteforce():
    rng = np.random.default_rng(2)
    C, V = 64, 40
    logits = rng.normal(scale=2.0, size=(C, V)).astype(np.float32)
    tok = rng.integers(0, V, size=C)
    committed = np.zeros(C, dtype=bool)
    committed[rng.choice(C, 10, replace=False)] = True
    c = cfg(renoise_conf=0.0)
    r = S.sampler_step(c, logits, tok, committed, None, 3, seed=1, b=0, block=0)
    assert r.commit_mask.sum() == 16
    assert not np.any(r.commit_mask & committed)
    unc = np.flatnonzero(~committed)
    best = heapq.nlargest(16, unc.tolist(), key=lambda i: (r.logconf[i], -i))
    assert set(best) == set(np.flatnonzero(r.commit_mask).tolist())
    assert np.all(r.tok[r.commit_mask] == r.x_hat[r.commit_mask])


def test_logconf_definition_on_both_sets():
    rng = np.random.default_rng(3)
    C, V = 8, 16
    logits = rng.normal(size=(C, V)).astype(np.float32)
    tok = rng.integers(0, V, size=C)
    committed = np.array([1, 0, 1, 0, 0, 1, 0, 0], dtype=bool)
    c = S.SamplerCfg()
    r = S.sampler_step(c, logits, tok, committed, None, 5, 0, 0, 0)
    temp = S.temperature(c, 5)
    for i in range(C):
        p = np.exp(logits[i].astype(np.float64) / temp)
        p /= p.sum()
        x = tok[i] if committed[i] else r.x_hat[i]
        assert r.logconf[i] == pytest.approx(math.log(p[x]), abs=1e-12)


def test_completes_in_sixteen_steps_without_renoise():
    # k = 16 on a 256-token canvas with re-noise off: exactly 16 steps.
    rng = np.random.default_rng(4)
    C, V = 256, 32
    c = cfg(renoise_conf=0.0)
    tok = S.init_canvas(0, 0, 0, C, V)
    committed = np.zeros(C, dtype=bool)
    prev = None
    for s in range(c.max_steps):
        logits = rng.normal(size=(C, V)).astype(np.float32)
        r = S.sampler_step(c, logits, tok, committed, prev, s, 0, 0, 0)
        assert r.commit_mask.sum() == 16
        tok, committed, prev = r.tok, r.committed, r.argmax
        if r.stopped:
            break
    assert s == 15 and r.reason == "complete"
    ss = __import__("conftest").sampler_settings()
    assert ss["typical_steps_min"] <= s + 1 <= ss["typical_steps_max"]


def test_renoise_fires_iff_confidence_below_threshold():
    C, V = 6, 32
    c = S.SamplerCfg()
    temp = S.temperature(c, 2)
    # committed tokens with planted softmax confidences on either side of 0.05
    confs = [0.9, 0.2, 0.051, 0.049, 0.01, 0.5]
    logits = np.zeros((C, V), dtype=np.float64)
    tok = np.zeros(C, dtype=np.int64)
    for i, q in enumerate(confs):
        # confidence q on token 0, the rest uniform: z0 - z_rest = ln(q (V-1) / (1-q))
        logits[i, 0] = temp * math.log(q * (V - 1) / (1 - q))
    logits = logits.astype(np.float32)
    committed = np.ones(C, dtype=bool)
    r = S.sampler_step(c, logits, tok, committed, None, 2, 0, 0, 0)
    lam = r.logconf
    assert np.all(r.renoise_mask == (lam < math.log(0.05)))
    assert list(r.renoise_mask) == [False, False, False, True, True, False]
    for i in np.flatnonzero(r.renoise_mask):
        assert r.tok[i] == S.renoise_token(0, 0, 0, 2, i, V) and not r.committed[i]
    for i in np.flatnonzero(~r.renoise_mask):
        assert r.tok[i] == tok[i] and r.committed[i]


def test_never_renoised_tokens_stay_fixed():
    rng = np.random.default_rng(7)
    C, V = 64, 50
    c = S.SamplerCfg()
    tok = S.init_canvas(1, 0, 0, C, V)
    committed = np.zeros(C, dtype=bool)
    prev = None
    first_value = {}
    renoised = set()
    for s in range(c.max_steps):
        logits = rng.normal(scale=0.5, size=(C, V)).astype(np.float32)
        # make each committed token confident so most survive
        for i in np.flatnonzero(committed):
            logits[i, tok[i]] += 6.0
        r = S.sampler_step(c, logits, tok, committed, prev, s, 1, 0, 0)
        renoised |= set(np.flatnonzero(r.renoise_mask).tolist())
        for i in np.flatnonzero(r.commit_mask):
            first_value.setdefault(int(i), int(r.tok[i]))
        tok, committed, prev = r.tok, r.committed, r.argmax
        if r.stopped:
            break
    for i, v0 in first_value.items():
        if i not in renoised:
            assert tok[i] == v0


def test_stop_on_entropy_and_identical_predictions():
    C, V = 32, 64
    c = S.SamplerCfg()
    rng = np.random.default_rng(8)
    planted = rng.integers(0, V, size=C)
    logits = np.zeros((C, V), dtype=np.float32)
    logits[np.arange(C), planted] = 50.0
    tok = S.init_canvas(0, 0, 0, C, V)
    committed = np.zeros(C, dtype=bool)
    prev = None
    for s in range(c.max_steps):
        r = S.sampler_step(c, logits, tok, committed, prev, s, 0, 0, 0)
        tok, committed, prev = r.tok, r.committed, r.argmax
        if r.stopped:
            break
    assert s == 1 and r.reason == "entropy"
    assert np.all(tok == planted) and np.all(committed)


def test_random_logits_run_to_the_cap():
    C, V = 32, 64
    c = S.SamplerCfg()
    rng = np.random.default_rng(9)
    tok = S.init_canvas(0, 0, 0, C, V)
    committed = np.zeros(C, dtype=bool)
    prev = None
    for s in range(c.max_steps):
        logits = rng.normal(scale=0.01, size=(C, V)).astype(np.float32)
        r = S.sampler_step(c, logits, tok, committed, prev, s, 0, 0, 0)
        tok, committed, prev = r.tok, r.committed, r.argmax
        if r.stopped:
            break
    assert s == c.max_steps - 1 and r.reason == "cap" and np.all(committed)


def test_unselected_policies():
    rng = np.random.default_rng(10)
    C, V = 40, 30
    logits = rng.normal(size=(C, V)).astype(np.float32)
    tok = rng.integers(0, V, size=C)
    committed = np.zeros(C, dtype=bool)
    keep = S.sampler_step(cfg(), logits, tok, committed, None, 4, 2, 0, 1)
    ren = S.sampler_step(cfg(unselected_policy=S.POLICY_RENOISE), logits, tok, committed, None,
                         4, 2, 0, 1)
    assert np.all(keep.commit_mask == ren.commit_mask)
    uns = ~keep.commit_mask
    assert np.all(keep.tok[uns] == keep.x_hat[uns]) and not np.any(keep.committed[uns])
    for i in np.flatnonzero(uns):
        assert ren.tok[i] == S.renoise_token(2, 0, 1, 4, i, V)


def test_canvas_init_uniform_and_keyed():
    a = S.init_canvas(0, 0, 0, 256, 512)
    b = S.init_canvas(0, 0, 1, 256, 512)
    c = S.init_canvas(0, 1, 0, 256, 512)
    assert a.min() >= 0 and a.max() < 512
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    assert a[0] == P.token_from_word(P.position_word(0, 0, 0, 0, 0, P.TAG_INIT), 512)


def two_outcome_logits(ps, T, V=4):
    """Rows whose tempered softmax is (p, 1 - p, 0, ...): z = (ln p, ln(1 - p), -inf...)."""
    rows = np.full((len(ps), V), -1e30)
    for i, p in enumerate(ps):
        rows[i, 0] = T * math.log(p)
        rows[i, 1] = T * math.log1p(-p)
    return rows


def binary_entropy(p):
    return -p * math.log(p) - (1 - p) * math.log1p(-p)


def test_entropy_bounded_selection_worked_example():
    """GDocs table row "Selecao de token" (entropy limit 0.1), worked by hand.

    Six positions with two-outcome softmaxes p = 0.99, 0.5, 0.999, 0.98,
    0.995, 0.9 have entropies 0.0560, 0.6931, 0.0079, 0.0980, 0.0314,
    0.3251 nats.  In increasing entropy: positions 2, 4, 0, 3, 5, 1 with
    running sums 0.0079, 0.0393, 0.0953, 0.1933, ...  The bound 0.1 admits
    the first three: positions {2, 4, 0} are committed, the rest are not.
    """
    ss = sampler_settings()
    c = cfg(selection=S.SELECT_ENTROPY, entropy_bound=ss["select_entropy"], renoise_conf=0.0)
    step = 5
    ps = [0.99, 0.5, 0.999, 0.98, 0.995, 0.9]
    logits = two_outcome_logits(ps, S.temperature(c, step))
    r = S.sampler_step(c, logits, np.zeros(6, dtype=int), np.zeros(6, dtype=bool), None, step,
                       seed=0, b=0, block=0)
    for p, h in zip(ps, r.entropy):
        assert h == pytest.approx(binary_entropy(p), abs=1e-12)
    assert sorted(np.flatnonzero(r.commit_mask).tolist()) == [0, 2, 4]


def test_entropy_bounded_selection_always_progresses_and_skips_committed():
    """All entropies above the bound: exactly the lowest-entropy uncommitted
    position is committed; committed positions are never reselected."""
    c = cfg(selection=S.SELECT_ENTROPY, renoise_conf=0.0)
    step = 2
    ps = [0.9, 0.8, 0.7, 0.95, 0.6]          # entropies 0.325 .. 0.673, all > 0.1
    logits = two_outcome_logits(ps, S.temperature(c, step))
    committed = np.array([False, False, False, True, False])  # 0.95 is the lowest, but committed
    r = S.sampler_step(c, logits, np.zeros(5, dtype=int), committed, None, step, seed=0, b=0,
                       block=0)
    assert np.flatnonzero(r.commit_mask).tolist() == [0]  # p = 0.9 is the lowest uncommitted


def test_entropy_bounded_selection_invariants_on_random_rows():
    """The committed set is a prefix of the entropy order of U whose sum is
    within the bound unless it is a single position, and the next position
    would break the bound."""
    rng = np.random.default_rng(7)
    C, V = 48, 64
    sharp = rng.random(C) < 0.5
    logits = rng.normal(size=(C, V))
    logits[sharp, rng.integers(0, V, size=sharp.sum())] += rng.uniform(8, 30, size=sharp.sum())
    committed = rng.random(C) < 0.2
    c = cfg(selection=S.SELECT_ENTROPY, renoise_conf=0.0)
    r = S.sampler_step(c, logits, rng.integers(0, V, size=C), committed, None, 4, seed=3, b=0,
                       block=0)
    chosen = np.flatnonzero(r.commit_mask)
    unc = np.flatnonzero(~committed)
    assert len(chosen) >= 1 and not np.any(committed[chosen])
    worst_in = max(r.entropy[chosen])
    rest = np.setdiff1d(unc, chosen)
    assert rest.size == 0 or min(r.entropy[rest]) >= worst_in
    total = float(np.sum(r.entropy[chosen]))
    assert len(chosen) == 1 or total <= c.entropy_bound
    if rest.size:
        assert total + min(r.entropy[rest]) > c.entropy_bound
    assert len(chosen) > 1  # the sharp rows have tiny entropies: several fit
