"""dg_sample_commit against the oracle sampler on identical fp32 logits.

Sampled tokens, argmaxes, commit and re-noise decisions and the stop step must
be bit-exact, except at positions whose decision lies within 1e-4 (log space)
of flipping; those are excluded and counted.
"""
import numpy as np
import pytest
import torch

from oracle import sampler as S
from canvas_denoising_denoise_b200 import synth

pytestmark = pytest.mark.gpu


def gpu_step(logits, tok, committed, prev, status, settings, seed, block, step):
    import canvas_denoising_denoise_b200 as dg
    B, C, V = logits.shape
    dev = "cuda"
    t_tok = torch.as_tensor(tok, dtype=torch.int32).to(dev).contiguous()
    t_com = torch.as_tensor(committed, dtype=torch.uint8).to(dev).contiguous()
    t_prev = torch.as_tensor(prev, dtype=torch.int32).to(dev).contiguous()
    t_stat = torch.as_tensor(status, dtype=torch.int32).to(dev).contiguous()
    out = {"x_hat": torch.empty((B, C), dtype=torch.int32, device=dev),
           "argmax": torch.empty((B, C), dtype=torch.int32, device=dev),
           "logconf": torch.empty((B, C), dtype=torch.float32, device=dev),
           "entropy": torch.empty((B, C), dtype=torch.float32, device=dev),
           "flags": torch.empty((B, C), dtype=torch.uint8, device=dev),
           "near_ties": torch.full((B, 3), -1, dtype=torch.int32, device=dev)}
    dg.sample_commit(logits, t_tok, t_com, t_prev, t_stat, settings, seed, block, step, out=out)
    torch.cuda.synchronize()
    dg.check_device_errors()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res.update(tok=t_tok.cpu().numpy(), committed=t_com.cpu().numpy().astype(bool),
               prev=t_prev.cpu().numpy(), status=t_stat.cpu().numpy())
    return res


def compare(g, r, b, committed_in, counters):
    """Compare GPU sequence b with oracle result r; returns nothing, asserts."""
    near = r.near_tie
    if "near_ties" in g:
        # the device's counters of the decisions it can see near a flip
        assert g["near_ties"][b].tolist() == [int(near["commit_boundary"].sum()),
                                              int(near["renoise"].sum()), int(near["stop"])]
    ok_pos = ~near["gumbel"]
    counters["near_gumbel"] += int(near["gumbel"].sum())
    assert np.array_equal(g["argmax"][b], r.argmax), "raw-logit argmax must be exact"
    assert np.array_equal(g["x_hat"][b][ok_pos], r.x_hat[ok_pos])
    same_x = g["x_hat"][b] == r.x_hat
    np.testing.assert_allclose(g["logconf"][b][same_x], r.logconf[same_x], atol=2e-4, rtol=0)
    np.testing.assert_allclose(g["entropy"][b], r.entropy, atol=2e-4, rtol=1e-5)
    global_tie = (near["commit_boundary"].any() or near["stop"] or
                  (near["gumbel"] & ~committed_in).any())
    if global_tie:
        counters["skipped_sequences"] += 1
        return
    renoise_ok = ~near["renoise"]
    counters["near_renoise"] += int(near["renoise"].sum())
    g_commit = (g["flags"][b] & 1) != 0
    g_renoise = (g["flags"][b] & 2) != 0
    committed_now = ~committed_in & r.committed
    assert np.array_equal(g_commit[renoise_ok], committed_now[renoise_ok])
    assert np.array_equal(g_renoise[renoise_ok], r.renoise_mask[renoise_ok])
    assert np.array_equal(g["tok"][b][renoise_ok], r.tok[renoise_ok])
    assert np.array_equal(g["committed"][b][renoise_ok], r.committed[renoise_ok])
    assert (g["status"][b] != 0) == r.stopped


@pytest.mark.parametrize("B,C,V,step", [(2, 256, 512, 0), (3, 200, 1000, 17), (1, 64, 4096, 47)])
def test_sampler_parity_small(B, C, V, step):
    import canvas_denoising_denoise_b200 as dg
    rng = np.random.default_rng(B * 1000 + V + step)
    logits = synth.make_sampler_logits(B, C, V, seed=5, step=step)
    tok = rng.integers(0, V, size=(B, C))
    committed = rng.random((B, C)) < 0.3
    prev = rng.integers(0, V, size=(B, C))
    settings = dg.SamplerSettings()
    scfg = S.SamplerCfg()
    g = gpu_step(logits.cuda(), tok, committed, prev, np.zeros(B), settings, 11, 2, step)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    lg = logits.numpy()
    for b in range(B):
        r = S.sampler_step(scfg, lg[b], tok[b], committed[b], prev[b], step, 11, b, 2)
        compare(g, r, b, committed[b], counters)
    print("near-tie counts", counters)
    assert counters["skipped_sequences"] < B


def test_sampler_parity_full_vocab():
    """The sampler workload row size (V = 262144), one sequence, mid-schedule."""
    import canvas_denoising_denoise_b200 as dg
    B, C, V, step = 1, 256, 262144, 20
    logits = synth.make_sampler_logits(B, C, V, seed=1, step=step)
    rng = np.random.default_rng(3)
    tok = rng.integers(0, V, size=(B, C))
    committed = rng.random((B, C)) < 0.25
    prev = np.full((B, C), -1)
    g = gpu_step(logits.cuda(), tok, committed, prev, np.zeros(B), dg.SamplerSettings(), 7, 0,
                 step)
    r = S.sampler_step(S.SamplerCfg(), logits[0].numpy(), tok[0], committed[0], prev[0], step, 7,
                       0, 0)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    compare(g, r, 0, committed[0], counters)
    print("near-tie counts", counters)
    # the one sequence was compared in full, not skipped as a global tie
    assert counters["skipped_sequences"] == 0
    assert int((g["flags"][0] & 1).sum()) == 16


@pytest.mark.parametrize("B,seqs", [(4, (0, 1, 2, 3)), (16, (0, 6, 15))])
def test_sampler_parity_full_vocab_batched(B, seqs):
    """The sampler sweep's batches (B = 4 and 16, V = 262144) in one call; the
    oracle checks every sequence at B = 4 and three of them at B = 16
    (sequences are independent: each has its own Philox key)."""
    import canvas_denoising_denoise_b200 as dg
    C, V, step = 256, 262144, 31
    logits = synth.make_sampler_logits(B, C, V, seed=8, step=step, device="cuda")
    rng = np.random.default_rng(B)
    tok = rng.integers(0, V, size=(B, C))
    committed = rng.random((B, C)) < 0.25
    prev = rng.integers(0, V, size=(B, C))
    prev[:, ::3] = -1
    g = gpu_step(logits, tok, committed, prev, np.zeros(B), dg.SamplerSettings(), 21, 4, step)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    for b in seqs:
        r = S.sampler_step(S.SamplerCfg(), logits[b].cpu().numpy(), tok[b], committed[b], prev[b],
                           step, 21, b, 4)
        compare(g, r, b, committed[b], counters)
    print("near-tie counts", counters)
    assert counters["skipped_sequences"] == 0


def test_frozen_sequences_are_untouched():
    import canvas_denoising_denoise_b200 as dg
    B, C, V = 2, 32, 256
    logits = synth.make_sampler_logits(B, C, V, seed=2, step=0)
    tok = np.arange(B * C).reshape(B, C) % V
    status = np.array([5, 0])
    g = gpu_step(logits.cuda(), tok, np.zeros((B, C), bool), np.full((B, C), -1), status,
                 dg.SamplerSettings(), 0, 0, 3)
    assert np.array_equal(g["tok"][0], tok[0]) and g["status"][0] == 5
    assert (g["flags"][1] & 1).sum() == 16


@pytest.mark.parametrize("policy", [0, 1])
def test_unselected_policy_on_device(policy):
    import canvas_denoising_denoise_b200 as dg
    B, C, V, step = 1, 64, 512, 4
    logits = synth.make_sampler_logits(B, C, V, seed=9, step=step)
    tok = np.zeros((B, C), dtype=np.int64)
    committed = np.zeros((B, C), bool)
    g = gpu_step(logits.cuda(), tok, committed, np.full((B, C), -1), np.zeros(B),
                 dg.SamplerSettings(unselected_policy=policy), 4, 1, step)
    r = S.sampler_step(S.SamplerCfg(unselected_policy=policy), logits[0].numpy(), tok[0],
                       committed[0], None, step, 4, 0, 1)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    compare(g, r, 0, committed[0], counters)
    assert counters["skipped_sequences"] == 0
    assert np.array_equal(g["tok"][0], r.tok)
    unsel = ~r.commit_mask
    if policy == 0:  # unselected positions hold the step's sample
        assert np.array_equal(g["tok"][0][unsel], g["x_hat"][0][unsel])
    else:            # unselected positions hold a fresh uniform token
        assert not np.array_equal(g["tok"][0][unsel], g["x_hat"][0][unsel])


def test_sixteen_step_completion_on_device():
    """Re-noise off and k = 16: a 256-token canvas completes in exactly 16 steps."""
    import canvas_denoising_denoise_b200 as dg
    B, C, V = 1, 256, 512
    settings = dg.SamplerSettings(renoise_conf=0.0)
    dev = "cuda"
    tok = torch.zeros((B, C), dtype=torch.int32, device=dev)
    com = torch.zeros((B, C), dtype=torch.uint8, device=dev)
    prev = torch.full((B, C), -1, dtype=torch.int32, device=dev)
    stat = torch.zeros(B, dtype=torch.int32, device=dev)
    for s in range(48):
        logits = synth.make_sampler_logits(B, C, V, seed=3, step=s).cuda()
        dg.sample_commit(logits, tok, com, prev, stat, settings, 0, 0, s)
        if int(stat.item()) != 0:
            break
    assert int(stat.item()) == 16 and int(com.sum().item()) == C


@pytest.mark.parametrize("step", [3, 20])
def test_entropy_bounded_selection_parity(step):
    """DG_SELECT_ENTROPY against the oracle: half the positions carry one
    planted token raised by U(6, 14), so their entropies spread from ~0.4
    nats down to ~0 and the summed-entropy bound cuts inside that range."""
    import canvas_denoising_denoise_b200 as dg
    B, C, V = 2, 256, 512
    rng = np.random.default_rng(100 + step)
    logits = rng.normal(size=(B, C, V)).astype(np.float32)
    sharp = rng.random((B, C)) < 0.5
    bi, ci = np.nonzero(sharp)
    logits[bi, ci, rng.integers(0, V, size=bi.size)] += rng.uniform(6, 14, size=bi.size)
    logits = torch.from_numpy(logits)
    tok = rng.integers(0, V, size=(B, C))
    committed = rng.random((B, C)) < 0.2
    prev = rng.integers(0, V, size=(B, C))
    settings = dg.SamplerSettings(selection=1, entropy_bound=0.1)
    scfg = S.SamplerCfg(selection=S.SELECT_ENTROPY, entropy_bound=0.1)
    g = gpu_step(logits.cuda(), tok, committed, prev, np.zeros(B), settings, 9, 1, step)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    n_commit = []
    for b in range(B):
        r = S.sampler_step(scfg, logits[b].numpy(), tok[b], committed[b], prev[b], step, 9, b, 1)
        compare(g, r, b, committed[b], counters)
        n_commit.append(int(r.commit_mask.sum()))
    assert max(n_commit) > 1  # the bound admitted several positions
    assert counters["skipped_sequences"] < B


def test_near_tie_counters_on_planted_margins():
    """The device's near-tie counters against the oracle's classifier on rows
    whose deciding quantity is planted 0.5e-4 inside or 2e-4 outside the
    margin (two live outcomes, two far below: closed-form confidences and
    entropies, as in the oracle's own pins)."""
    import math
    import canvas_denoising_denoise_b200 as dg
    V, step, block = 4, 3, 0
    T = S.temperature(S.SamplerCfg(), step)

    def rows(deltas):
        lg = np.full((1, len(deltas), V), -1e4 * T, dtype=np.float32)
        lg[0, :, 0] = np.asarray(deltas) * T
        lg[0, :, 1] = 0.0
        return torch.from_numpy(lg)

    def run_case(deltas, committed, settings, scfg, want):
        lg = rows(deltas)
        C = len(deltas)
        tok = np.zeros((1, C), dtype=np.int64)
        com = np.asarray(committed, bool).reshape(1, C)
        for seed in range(100):  # a seed under which the uncommitted rows sample outcome 0
            r = S.sampler_step(scfg, lg[0].numpy(), tok[0], com[0], None, step, seed, 0, block)
            if np.all(r.x_hat[~com[0]] == 0):
                break
        g = gpu_step(lg.cuda(), tok, com, np.full((1, C), -1), np.zeros(1), settings, seed,
                     block, step)
        got = g["near_ties"][0].tolist()
        assert got == [int(r.near_tie["commit_boundary"].sum()), int(r.near_tie["renoise"].sum()),
                       int(r.near_tie["stop"])]
        assert got == want
        assert np.array_equal(g["x_hat"][0], r.x_hat)

    softplus = lambda x: math.log1p(math.exp(x))
    sp_inv = lambda y: math.log(math.expm1(y))

    def h_delta(h):  # two-outcome delta > 0 with entropy h
        lo, hi = 1e-9, 60.0
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            p = 1 / (1 + math.exp(-mid))
            lo, hi = (mid, hi) if -(p * math.log(p) + (1 - p) * math.log(1 - p)) > h else (lo, mid)
        return 0.5 * (lo + hi)

    topk = (dg.SamplerSettings(commit_k=1), S.SamplerCfg(commit_k=1))
    for gap, n in ((0.5e-4, 2), (2e-4, 0)):
        run_case([3.0, -sp_inv(softplus(-3.0) + gap)], [False, False], *topk, want=[n, 0, 0])
    ent = (dg.SamplerSettings(selection=1, entropy_bound=0.1),
           S.SamplerCfg(selection=S.SELECT_ENTROPY, entropy_bound=0.1))
    for e, n in ((0.5e-4, 2), (2e-4, 0)):
        run_case([h_delta(x) for x in (0.05 + e, 0.02, 0.03)], [False] * 3, *ent, want=[n, 0, 0])
    for e, n in ((0.5e-4, 1), (2e-4, 0)):
        run_case([h_delta(x) for x in (0.05 - e, 0.02, 0.03)], [False] * 3, *ent, want=[n, 0, 0])
    dflt = (dg.SamplerSettings(), S.SamplerCfg())
    lt = math.log(0.05)
    offs = [-0.5e-4, 0.5e-4, -2e-4, 2e-4]
    run_case([-sp_inv(-(lt + o)) for o in offs], [True] * 4, *dflt, want=[0, 2, 0])
    for off, n in ((0.5e-4, 1), (-2e-4, 0)):
        run_case([h_delta(0.005 + off)] * 4, [True] * 4, *dflt, want=[0, 0, n])
