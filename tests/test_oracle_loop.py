"""The oracle's composed loop: prefill, denoise to stop, block commit, next canvas."""
import numpy as np

from oracle import loop as LP
from oracle import model as M
from oracle import sampler as S
from test_oracle_model import rand_weights

SMALL = M.ModelCfg(d=32, n_layers=2, n_q_heads=2, n_kv_heads=1, head_dim=16, ffn=64, vocab=64)


def test_random_model_runs_to_the_step_cap_and_commits():
    # Random weights give confidences near 1/V, far below 0.05: every committed
    # token is re-noised on the next step, so the canvas never completes and the
    # loop ends at the 48-step cap with a final fill.
    w = rand_weights(SMALL, seed=2, std=0.02)
    scfg = S.SamplerCfg()
    prompt = np.arange(8) % SMALL.vocab
    trace = []
    kc, vc = M.empty_cache(SMALL, 8 + 2 * 32)
    L = M.prefill(SMALL, w, prompt, kc, vc)
    tok, steps, L2 = LP.denoise_block(SMALL, w, scfg, kc, vc, L, seed=0, b=0, block=0, canvas=32,
                                      trace=trace)
    assert steps == 48 and L2 == L + 32
    assert trace[-1]["result"].reason == "cap"
    for t in trace[:-1]:
        r = t["result"]
        assert r.commit_mask.sum() == 16
        assert np.array_equal(r.renoise_mask, t["committed_in"])


def test_generate_two_blocks_matches_prefill_of_the_output():
    w = rand_weights(SMALL, seed=4, std=0.02)
    scfg = S.SamplerCfg(max_steps=6)
    prompt = (np.arange(8) * 7) % SMALL.vocab
    toks, steps = LP.generate(SMALL, w, scfg, prompt, n_blocks=2, seed=3, canvas=32)
    assert toks.shape == (64,) and steps == [6, 6]
    # the second canvas is conditioned on the first: different Philox block index
    assert not np.array_equal(toks[:32], toks[32:])
