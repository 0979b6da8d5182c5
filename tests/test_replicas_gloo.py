"""The N>1 host path on CPU: two gloo ranks running independent replicas.

The denoising path shards as independent replicas (no data-path exchange), so
what multi-GPU runs add is host logic: per-rank seeds, the barrier, the
maximum of the per-rank times and the whole-job rate.  These tests run that
logic with world size 2 on the gloo backend and check each rank's replica
against the same replica computed alone in this process.
"""
import multiprocessing as mp
import socket

import numpy as np
import pytest

from replica_worker import run_rank

CANVAS, VOCAB = 64, 512


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, fake_elapsed, leave_early=False, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=run_rank,
                         args=(r, world, port, q, CANVAS, VOCAB, fake_elapsed, leave_early))
             for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            rank, res = q.get(timeout=timeout)
            out[rank] = res
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_rank_env_and_seeds():
    from canvas_denoising_denoise_b200 import replicas
    e = replicas.rank_env({"RANK": "1", "WORLD_SIZE": "4", "LOCAL_RANK": "1"})
    assert (e.rank, e.world, e.local) == (1, 4, 1)
    assert replicas.rank_env({}) == replicas.RankEnv(0, 1, 0)
    with pytest.raises(ValueError):
        replicas.rank_env({"RANK": "4", "WORLD_SIZE": "4"})
    seeds = {replicas.replica_seeds(r) for r in range(8)}
    assert len({s.prompt for s in seeds}) == 8 and len({s.sampler for s in seeds}) == 8
    # one rank: the reduction is the identity and the rate is units / time
    assert replicas.max_over_ranks(0.25, 1) == 0.25
    assert replicas.whole_job_rate(256, 1, 0.5) == 512.0
    assert replicas.whole_job_rate(256, 8, 0.5) == 4096.0
    with pytest.raises(ValueError):
        replicas.whole_job_rate(256, 1, 0.0)


def test_two_gloo_ranks_run_independent_replicas():
    from canvas_denoising_denoise_b200 import replicas, synth
    from oracle import sampler as S
    fake = [0.75, 1.25]
    out = _run(2, fake)
    for r in (0, 1):
        assert "error" not in out[r], out[r]
    # the slowest rank's time on every rank; rate = all ranks' tokens / that time
    for r in (0, 1):
        assert out[r]["max_elapsed"] == 1.25
        assert out[r]["rate"] == pytest.approx(2 * CANVAS / 1.25)
    # every rank saw both prompts, and they differ (distinct replicas)
    assert out[0]["prompts"] == out[1]["prompts"]
    assert out[0]["prompts"][0] != out[0]["prompts"][1]
    # each rank's step equals the same replica run alone: nothing crossed ranks
    for r in (0, 1):
        seeds = replicas.replica_seeds(r)
        assert out[r]["prompts"][r] == synth.make_prompt(1, 32, VOCAB,
                                                         seed=seeds.prompt).numpy().tolist()
        logits = synth.make_sampler_logits(1, CANVAS, VOCAB, seed=seeds.sampler, step=0)
        tok = S.init_canvas(seeds.sampler, 0, 0, CANVAS, VOCAB)
        res = S.sampler_step(S.SamplerCfg(), logits[0].numpy(), tok, np.zeros(CANVAS, bool),
                             None, 0, seeds.sampler, 0, 0)
        assert out[r]["tok"] == res.tok.tolist()
        assert out[r]["committed"] == res.committed.tolist()
    assert out[0]["tok"] != out[1]["tok"]


def test_rank_leaving_between_steps_ends_the_others_collective_with_an_error():
    out = _run(2, [1.0, 1.0], leave_early=True)
    assert out[1] == {"left": True}
    assert "collective_error" in out[0], out[0]
