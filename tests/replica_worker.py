"""Rank body of the world-size-2 gloo tests (imported by spawned processes).

Each rank joins a gloo process group through the same helpers the benchmark
uses on NCCL, runs its replica's sampler step with the CPU oracle on its own
seeded inputs, and takes part in the timing reduction.  The result is put on a
queue for the parent test to check.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_rank(rank, world, port, queue, canvas, vocab, fake_elapsed, leave_early=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    try:
        import numpy as np
        import torch.distributed as dist

        from canvas_denoising_denoise_b200 import replicas, synth
        from oracle import sampler as S

        env = replicas.rank_env()
        replicas.init("gloo", timeout_s=20)
        seeds = replicas.replica_seeds(env.rank)
        prompt = synth.make_prompt(1, 32, vocab, seed=seeds.prompt)
        logits = synth.make_sampler_logits(1, canvas, vocab, seed=seeds.sampler, step=0)
        tok = S.init_canvas(seeds.sampler, 0, 0, canvas, vocab)
        res = S.sampler_step(S.SamplerCfg(), logits[0].numpy(), tok, np.zeros(canvas, bool),
                             None, 0, seeds.sampler, 0, 0)
        if leave_early and env.rank == 1:
            # a rank that leaves between steps: it never reaches the timing
            # reduction, so the other rank's collective must end with an error
            queue.put((env.rank, {"left": True}))
            return
        try:
            replicas.barrier(env.world)
        except Exception as e:
            queue.put((env.rank, {"collective_error": f"{type(e).__name__}: {e}"}))
            return
        m = replicas.max_over_ranks(fake_elapsed[env.rank], env.world)
        rate = replicas.whole_job_rate(canvas, env.world, m)
        gathered = [None] * env.world
        dist.all_gather_object(gathered, prompt.numpy().tolist())
        replicas.finish(env.world)
        queue.put((env.rank, {"max_elapsed": m, "rate": rate, "prompts": gathered,
                              "tok": res.tok.tolist(), "committed": res.committed.tolist()}))
    except Exception as e:  # reported to the parent, which fails the test
        queue.put((rank, {"error": f"{type(e).__name__}: {e}"}))
