"""The block-autoregressive denoising loop, composed from the oracle's model and sampler.

TEST INFRASTRUCTURE ONLY: only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.

Order of work per request ("DiffusionGemma Guia do Desenvolvedor ...",
section "Block Autoregressive Diffusion para Sequencias Longas"; aiexpert.news
architecture paragraph): causal prefill of the prompt into the KV cache; then
per 256-token canvas: random placeholder tokens, denoising steps until the
adaptive stop, causal re-encode of the finished block, append of its K/V to the
cache, and the next canvas conditioned on everything committed so far.
"""
import numpy as np

from . import model as M
from . import sampler as S


def denoise_block(mcfg, weights, scfg, k_cache, v_cache, prefix_len, seed, b, block,
                  canvas=256, bf16_storage=True, trace=None):
    """Denoise one canvas of one sequence to its stop; commit its K/V.

    Returns (final tokens [canvas], steps taken, new cache length).
    If `trace` is a list, one dict per step is appended (tokens in, logits, result).
    """
    tok = S.init_canvas(seed, b, block, canvas, mcfg.vocab)
    committed = np.zeros(canvas, dtype=bool)
    prev = None
    steps = 0
    for s in range(scfg.max_steps):
        logits = M.denoise_logits(mcfg, weights, tok, k_cache, v_cache, prefix_len, bf16_storage)
        logits32 = logits.astype(np.float32)
        res = S.sampler_step(scfg, logits32, tok, committed, prev, s, seed, b, block)
        if trace is not None:
            trace.append({"step": s, "tok_in": tok.copy(), "committed_in": committed.copy(),
                          "logits": logits32, "result": res})
        tok, committed, prev = res.tok, res.committed, res.argmax
        steps = s + 1
        if res.stopped:
            break
    new_len = M.block_commit(mcfg, weights, tok, k_cache, v_cache, prefix_len, bf16_storage)
    return tok, steps, new_len


def generate(mcfg, weights, scfg, prompt, n_blocks, seed, b=0, canvas=256, bf16_storage=True):
    """Prefill + n_blocks canvases for one sequence.  Returns (tokens, steps per block)."""
    lmax = len(prompt) + n_blocks * canvas
    k_cache, v_cache = M.empty_cache(mcfg, lmax)
    length = M.prefill(mcfg, weights, prompt, k_cache, v_cache, bf16_storage)
    out, steps = [], []
    for j in range(n_blocks):
        tok, st, length = denoise_block(mcfg, weights, scfg, k_cache, v_cache, length, seed, b, j,
                                        canvas, bf16_storage)
        out.append(tok)
        steps.append(st)
    return np.concatenate(out), steps
