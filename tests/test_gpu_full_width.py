"""The composed path at the full model's widths against the oracle.

Layer shapes of the full workload (d = 2048, 16 q / 8 kv heads, head_dim 128,
MLP 8192, vocabulary 262144) with 2 layers, over a seeded prefix cache that is
written identically into the device state and into the oracle's cache (so no
oracle prefill is needed):

* one bidirectional forward of a 256-token canvas over a 4096-row prefix
  (the split-K projections, the 2048-wide RMSNorm, hd = 128 attention inside
  the model, the K = 8192 MLP down projection): logits of
  sampled rows within rel-L2 1e-2 and max-abs 3e-2 of the oracle's;
* the block driver (fused unembedding + sampler, step advance, final fill,
  causal re-encode and block commit), teacher-forced: the oracle's sampler is
  run on the GPU's own logits of the GPU's canvas at every step, and the
  driver's decisions must match it bit for bit outside the oracle's near-ties;
* eight sequences at once (2048 canvas tokens: every projection on the
  CTA-pair pipeline), sampled sequences
  against the oracle.

Sources: Google docs page "DiffusionGemma", bullet "Arquitetura de
codificador-decodificador" (the canvas over the cached prefix); "DiffusionGemma
Guia do Desenvolvedor ...", section "Block Autoregressive Diffusion para
Sequencias Longas" (block commit into the cache).
"""
import dataclasses

import numpy as np
import pytest
import torch

from helpers import assert_close, assert_close_bf16, to64
from oracle import model as M
from oracle import sampler as S
from canvas_denoising_denoise_b200 import synth

pytestmark = pytest.mark.gpu

SHAPE = dataclasses.replace(synth.FULL, n_layers=2)
OCFG = M.ModelCfg(SHAPE.d, SHAPE.n_layers, SHAPE.n_q_heads, SHAPE.n_kv_heads, SHAPE.head_dim,
                  SHAPE.ffn, SHAPE.vocab, SHAPE.eps)
C = 256


class _EmbedRows:
    """Row access to the bf16 embedding as fp64, without an fp64 copy of the
    whole table (the oracle only gathers the canvas rows)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, idx):
        return self.t[torch.as_tensor(np.asarray(idx, dtype=np.int64))].double().numpy()


@pytest.fixture(scope="module")
def full():
    import canvas_denoising_denoise_b200 as dg
    w_cpu = synth.make_weights(SHAPE, seed=0)
    w_gpu = {"embed": w_cpu["embed"].cuda(), "unembed": w_cpu["unembed"].cuda(),
             "layers": [{k: v.cuda() for k, v in lw.items()} for lw in w_cpu["layers"]]}
    model = dg.DgModel(SHAPE, w_gpu)
    w64 = {"embed": _EmbedRows(w_cpu["embed"]), "unembed": w_cpu["unembed"].double().numpy(),
           "layers": [{k: v.double().numpy() for k, v in lw.items()} for lw in w_cpu["layers"]]}
    return dg, model, w64


def seeded_prefix(P, seed):
    """Per-layer prefix K/V [Hkv, P, hd] in bf16, N(0, 1)."""
    g = torch.Generator().manual_seed(seed)
    shape = (SHAPE.n_kv_heads, P, SHAPE.head_dim)
    return [(torch.randn(shape, generator=g).to(torch.bfloat16),
             torch.randn(shape, generator=g).to(torch.bfloat16)) for _ in range(SHAPE.n_layers)]


def state_with_prefix(dg, prefixes, P, lmax):
    """A device state whose sequence b holds prefixes[b] in cache rows [0, P)."""
    st = dg.DgState(SHAPE, len(prefixes), lmax, C)
    for b, pre in enumerate(prefixes):
        for l, (k, v) in enumerate(pre):
            st.k_cache[l][b, :, :P].copy_(k)
            st.v_cache[l][b, :, :P].copy_(v)
    st.cache_len.fill_(P)
    st.cache_len_host = P
    return st


def oracle_cache(pre, P, lmax):
    kc, vc = M.empty_cache(OCFG, lmax)
    for l, (k, v) in enumerate(pre):
        kc[l][:, :P] = k.double().numpy()
        vc[l][:, :P] = v.double().numpy()
    return kc, vc


def gpu_logits(dg, model, st, canvas):
    st.tok.copy_(torch.as_tensor(canvas, dtype=torch.int32).view(st.batch, C))
    logits = torch.empty((st.batch, C, SHAPE.vocab), dtype=torch.float32, device="cuda")
    dg.denoise_logits(model, st, logits)
    torch.cuda.synchronize()
    dg.check_device_errors()
    return logits


def test_full_width_denoise_logits_match_oracle(full):
    import canvas_denoising_denoise_b200 as dg
    _, model, w64 = full
    P = 4096
    assert dg.model_residual_on_pairs(model, C) == 0  # one canvas: the split-K projections
    pre = seeded_prefix(P, seed=11)
    st = state_with_prefix(dg, [pre], P, P + C)
    canvas = synth.make_prompt(1, C, SHAPE.vocab, seed=12)[0].numpy()
    logits = gpu_logits(dg, model, st, canvas)
    rows = np.sort(np.random.default_rng(13).choice(C, size=48, replace=False))
    kc, vc = oracle_cache(pre, P, P + C)
    want = M.denoise_logits(OCFG, w64, canvas, kc, vc, P, rows=rows)
    assert_close(logits[0, torch.as_tensor(rows)].cpu(), want, what="full-width logits")


def test_full_width_block_driver_teacher_forced(full):
    """Two sampler steps (max_steps = 2: a top-16 commit at T = 0.8, then the
    cap's final fill at T = 0.4), then the causal re-encode and block commit."""
    import canvas_denoising_denoise_b200 as dg
    _, model, w64 = full
    P = 4096
    pre = seeded_prefix(P, seed=21)
    scfg = S.SamplerCfg(max_steps=2)
    settings = dg.SamplerSettings(max_steps=2)
    # a sampler seed whose first step has no near-tie, so that the driver's
    # canvas after step 0 is fixed and step 1 can be teacher-forced from it
    st_tf = state_with_prefix(dg, [pre], P, P + C)
    for seed in range(4):
        tok0 = S.init_canvas(seed, 0, 0, C, SHAPE.vocab)
        l0 = gpu_logits(dg, model, st_tf, tok0)[0].cpu().numpy()
        r0 = S.sampler_step(scfg, l0, tok0, np.zeros(C, bool), None, 0, seed, 0, 0)
        if not (r0.near_tie["gumbel"].any() or r0.near_tie["commit_boundary"].any()):
            break
    else:
        raise AssertionError("every tried seed has a near-tie in step 0")
    assert int(r0.commit_mask.sum()) == 16 and not r0.stopped
    l1 = gpu_logits(dg, model, st_tf, r0.tok)[0].cpu().numpy()
    r1 = S.sampler_step(scfg, l1, r0.tok, r0.committed, r0.argmax, 1, seed, 0, 0)
    assert r1.stopped and r1.reason == "cap"

    st = state_with_prefix(dg, [pre], P, P + C)
    steps = dg.denoise_block(model, st, settings, seed, 0)
    torch.cuda.synchronize()
    dg.check_device_errors()
    assert steps == 2 and st.seq_status.tolist() == [2]
    assert st.cache_len.tolist() == [P + C] and st.cache_len_host == P + C
    assert bool(st.committed.all())
    got = st.tok[0].cpu().numpy()
    # the fill takes every position's step-1 sample; near-ties may differ
    ok = ~r1.near_tie["gumbel"]
    print("step-1 gumbel near-ties:", int((~ok).sum()))
    assert np.array_equal(got[ok], r1.tok[ok])
    # the 16 positions committed in step 0 keep the step-0 sample
    assert np.array_equal(got[r0.commit_mask], r0.tok[r0.commit_mask])

    # the block's K/V: the oracle's causal re-encode of the driver's tokens
    kc, vc = oracle_cache(pre, P, P + C)
    M.block_commit(OCFG, w64, got, kc, vc, P)
    for l in range(SHAPE.n_layers):
        assert_close_bf16(st.k_cache[l][0, :, P:P + C].cpu(), kc[l][:, P:P + C], what=f"block K {l}")
        assert_close_bf16(st.v_cache[l][0, :, P:P + C].cpu(), vc[l][:, P:P + C], what=f"block V {l}")


def test_full_width_eight_sequences_pair_path(full):
    import canvas_denoising_denoise_b200 as dg
    _, model, w64 = full
    Bn, P = 8, 2048
    assert dg.model_residual_on_pairs(model, Bn * C) == 1  # every projection on CTA pairs
    pres = [seeded_prefix(P, seed=100 + b) for b in range(Bn)]
    st = state_with_prefix(dg, pres, P, P + C)
    canvas = synth.make_prompt(Bn, C, SHAPE.vocab, seed=31).numpy()
    logits = gpu_logits(dg, model, st, canvas)
    rng = np.random.default_rng(32)
    for b in (0, 5, 7):
        rows = np.sort(rng.choice(C, size=32, replace=False))
        kc, vc = oracle_cache(pres[b], P, P + C)
        want = M.denoise_logits(OCFG, w64, canvas[b], kc, vc, P, rows=rows)
        assert_close(logits[b, torch.as_tensor(rows)].cpu(), want, what=f"sequence {b}")
