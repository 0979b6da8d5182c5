"""dg_unembed_sample_commit: the unembedding fused with one sampler step.

The oracle computes the logits h w_u^T in fp64 (rounded to fp32, as the GPU
keeps them) and runs its sampler step on them; the fused GPU path must agree
exactly on every decision outside the oracle's near-tie margins and to
rounding on the log confidences and entropies.  At the full vocabulary the
fused path is also checked against the unfused one (dg_unembed followed by
dg_sample_commit), with the oracle's per-position statistics on sampled rows.
"""
import numpy as np
import pytest
import torch

from oracle import sampler as S
from test_gpu_sampler import compare

pytestmark = pytest.mark.gpu


def rand_bf16(shape, scale, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def make_case(B, C, V, d, seed, commit_frac):
    """h ~ N(0, 1), w_u ~ N(0, 3/sqrt(d)): logits with the spread of the sampler workload."""
    h = rand_bf16((B * C, d), 1.0, seed)
    w = rand_bf16((V, d), 3.0 / d ** 0.5, seed + 1)
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, V, size=(B, C))
    committed = rng.random((B, C)) < commit_frac
    prev = rng.integers(0, V, size=(B, C))
    return h, w, tok, committed, prev


def run(path, h, w, tok, committed, prev, settings, seed, block, step):
    import canvas_denoising_denoise_b200 as dg
    B, C = tok.shape
    dev = "cuda"
    t_tok = torch.as_tensor(tok, dtype=torch.int32).to(dev).contiguous()
    t_com = torch.as_tensor(committed, dtype=torch.uint8).to(dev).contiguous()
    t_prev = torch.as_tensor(prev, dtype=torch.int32).to(dev).contiguous()
    t_stat = torch.zeros(B, dtype=torch.int32, device=dev)
    out = {"x_hat": torch.empty((B, C), dtype=torch.int32, device=dev),
           "argmax": torch.empty((B, C), dtype=torch.int32, device=dev),
           "logconf": torch.empty((B, C), dtype=torch.float32, device=dev),
           "entropy": torch.empty((B, C), dtype=torch.float32, device=dev),
           "flags": torch.empty((B, C), dtype=torch.uint8, device=dev),
           "near_ties": torch.full((B, 3), -1, dtype=torch.int32, device=dev)}
    hd, wd = h.to(dev), w.to(dev)
    if path == "fused":
        dg.unembed_sample_commit(hd, wd, t_tok, t_com, t_prev, t_stat, settings, seed, block,
                                 step, out=out)
    else:
        logits = torch.empty((B * C, w.shape[0]), dtype=torch.float32, device=dev)
        dg.unembed(hd, wd, logits)
        dg.sample_commit(logits.view(B, C, -1), t_tok, t_com, t_prev, t_stat, settings, seed,
                         block, step, out=out)
    torch.cuda.synchronize()
    dg.check_device_errors()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res.update(tok=t_tok.cpu().numpy(), committed=t_com.cpu().numpy().astype(bool),
               prev=t_prev.cpu().numpy(), status=t_stat.cpu().numpy())
    return res


# (B, C, V, d, step): several vocabulary segments per pair; C = 200 leaves a
# ragged token tile; B = 3 x 200 spans three token tiles; step 47 is the
# final step (fill, no re-noise); step 0 has no previous prediction.
@pytest.mark.parametrize("B,C,V,d,step", [(1, 256, 512, 256, 0), (2, 256, 4096, 512, 9),
                                          (1, 200, 8192, 256, 17), (3, 200, 2048, 128, 33),
                                          (1, 256, 1024, 2048, 47)])
def test_fused_step_against_oracle(B, C, V, d, step):
    import canvas_denoising_denoise_b200 as dg
    h, w, tok, committed, prev = make_case(B, C, V, d, seed=B * 100 + V + step,
                                           commit_frac=0.3)
    g = run("fused", h, w, tok, committed, prev, dg.SamplerSettings(), 13, 3, step)
    logits = (h.double() @ w.double().T).float().numpy().reshape(B, C, V)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    for b in range(B):
        r = S.sampler_step(S.SamplerCfg(), logits[b], tok[b], committed[b], prev[b], step, 13, b,
                           3)
        compare(g, r, b, committed[b], counters)
    assert counters["skipped_sequences"] < B or B == 1
    print("near-tie counts", counters)


def test_fused_matches_unfused_at_full_vocab():
    """256 x 262144 x 2048, mid-schedule: fused vs dg_unembed + dg_sample_commit,
    and both against the oracle on all 256 rows."""
    import canvas_denoising_denoise_b200 as dg
    B, C, V, d, step = 1, 256, 262144, 2048, 20
    h, w, tok, committed, prev = make_case(B, C, V, d, seed=77, commit_frac=0.25)
    settings = dg.SamplerSettings()
    f = run("fused", h, w, tok, committed, prev, settings, 7, 0, step)
    u = run("unfused", h, w, tok, committed, prev, settings, 7, 0, step)
    # identical logits, different merge order: decisions agree, sums to rounding
    assert (f["argmax"] != u["argmax"]).sum() == 0
    assert (f["x_hat"] != u["x_hat"]).sum() <= 1
    same = f["x_hat"] == u["x_hat"]
    np.testing.assert_allclose(f["logconf"][same], u["logconf"][same], rtol=0, atol=1e-4)
    np.testing.assert_allclose(f["entropy"], u["entropy"], rtol=1e-5, atol=1e-5)
    if same.all():
        assert np.array_equal(f["flags"], u["flags"])
        assert np.array_equal(f["tok"], u["tok"])
        assert np.array_equal(f["committed"], u["committed"])
    # every row against the oracle's sampler on the fp64 logits (rounded to
    # fp32): bit-exact decisions outside its near-ties; a sample on which the
    # fused and unfused paths differ must be one of those near-ties
    logits = (h.double() @ w.double().T).float().numpy()
    r = S.sampler_step(S.SamplerCfg(), logits, tok[0], committed[0], prev[0], step, 7, 0, 0)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    compare(f, r, 0, committed[0], counters)
    compare(u, r, 0, committed[0], counters)
    assert counters["skipped_sequences"] == 0
    assert np.all(r.near_tie["gumbel"][~same[0]])
    print("near-tie counts", counters, "fused/unfused sample differences", int((~same).sum()))


def test_fused_step_entropy_bounded_selection():
    """The fused path with DG_SELECT_ENTROPY against the oracle."""
    import canvas_denoising_denoise_b200 as dg
    B, C, V, d, step = 1, 256, 1024, 256, 12
    h, w, tok, committed, prev = make_case(B, C, V, d, seed=4242, commit_frac=0.2)
    # sharpen half the rows: adding 18 w_t / |w_t|^2 to h raises logit t by 18
    g = torch.Generator().manual_seed(5)
    rows = torch.randperm(C, generator=g)[: C // 2]
    targets = torch.randint(0, V, (rows.numel(),), generator=g)
    hf = h.float()
    wf = w.float()
    hf[rows] += 18.0 * wf[targets] / wf[targets].norm(dim=1, keepdim=True) ** 2
    h = hf.to(torch.bfloat16)
    settings = dg.SamplerSettings(selection=1, entropy_bound=0.1)
    gres = run("fused", h, w, tok, committed, prev, settings, 13, 3, step)
    logits = (h.double() @ w.double().T).float().numpy().reshape(B, C, V)
    counters = {"near_gumbel": 0, "near_renoise": 0, "skipped_sequences": 0}
    r = S.sampler_step(S.SamplerCfg(selection=S.SELECT_ENTROPY, entropy_bound=0.1), logits[0],
                       tok[0], committed[0], prev[0], step, 13, 0, 3)
    compare(gres, r, 0, committed[0], counters)
    assert int(r.commit_mask.sum()) > 1
