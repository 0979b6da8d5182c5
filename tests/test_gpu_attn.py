"""tcgen05 canvas attention (dg_canvas_attn) against the oracle's fp64 attention."""
import math

import numpy as np
import pytest
import torch

from helpers import assert_close, to64
from oracle import model as M
from canvas_denoising_denoise_b200 import synth

pytestmark = pytest.mark.gpu


def oracle_attn(q, kn, vn, kc, vc, lens, Hq, Hkv, hd, causal):
    B, Lq = q.shape[0], q.shape[1]
    out = np.zeros((B, Lq, Hq * hd))
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        L = int(lens[b])
        qb = to64(q[b]).reshape(Lq, Hq, hd)
        knb = to64(kn[b]).reshape(Lq, Hkv, hd)
        vnb = to64(vn[b]).reshape(Lq, Hkv, hd)
        o = M.gqa_attention(qb, knb, vnb, to64(kc[b])[:, :L], to64(vc[b])[:, :L], causal,
                            1 / math.sqrt(hd))
        out[b] = o.reshape(Lq, Hq * hd)
    return out


def run_case(B, Hq, Hkv, hd, Lq, lens, lmax, causal, seed=0, check_lse=False):
    import canvas_denoising_denoise_b200 as dg
    q, kn, vn, kc, vc = synth.make_attn_inputs(B, Hq, Hkv, hd, Lq, max(lens), seed=seed,
                                               lmax=lmax)
    cl = torch.tensor(lens, dtype=torch.int32)
    out = torch.zeros((B, Lq, Hq * hd), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, Hq, Lq), dtype=torch.float32, device="cuda")
    dg.canvas_attn(q.cuda(), kn.cuda(), vn.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), max(lens),
                   out, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=hd, lse=lse,
                   mask=dg.MASK_CAUSAL if causal else dg.MASK_BIDIR)
    torch.cuda.synchronize()
    dg.check_device_errors()
    want = oracle_attn(q, kn, vn, kc, vc, lens, Hq, Hkv, hd, causal)
    assert_close(out.cpu(), want, what=f"attn B{B} hd{hd} Lq{Lq} L{lens} causal{causal}")
    return out


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,lens", [(256, [0]), (256, [1]), (256, [127]), (256, [129]),
                                     (256, [300]), (64, [64]), (200, [77]), (384, [513])])
def test_attention_shapes(hd, causal, Lq, lens):
    run_case(1, 4, 2, hd, Lq, lens, lmax=max(lens) + 40, causal=causal)


@pytest.mark.parametrize("hd", [64, 128])
def test_attention_batch_ragged_prefix_and_gqa(hd):
    # different prefix length per sequence; rows beyond each length hold noise
    run_case(3, 8, 2, hd, 256, [100, 700, 0], lmax=800, causal=False, seed=3)
    run_case(2, 4, 4, hd, 256, [257, 5], lmax=300, causal=True, seed=4)


@pytest.mark.parametrize("L", [4096, 16384, 32768])
def test_attention_microbench_shape_sampled(L):
    """The attention microbench shape, Q [32, 256, 128] over KV [8, L, 128]
    plus the canvas's own 256 keys: rows sampled from every 128-row query
    tile of every head (so from every CTA and every key split) against the
    oracle's attention."""
    import canvas_denoising_denoise_b200 as dg
    B, Hq, Hkv, hd, Lq = 1, 32, 8, 128, 256
    q, kn, vn, kc, vc = synth.make_attn_inputs(B, Hq, Hkv, hd, Lq, L, seed=7)
    out = torch.zeros((B, Lq, Hq * hd), dtype=torch.bfloat16, device="cuda")
    dg.canvas_attn(q.cuda(), kn.cuda(), vn.cuda(), kc.cuda(), vc.cuda(),
                   torch.tensor([L], dtype=torch.int32, device="cuda"), L, out, n_q_heads=Hq,
                   n_kv_heads=Hkv, head_dim=hd)
    torch.cuda.synchronize()
    dg.check_device_errors()
    rng = np.random.default_rng(L)
    got = to64(out.cpu())
    for g in range(Hkv):
        k = np.concatenate([to64(kc[0, g]), to64(kn[0, :, g * hd:(g + 1) * hd])])
        v = np.concatenate([to64(vc[0, g]), to64(vn[0, :, g * hd:(g + 1) * hd])])
        for h in range(g * (Hq // Hkv), (g + 1) * (Hq // Hkv)):
            rows = np.concatenate([rng.integers(0, 128, size=3), rng.integers(128, 256, size=3)])
            qh = to64(q[0, rows, h * hd:(h + 1) * hd])
            want = M.attention_head(qh, k, v, np.ones((len(rows), len(k)), bool), hd ** -0.5)
            assert_close(got[0, rows, h * hd:(h + 1) * hd], want, what=f"L {L} head {h}")


def test_permutation_equivariance_on_device():
    import canvas_denoising_denoise_b200 as dg
    B, Hq, Hkv, hd, Lq, L = 1, 4, 2, 64, 256, 100
    q, kn, vn, kc, vc = synth.make_attn_inputs(B, Hq, Hkv, hd, Lq, L, seed=11)
    perm = torch.randperm(Lq, generator=torch.Generator().manual_seed(0))
    cl = torch.tensor([L], dtype=torch.int32, device="cuda")
    outs = []
    for p in (None, perm):
        qq, kk, vv = (q, kn, vn) if p is None else (q[:, p], kn[:, p], vn[:, p])
        o = torch.zeros((B, Lq, Hq * hd), dtype=torch.bfloat16, device="cuda")
        dg.canvas_attn(qq.contiguous().cuda(), kk.contiguous().cuda(), vv.contiguous().cuda(),
                       kc.cuda(), vc.cuda(), cl, L, o, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=hd)
        outs.append(o)
    torch.cuda.synchronize()
    dg.check_device_errors()
    # only the fp32 summation order within the canvas tile changes
    assert_close(outs[1].cpu(), to64(outs[0].cpu())[:, perm.numpy()], rel_l2=1e-3, max_abs=1.6e-2,
                 what="equivariance")
