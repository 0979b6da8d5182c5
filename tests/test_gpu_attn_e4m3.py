"""e4m3 canvas attention (dg_canvas_attn_e4m3) against the oracle's FP8 attention.

The inputs are e4m3 codes that the oracle's quantiser makes from seeded bf16
draws (per-token query scales, one K and one V scale), passed to both sides.
Two bars:
  * exact probabilities: integer scores in log2 units, so every probability is
    a power of two that e4m3 holds exactly whatever maximum it is taken against;
    the output then matches to the bf16 rounding of the result;
  * random N(0, 1) inputs: the kernel rounds its probabilities against a running
    maximum that lags the row's (by a factor up to 2^8), the oracle against the
    row's own, so single roundings differ; the bar is 1.5 times what moving the
    oracle's reference by half a binade does to its own output.
"""
import math

import numpy as np
import pytest
import torch

from helpers import to64
from oracle import fp8
from canvas_denoising_denoise_b200 import synth

pytestmark = pytest.mark.gpu

HD = 128


def pad16(n):
    return (n + 15) // 16 * 16


def device_inputs(q8, qs, kn8, vn8, kc8, vc8, ks, vs):
    """Device tensors in the kernel's layouts from oracle-layout codes.

    q8 [B, Lq, Hq*hd], qs [B*Lq]; kn8/vn8 [B, Lq, Hkv*hd]; kc8/vc8 [B, Hkv, lmax, hd]."""
    B, Lq = q8.shape[0], q8.shape[1]
    Hkv, lmax = kc8.shape[1], kc8.shape[2]
    vt_new = np.zeros((B, Hkv, HD, pad16(Lq)), dtype=np.uint8)
    vt_new[..., :Lq] = vn8.reshape(B, Lq, Hkv, HD).transpose(0, 2, 3, 1)
    vt_cache = np.ascontiguousarray(vc8.transpose(0, 1, 3, 2))
    cuda = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    f32 = lambda a: torch.tensor(np.atleast_1d(np.asarray(a, dtype=np.float32))).cuda()
    return dict(q=cuda(q8), q_scale=f32(qs), k_new=cuda(kn8), vt_new=cuda(vt_new),
                k_cache=cuda(kc8), vt_cache=cuda(vt_cache), k_scale=f32(ks), v_scale=f32(vs))


def run_gpu(d, lens, lmax_prefix, Hq, Hkv, causal):
    import canvas_denoising_denoise_b200 as dg
    B, Lq = d["q"].shape[0], d["q"].shape[1]
    out = torch.zeros((B, Lq, Hq * HD), dtype=torch.bfloat16, device="cuda")
    dg.canvas_attn_e4m3(d["q"], d["q_scale"], d["k_new"], d["vt_new"], d["k_cache"],
                        d["vt_cache"], d["k_scale"], d["v_scale"],
                        torch.tensor(lens, dtype=torch.int32, device="cuda"), lmax_prefix, out,
                        n_q_heads=Hq, n_kv_heads=Hkv,
                        mask=dg.MASK_CAUSAL if causal else dg.MASK_BIDIR)
    torch.cuda.synchronize()
    dg.check_device_errors()
    return to64(out.cpu())


def oracle(q8, qs, kn8, vn8, kc8, vc8, ks, vs, lens, Hq, Hkv, causal, shift=0.0):
    B, Lq = q8.shape[0], q8.shape[1]
    out = np.zeros((B, Lq, Hq * HD))
    for b in range(B):
        L = int(lens[b])
        o = fp8.gqa_attention_e4m3(q8[b].reshape(Lq, Hq, HD), qs[b * Lq:(b + 1) * Lq],
                                   kn8[b].reshape(Lq, Hkv, HD), vn8[b].reshape(Lq, Hkv, HD),
                                   kc8[b][:, :L], vc8[b][:, :L], ks, vs, causal,
                                   1 / math.sqrt(HD), shift)
        out[b] = o.reshape(Lq, Hq * HD)
    return out


def quantise(q, kn, vn, kc, vc):
    """The oracle's codes: per-token Q, one scale for all of K (cache and new
    rows), one for all of V."""
    B, Lq = q.shape[0], q.shape[1]
    f = lambda t: t.float().numpy()
    q8, qs = fp8.quantize_rows(f(q).reshape(B * Lq, -1))
    k8, ks = fp8.quantize_tensor(np.concatenate([f(kc).ravel(), f(kn).ravel()]))
    v8, vs = fp8.quantize_tensor(np.concatenate([f(vc).ravel(), f(vn).ravel()]))
    nc = kc.numel()
    return (q8.reshape(q.shape), qs, k8[nc:].reshape(kn.shape), v8[nc:].reshape(vn.shape),
            k8[:nc].reshape(kc.shape), v8[:nc].reshape(vc.shape), ks, vs)


def random_codes_case(B, Hq, Hkv, Lq, lens, lmax, seed):
    q, kn, vn, kc, vc = synth.make_attn_inputs(B, Hq, Hkv, HD, Lq, max(lens), seed=seed,
                                               lmax=lmax)
    return quantise(q, kn, vn, kc, vc)


def check_reference_bar(got, codes, lens, Hq, Hkv, causal, what):
    want = oracle(*codes, lens, Hq, Hkv, causal)
    moved = oracle(*codes, lens, Hq, Hkv, causal, shift=0.5)
    nrm = np.linalg.norm(want)
    sens = np.linalg.norm(moved - want) / nrm
    sens_max = np.max(np.abs(moved - want))
    rel = np.linalg.norm(got - want) / nrm
    mx = np.max(np.abs(got - want))
    print(f"{what}: rel {rel:.3e} (reference sensitivity {sens:.3e}), max {mx:.3e} "
          f"({sens_max:.3e})")
    assert 0 < sens < 0.1
    assert rel <= 1.5 * sens and mx <= 2.0 * sens_max + 2.0 ** -8 * np.max(np.abs(want)), what


def exact_codes_case(B, Hq, Hkv, Lq, lens, lmax, seed):
    """Codes whose scores are integers in log2 units: each query row-head has
    three nonzero dims of +-1, every key dim is +-1, and the query scale turns
    scale * log2(e) into 1; values are random codes (finite)."""
    rng = np.random.default_rng(seed)
    qv = np.zeros((B, Lq, Hq, HD))
    for b in range(B):
        for i in range(Lq):
            for h in range(Hq):
                dims = rng.choice(HD, size=3, replace=False)
                qv[b, i, h, dims] = rng.choice([-1.0, 1.0], size=3)
    q8 = fp8.encode(qv).reshape(B, Lq, Hq * HD)
    qs = np.full(B * Lq, np.float32(math.sqrt(HD) / math.log2(math.e)), dtype=np.float32)
    kn8 = fp8.encode(rng.choice([-1.0, 1.0], size=(B, Lq, Hkv * HD)))
    kc8 = fp8.encode(rng.choice([-1.0, 1.0], size=(B, Hkv, lmax, HD)))
    vn8 = fp8.encode(rng.normal(size=(B, Lq, Hkv * HD)) * 16)
    vc8 = fp8.encode(rng.normal(size=(B, Hkv, lmax, HD)) * 16)
    return q8, qs, kn8, vn8, kc8, vc8, np.float32(1.0), np.float32(1 / 16)


@pytest.mark.parametrize("B,Hq,Hkv,Lq,lens,causal", [
    (2, 8, 2, 256, [300, 1029], False),   # several tiles, a ragged tail, split keys
    (1, 4, 2, 200, [129], True),          # ragged canvas, causal mask, split keys
    (1, 4, 4, 256, [0], False),           # no prefix
    (2, 32, 8, 456, [300, 1029], False),  # enough CTAs for one key range each
    (2, 32, 8, 456, [129, 0], True),
])
def test_e4m3_attention_exact_probabilities(B, Hq, Hkv, Lq, lens, causal):
    lmax = pad16(max(lens) + 40)
    codes = exact_codes_case(B, Hq, Hkv, Lq, lens, lmax, seed=21)
    got = run_gpu(device_inputs(*codes), lens, max(lens), Hq, Hkv, causal)
    want = oracle(*codes, lens, Hq, Hkv, causal)
    # The roundings left: fp32 sums, the bf16 output (2^-9 of |out|) and, where
    # the key range is split, each split's bf16 partial (2^-9 of its own value,
    # which the probability-weighted mean of |v| bounds).
    q8, qs, kn8, vn8, kc8, vc8, ks, vs = codes
    mean_abs = oracle(q8, qs, kn8, vn8 & 0x7F, kc8, vc8 & 0x7F, ks, vs, lens, Hq, Hkv, causal)
    err = np.abs(got - want)
    bound = 2.0 ** -8 * (np.abs(want) + mean_abs) + 1e-5 * np.max(np.abs(want))
    assert np.all(err <= bound), f"max excess {np.max(err - bound):.3e}"


@pytest.mark.parametrize("B,Hq,Hkv,Lq,lens,causal", [
    (2, 8, 2, 256, [300, 1029], False),
    (2, 4, 2, 200, [77, 0], True),
    (1, 32, 8, 256, [129], False),
])
def test_e4m3_attention_random_inputs(B, Hq, Hkv, Lq, lens, causal):
    lmax = pad16(max(lens) + 40)
    codes = random_codes_case(B, Hq, Hkv, Lq, lens, lmax, seed=5)
    got = run_gpu(device_inputs(*codes), lens, max(lens), Hq, Hkv, causal)
    check_reference_bar(got, codes, lens, Hq, Hkv, causal, f"e4m3 attn B{B} Lq{Lq} L{lens}")


@pytest.mark.parametrize("L", [4096, 32768])
def test_e4m3_attention_microbench_shape_sampled(L):
    """Q [32, 256, 128] over KV [8, L, 128] plus the canvas's 256 keys: rows from
    both query tiles of every head against the oracle."""
    Hq, Hkv, Lq = 32, 8, 256
    codes = random_codes_case(1, Hq, Hkv, Lq, [L], L, seed=7)
    got = run_gpu(device_inputs(*codes), [L], L, Hq, Hkv, False)
    q8, qs, kn8, vn8, kc8, vc8, ks, vs = codes
    rng = np.random.default_rng(L)
    rows = np.concatenate([rng.integers(0, 128, size=3), rng.integers(128, 256, size=3)])
    g_rows, w0, w1 = [], [], []
    mask = np.ones((len(rows), L + Lq), dtype=bool)
    for g in range(Hkv):
        k = np.concatenate([kc8[0, g], kn8[0, :, g * HD:(g + 1) * HD]])
        v = np.concatenate([vc8[0, g], vn8[0, :, g * HD:(g + 1) * HD]])
        for h in range(g * (Hq // Hkv), (g + 1) * (Hq // Hkv)):
            qh = q8[0, rows, h * HD:(h + 1) * HD]
            args = (qh, qs[rows], k, v, ks, vs, mask, 1 / math.sqrt(HD))
            w0.append(fp8.attention_head_e4m3(*args))
            w1.append(fp8.attention_head_e4m3(*args, shift=0.5))
            g_rows.append(got[0, rows, h * HD:(h + 1) * HD])
    got_s, want, moved = (np.stack(a) for a in (g_rows, w0, w1))
    nrm = np.linalg.norm(want)
    sens = np.linalg.norm(moved - want) / nrm
    rel = np.linalg.norm(got_s - want) / nrm
    print(f"L {L}: rel {rel:.3e} (reference sensitivity {sens:.3e})")
    assert 0 < sens < 0.1 and rel <= 1.5 * sens


def test_e4m3_attention_rejects_bad_arguments():
    import canvas_denoising_denoise_b200 as dg
    codes = exact_codes_case(1, 4, 2, 64, [16], 64, seed=1)
    d = device_inputs(*codes)
    lib = dg._lib.load()
    out = torch.zeros((1, 64, 4 * HD), dtype=torch.bfloat16, device="cuda")
    cl = torch.tensor([16], dtype=torch.int32, device="cuda")
    p = lambda t: t.data_ptr()
    base = [p(d["q"]), 4 * HD, p(d["q_scale"]), p(d["k_new"]), 2 * HD, p(d["vt_new"]), 64,
            p(d["k_cache"]), p(d["vt_cache"]), p(d["k_scale"]), p(d["v_scale"]), p(cl), 16, 64,
            p(out), 4 * HD, None, 1, 4, 2, 64, HD, HD ** -0.5, dg.MASK_BIDIR, None, 0, None]
    assert lib.dg_canvas_attn_e4m3(*base) == 0
    torch.cuda.synchronize()
    for idx, val, code in [(21, 64, 2),      # hd 64: DG_ERR_UNSUPPORTED_SHAPE
                           (6, 40, 3),       # ldvt < Lq: DG_ERR_ALIGNMENT
                           (2, None, 1)]:    # no q_scale: DG_ERR_INVALID_ARG
        args = list(base)
        args[idx] = val
        assert lib.dg_canvas_attn_e4m3(*args) == code
