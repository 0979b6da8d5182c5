"""tcgen05 GEMM (dg_linear, dg_unembed) against the oracle's fp64 matmul and epilogues."""
import numpy as np
import pytest
import torch

from helpers import assert_close, to64
from oracle import model as M

pytestmark = pytest.mark.gpu


def rand_bf16(*shape, scale=1.0, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("Mr,N,K", [(256, 128, 64), (256, 384, 320), (200, 256, 2048),
                                    (64, 512, 256), (1000, 128, 128), (256, 2048, 2048)])
@pytest.mark.parametrize("epi", ["f32", "bf16", "gelu", "resid"])
def test_linear_epilogues(Mr, N, K, epi):
    import canvas_denoising_denoise_b200 as dg
    x = rand_bf16(Mr, K, seed=1)
    w = rand_bf16(N, K, scale=K ** -0.5, seed=2)
    ref = to64(x) @ to64(w).T
    xd, wd = x.cuda(), w.cuda()
    if epi == "f32":
        out = torch.empty((Mr, N), dtype=torch.float32, device="cuda")
        dg.linear(xd, wd, out, dg.EPI_F32)
        want = ref
    elif epi == "bf16":
        out = torch.empty((Mr, N), dtype=torch.bfloat16, device="cuda")
        dg.linear(xd, wd, out, dg.EPI_BF16)
        want = ref
    elif epi == "gelu":
        out = torch.empty((Mr, N), dtype=torch.bfloat16, device="cuda")
        dg.linear(xd, wd, out, dg.EPI_GELU_BF16)
        want = M.gelu(ref)
    else:
        base = torch.randn((Mr, N), generator=torch.Generator().manual_seed(3))
        out = base.clone().cuda()
        dg.linear(xd, wd, out, dg.EPI_RESID_F32)
        want = to64(base) + ref
    torch.cuda.synchronize()
    dg.check_device_errors()
    assert_close(out, want, rel_l2=5e-3, max_abs=3e-2, what=f"{epi} {Mr}x{N}x{K}")


# V % 256 == 0 runs on CTA pairs (256 x 256 tiles, persistent, double-buffered
# accumulators); V = 384 on the single-CTA GEMM.  600 and 1024 rows span
# several token tiles (600 with a ragged one); V = 65536 gives each pair
# several tiles, so both accumulator buffers are reused.
@pytest.mark.parametrize("Mr,d,V", [(256, 256, 512), (256, 2048, 4096), (131, 512, 1024),
                                    (256, 256, 384), (600, 512, 2048), (1024, 256, 8192),
                                    (256, 512, 65536), (1, 64, 256)])
def test_unembed_against_oracle(Mr, d, V):
    import canvas_denoising_denoise_b200 as dg
    h = rand_bf16(Mr, d, seed=4)
    w = rand_bf16(V, d, scale=0.02, seed=5)
    logits = torch.empty((Mr, V), dtype=torch.float32, device="cuda")
    dg.unembed(h.cuda(), w.cuda(), logits)
    torch.cuda.synchronize()
    assert_close(logits, to64(h) @ to64(w).T, rel_l2=1e-5, max_abs=1e-4, what="unembed")


def test_unembed_full_vocab_sampled_rows():
    """Full-size unembedding (M = 256, d = 2048, V = 262144) checked on sampled outputs."""
    import canvas_denoising_denoise_b200 as dg
    Mr, d, V = 256, 2048, 262144
    h = rand_bf16(Mr, d, seed=6).cuda()
    w = rand_bf16(V, d, scale=0.02, seed=7).cuda()
    logits = torch.empty((Mr, V), dtype=torch.float32, device="cuda")
    dg.unembed(h, w, logits)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = rng.integers(0, Mr, size=16)
    cols = rng.integers(0, V, size=512)
    hs = to64(h[rows].cpu())
    ws = to64(w[cols].cpu())
    got = logits[rows][:, cols].cpu()
    assert_close(got, hs @ ws.T, rel_l2=1e-5, max_abs=1e-4, what="unembed full")
    # determinism: a second run gives identical bits
    again = torch.empty_like(logits)
    dg.unembed(h, w, again)
    torch.cuda.synchronize()
    assert torch.equal(again, logits)


def test_gelu_epilogue_matches_exact_gelu_to_the_bf16_step():
    """Identity weights make the accumulator equal the input, so each output is
    bf16(gelu(x)) of one bf16 x; the epilogue's erf (Abramowitz & Stegun 7.1.26,
    error <= 1.5e-7) must give the bf16 rounding of the exact GELU except within
    a hair of a rounding boundary, and never more than one bf16 step away."""
    import canvas_denoising_denoise_b200 as dg
    n = 128
    g = torch.Generator().manual_seed(8)
    x = (torch.rand((1024, n), generator=g) * 12 - 6).to(torch.bfloat16)
    w = torch.eye(n, dtype=torch.bfloat16)
    out = torch.empty((1024, n), dtype=torch.bfloat16, device="cuda")
    dg.linear(x.cuda(), w.cuda(), out, dg.EPI_GELU_BF16)
    torch.cuda.synchronize()
    exact = M.gelu(to64(x))                        # fp64, exact erf
    want = torch.from_numpy(exact).to(torch.bfloat16)
    got = out.cpu()
    diff = got != want
    # a mismatch is allowed only where the exact value lies within the erf
    # error (plus fp32 rounding) of the midpoint between want and its bf16
    # neighbour on the side of the exact value, and only by that one step
    ex = torch.from_numpy(exact)
    wi = want.view(torch.int16).int()
    away = ex.abs() > want.double().abs()            # exact beyond want in magnitude
    nb = (wi + torch.where(away, 1, -1)).short().view(torch.bfloat16)
    mid = (want.double() + nb.double()) / 2
    near = (ex - mid).abs() <= 1e-6 + 1e-6 * ex.abs()
    assert not (diff & ~near).any(), int((diff & ~near).sum())
    assert torch.equal(got[diff], nb[diff])
    # where the output is not tiny the absolute error is a negligible fraction
    # of the bf16 step, so mismatches (midpoint cases) must be rare
    big = ex.abs() >= 1e-2
    assert int((diff & big).sum()) <= 0.01 * int(big.sum())


def quant_gpu(t, per_row):
    import canvas_denoising_denoise_b200 as dg
    q = torch.empty(t.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(t.shape[0] if per_row else 1, dtype=torch.float32, device="cuda")
    dg.quantize_e4m3(t.cuda(), q, s, per_row=per_row)
    return q, s


# e4m3 operands (128-element k-blocks): K = 128 is one k-block; 8192 splits
# over a cluster of four; 200 and 1000 rows leave ragged token tiles.
@pytest.mark.parametrize("Mr,N,K", [(256, 128, 128), (256, 384, 384), (200, 256, 2048),
                                    (64, 512, 256), (1000, 128, 128), (256, 2048, 2048),
                                    (256, 2048, 8192)])
@pytest.mark.parametrize("epi", ["f32", "bf16", "gelu", "resid"])
def test_linear_e4m3_epilogues(Mr, N, K, epi):
    """Against the oracle's product of the same codes (exact e4m3 products in fp64)."""
    import canvas_denoising_denoise_b200 as dg
    from oracle import fp8
    x = rand_bf16(Mr, K, seed=1)
    w = rand_bf16(N, K, scale=K ** -0.5, seed=2)
    xq, xs = quant_gpu(x, True)
    wq, ws = quant_gpu(w, False)
    torch.cuda.synchronize()
    acc = (fp8.decode(xq.cpu().numpy()) @ fp8.decode(wq.cpu().numpy()).T) * (
        xs.cpu().numpy().astype(np.float64)[:, None] * np.float64(ws.cpu().numpy()[0]))
    tight = dict(rel_l2=1e-5, max_abs=1e-4)
    if epi == "f32":
        out = torch.empty((Mr, N), dtype=torch.float32, device="cuda")
        dg.linear_e4m3(xq, xs, wq, ws, out, dg.EPI_F32)
        want, tol = acc, tight
    elif epi == "bf16":
        out = torch.empty((Mr, N), dtype=torch.bfloat16, device="cuda")
        dg.linear_e4m3(xq, xs, wq, ws, out, dg.EPI_BF16)
        want, tol = acc, {}
    elif epi == "gelu":
        out = torch.empty((Mr, N), dtype=torch.bfloat16, device="cuda")
        dg.linear_e4m3(xq, xs, wq, ws, out, dg.EPI_GELU_BF16)
        want, tol = M.gelu(acc), {}
    else:
        base = torch.randn((Mr, N), generator=torch.Generator().manual_seed(3))
        out = base.clone().cuda()
        dg.linear_e4m3(xq, xs, wq, ws, out, dg.EPI_RESID_F32)
        want, tol = to64(base) + acc, tight
    torch.cuda.synchronize()
    dg.check_device_errors()
    assert_close(out, want, what=f"e4m3 {epi} {Mr}x{N}x{K}", **tol)


# Many tokens: the projections run on the persistent CTA-pair pipeline
# (256 x 256 tiles: at least one full wave of pairs, or 48 and more tiles with
# 1536 and more tokens, as 1600 x 2048 has: 56 tiles, some pairs idle); 1300
# and 1600 rows leave a ragged token tile; K = 128 / 256 are one or two e4m3
# k-blocks per stage.
@pytest.mark.parametrize("Mr,N,K", [(1024, 8192, 2048), (4096, 2048, 2048), (1300, 8192, 512),
                                    (2048, 4096, 768), (1600, 2048, 512)])
@pytest.mark.parametrize("epi", ["f32", "bf16", "gelu", "resid"])
def test_linear_many_tokens_pair_path(Mr, N, K, epi):
    test_linear_epilogues(Mr, N, K, epi)


@pytest.mark.parametrize("Mr,N,K", [(1024, 8192, 2048), (1300, 8192, 512), (4096, 2048, 384),
                                    (1600, 2048, 512)])
@pytest.mark.parametrize("epi", ["f32", "bf16", "resid"])
def test_linear_e4m3_many_tokens_pair_path(Mr, N, K, epi):
    test_linear_e4m3_epilogues(Mr, N, K, epi)
