"""Pins of the oracle's model half against library routines, closed forms and invariants."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import model as M

TINY = M.ModelCfg(d=64, n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=16, ffn=128, vocab=96)


def rand_weights(cfg, seed=0, std=0.05):
    rng = np.random.default_rng(seed)
    hq, hkv, hd, d, f, v = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.d, cfg.ffn, cfg.vocab
    w = {"embed": rng.normal(scale=std, size=(v, d)) * 20, "unembed": rng.normal(scale=std, size=(v, d)),
         "layers": []}
    for _ in range(cfg.n_layers):
        w["layers"].append({"w_qkv": rng.normal(scale=std * 3, size=((hq + 2 * hkv) * hd, d)),
                            "w_o": rng.normal(scale=std, size=(d, hq * hd)),
                            "w_up": rng.normal(scale=std, size=(f, d)),
                            "w_down": rng.normal(scale=std, size=(d, f))})
    return w


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(scale=3.0, size=(7, 33))
    y = M.rmsnorm(x, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-12)
    assert np.allclose(M.rmsnorm(5.0 * x, 0.0), y, atol=1e-12)
    # against the library routine (unit weight)
    t = F.rms_norm(torch.from_numpy(x), (33,), eps=1e-6).numpy()
    assert np.allclose(M.rmsnorm(x, 1e-6), t, atol=1e-12)


def test_gelu_against_library_and_limits():
    x = np.linspace(-8, 8, 1001)
    assert np.allclose(M.gelu(x), F.gelu(torch.from_numpy(x)).numpy(), atol=1e-14)
    assert M.gelu(np.array([0.0]))[0] == 0.0
    assert M.gelu(np.array([30.0]))[0] == pytest.approx(30.0)
    assert abs(M.gelu(np.array([-30.0]))[0]) < 1e-100


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.normal(scale=10, size=10000).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(M.round_bf16(x), want.astype(np.float64))


def _sdpa(q, k, v, mask=None, causal=False):
    # q [H, Lq, hd]
    return F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                          torch.from_numpy(v)[None], attn_mask=mask,
                                          is_causal=causal)[0].numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_attention_no_prefix_reduces_to_sdpa(causal):
    rng = np.random.default_rng(2)
    lq, hq, hkv, hd = 24, 4, 4, 8
    q = rng.normal(size=(lq, hq, hd))
    k = rng.normal(size=(lq, hkv, hd))
    v = rng.normal(size=(lq, hkv, hd))
    empty = np.zeros((hkv, 0, hd))
    o = M.gqa_attention(q, k, v, empty, empty, causal, 1 / math.sqrt(hd))
    want = _sdpa(q.transpose(1, 0, 2), k.transpose(1, 0, 2), v.transpose(1, 0, 2), causal=causal)
    assert np.allclose(o, want.transpose(1, 0, 2), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_with_prefix_and_gqa_against_sdpa(causal):
    rng = np.random.default_rng(3)
    lq, L, hq, hkv, hd = 10, 13, 6, 2, 8
    q = rng.normal(size=(lq, hq, hd))
    kn = rng.normal(size=(lq, hkv, hd))
    vn = rng.normal(size=(lq, hkv, hd))
    kp = rng.normal(size=(hkv, L, hd))
    vp = rng.normal(size=(hkv, L, hd))
    o = M.gqa_attention(q, kn, vn, kp, vp, causal, 1 / math.sqrt(hd))
    kfull = np.concatenate([kp, kn.transpose(1, 0, 2)], axis=1)
    vfull = np.concatenate([vp, vn.transpose(1, 0, 2)], axis=1)
    group = hq // hkv
    kfull = np.repeat(kfull, group, axis=0)
    vfull = np.repeat(vfull, group, axis=0)
    mask = torch.ones(lq, L + lq, dtype=torch.bool)
    if causal:
        mask[:, L:] = torch.tril(torch.ones(lq, lq, dtype=torch.bool))
    want = _sdpa(q.transpose(1, 0, 2), kfull, vfull, mask=mask)
    assert np.allclose(o, want.transpose(1, 0, 2), atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(4)
    hd = 8
    q = rng.normal(size=(5, hd))
    v = rng.normal(size=(1, hd))
    k = rng.normal(size=(1, hd))
    mask = np.ones((5, 1), dtype=bool)
    assert np.allclose(M.attention_head(q, k, v, mask, 0.3), np.repeat(v, 5, axis=0))
    k = np.repeat(rng.normal(size=(1, hd)), 7, axis=0)
    v = rng.normal(size=(7, hd))
    mask = np.ones((5, 7), dtype=bool)
    assert np.allclose(M.attention_head(q, k, v, mask, 0.3), np.repeat(v.mean(0, keepdims=True), 5, 0))


def test_canvas_attention_permutation_equivariant():
    rng = np.random.default_rng(5)
    lq, L, hq, hkv, hd = 12, 9, 4, 2, 8
    q = rng.normal(size=(lq, hq, hd))
    kn = rng.normal(size=(lq, hkv, hd))
    vn = rng.normal(size=(lq, hkv, hd))
    kp = rng.normal(size=(hkv, L, hd))
    vp = rng.normal(size=(hkv, L, hd))
    perm = rng.permutation(lq)
    o = M.gqa_attention(q, kn, vn, kp, vp, False, 0.25)
    op = M.gqa_attention(q[perm], kn[perm], vn[perm], kp, vp, False, 0.25)
    assert np.allclose(op, o[perm], atol=1e-12)
    # the causal pass is not equivariant (sanity of the mask)
    oc = M.gqa_attention(q, kn, vn, kp, vp, True, 0.25)
    ocp = M.gqa_attention(q[perm], kn[perm], vn[perm], kp, vp, True, 0.25)
    assert not np.allclose(ocp, oc[perm])


@pytest.mark.parametrize("bf16", [False, True])
def test_denoise_forward_permutation_equivariant(bf16):
    w = rand_weights(TINY)
    kc, vc = M.empty_cache(TINY, 40)
    rng = np.random.default_rng(6)
    prompt = rng.integers(0, TINY.vocab, size=8)
    L = M.prefill(TINY, w, prompt, kc, vc, bf16)
    canvas = rng.integers(0, TINY.vocab, size=16)
    perm = rng.permutation(16)
    lg = M.denoise_logits(TINY, w, canvas, kc, vc, L, bf16)
    lgp = M.denoise_logits(TINY, w, canvas[perm], kc, vc, L, bf16)
    assert np.allclose(lgp, lg[perm], atol=1e-9)


def test_block_commit_equals_one_shot_prefill():
    w = rand_weights(TINY, seed=11)
    rng = np.random.default_rng(7)
    prompt = rng.integers(0, TINY.vocab, size=8)
    blocks = [rng.integers(0, TINY.vocab, size=16) for _ in range(2)]
    kc, vc = M.empty_cache(TINY, 40)
    L = M.prefill(TINY, w, prompt, kc, vc, bf16_storage=False)
    for blk in blocks:
        L = M.block_commit(TINY, w, blk, kc, vc, L, bf16_storage=False)
    kc2, vc2 = M.empty_cache(TINY, 40)
    L2 = M.prefill(TINY, w, np.concatenate([prompt] + blocks), kc2, vc2, bf16_storage=False)
    assert L == L2 == 40
    for l in range(TINY.n_layers):
        assert np.allclose(kc[l], kc2[l], atol=1e-12) and np.allclose(vc[l], vc2[l], atol=1e-12)


def test_zero_projections_make_the_layer_an_identity():
    w = rand_weights(TINY)
    lw = dict(w["layers"][0])
    lw["w_o"] = np.zeros_like(lw["w_o"])
    lw["w_down"] = np.zeros_like(lw["w_down"])
    rng = np.random.default_rng(8)
    x = rng.normal(size=(5, TINY.d))
    empty = np.zeros((TINY.n_kv_heads, 0, TINY.head_dim))
    out, k, v = M.layer_forward(TINY, lw, x, empty, empty, False, bf16_storage=False)
    assert np.array_equal(out, x)
    # and K/V are the projections of the normalised input
    xn = M.rmsnorm(x, TINY.eps)
    qkv = xn @ lw["w_qkv"].T
    hq, hkv, hd = TINY.n_q_heads, TINY.n_kv_heads, TINY.head_dim
    assert np.allclose(k.reshape(5, -1), qkv[:, hq * hd:(hq + hkv) * hd])


def test_single_layer_against_torch_composition():
    """One layer equals the same pre-norm block assembled from torch library ops."""
    w = rand_weights(TINY, seed=3)
    lw = w["layers"][0]
    rng = np.random.default_rng(9)
    lq, L = 6, 5
    x = rng.normal(size=(lq, TINY.d))
    hq, hkv, hd = TINY.n_q_heads, TINY.n_kv_heads, TINY.head_dim
    kp = rng.normal(size=(hkv, L, hd))
    vp = rng.normal(size=(hkv, L, hd))
    out, _, _ = M.layer_forward(TINY, lw, x, kp, vp, False, bf16_storage=False)

    tx = torch.from_numpy(x)
    t = {k: torch.from_numpy(v) for k, v in lw.items()}
    xn = F.rms_norm(tx, (TINY.d,), eps=TINY.eps)
    qkv = F.linear(xn, t["w_qkv"])
    q = qkv[:, :hq * hd].view(lq, hq, hd).transpose(0, 1)
    k = qkv[:, hq * hd:(hq + hkv) * hd].view(lq, hkv, hd).transpose(0, 1)
    v = qkv[:, (hq + hkv) * hd:].view(lq, hkv, hd).transpose(0, 1)
    k = torch.cat([torch.from_numpy(kp), k], 1).repeat_interleave(hq // hkv, 0)
    v = torch.cat([torch.from_numpy(vp), v], 1).repeat_interleave(hq // hkv, 0)
    o = F.scaled_dot_product_attention(q[None], k[None], v[None])[0].transpose(0, 1).reshape(lq, -1)
    h = tx + F.linear(o, t["w_o"])
    y = h + F.linear(F.gelu(F.linear(F.rms_norm(h, (TINY.d,), eps=TINY.eps), t["w_up"])), t["w_down"])
    assert np.allclose(out, y.numpy(), atol=1e-10)


def test_bf16_storage_close_to_fp64():
    w = rand_weights(TINY, seed=5)
    rng = np.random.default_rng(10)
    prompt = rng.integers(0, TINY.vocab, size=8)
    canvas = rng.integers(0, TINY.vocab, size=16)
    out = []
    for bf16 in (False, True):
        kc, vc = M.empty_cache(TINY, 24)
        L = M.prefill(TINY, w, prompt, kc, vc, bf16)
        out.append(M.denoise_logits(TINY, w, canvas, kc, vc, L, bf16))
    rel = np.linalg.norm(out[0] - out[1]) / np.linalg.norm(out[0])
    assert 0 < rel < 2e-2


def test_e4m3_linear_exact_on_representable_operands():
    """Rows of a that are e4m3 values times 2^j with one entry at +-448 * 2^j, and a
    weight of e4m3 values times 2^-5 with one entry at 448 * 2^-5, quantise exactly
    (scale = amax / 448 is the power of two), so the FP8 product is the exact product."""
    from oracle import fp8
    rng = np.random.default_rng(12)
    finite = np.concatenate([np.arange(0, 127), np.arange(128, 255)]).astype(np.uint8)
    a = fp8.decode(rng.choice(finite, size=(7, 48)))
    a[:, 5] = 448.0 * np.where(rng.random(7) < 0.5, 1, -1)
    a = a * (2.0 ** rng.integers(-6, 6, size=(7, 1)))
    w = fp8.decode(rng.choice(finite, size=(24, 48)))
    w[3, 9] = 448.0
    w = w * 2.0 ** -5
    got = M.linear_e4m3(a, w)
    assert np.array_equal(got, a @ w.T)
    assert not np.allclose(got, a @ w[::-1].T)


def test_e4m3_layers_zero_projections_identity_and_equivariance():
    w = rand_weights(TINY, seed=13)
    lw = dict(w["layers"][0])
    lw["w_o"] = np.zeros_like(lw["w_o"])
    lw["w_down"] = np.zeros_like(lw["w_down"])
    rng = np.random.default_rng(14)
    x = rng.normal(size=(5, TINY.d))
    empty = np.zeros((TINY.n_kv_heads, 0, TINY.head_dim))
    out, _, _ = M.layer_forward(TINY, lw, x, empty, empty, False, bf16_storage=True, e4m3=True)
    assert np.array_equal(out, x)
    # per-token activation scales and one weight scale keep the canvas pass
    # permutation-equivariant
    kc, vc = M.empty_cache(TINY, 40)
    prompt = rng.integers(0, TINY.vocab, size=8)
    L = M.prefill(TINY, w, prompt, kc, vc, e4m3_layers=True)
    canvas = rng.integers(0, TINY.vocab, size=16)
    perm = rng.permutation(16)
    lg = M.denoise_logits(TINY, w, canvas, kc, vc, L, e4m3_layers=True)
    lgp = M.denoise_logits(TINY, w, canvas[perm], kc, vc, L, e4m3_layers=True)
    assert np.allclose(lgp, lg[perm], atol=1e-9)


def test_e4m3_layers_close_to_bf16_forward():
    """FP8 projections move the logits by the format's rounding (a few percent),
    not more, and not zero."""
    w = rand_weights(TINY, seed=15)
    rng = np.random.default_rng(16)
    prompt = rng.integers(0, TINY.vocab, size=8)
    canvas = rng.integers(0, TINY.vocab, size=16)
    out = []
    for e4m3 in (False, True):
        kc, vc = M.empty_cache(TINY, 24)
        L = M.prefill(TINY, w, prompt, kc, vc, e4m3_layers=e4m3)
        out.append(M.denoise_logits(TINY, w, canvas, kc, vc, L, e4m3_layers=e4m3))
    rel = np.linalg.norm(out[0] - out[1]) / np.linalg.norm(out[0])
    assert 1e-3 < rel < 0.1


@pytest.mark.parametrize("e4m3", [False, True])
def test_logit_rows_select_rows_of_the_full_unembedding(e4m3):
    """denoise_logits(rows=r) is the r-th rows of the full result, bit for bit
    (the selection happens after every row of the stack is computed)."""
    w = rand_weights(TINY, seed=4)
    kc, vc = M.empty_cache(TINY, 40)
    L = M.prefill(TINY, w, np.arange(8) % TINY.vocab, kc, vc)
    canvas = np.random.default_rng(2).integers(0, TINY.vocab, size=24)
    full = M.denoise_logits(TINY, w, canvas, kc, vc, L, e4m3_unembed=e4m3)
    rows = [17, 0, 5, 23]
    part = M.denoise_logits(TINY, w, canvas, kc, vc, L, e4m3_unembed=e4m3, rows=rows)
    if e4m3:
        # per-token scales: each row's codes and scale depend on that row only
        assert np.array_equal(part, full[rows])
    else:
        np.testing.assert_allclose(part, full[rows], rtol=1e-13, atol=1e-15)
