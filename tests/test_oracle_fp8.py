"""Pins of the oracle's e4m3 quantiser against the format's definition and
against PyTorch's float8_e4m3fn conversion (a library routine)."""
import numpy as np
import torch

from oracle import fp8


def torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_value_table_closed_forms():
    v = fp8.VALUES
    assert v[0] == 0.0 and v[1] == 2.0 ** -9          # smallest subnormal
    assert v[8] == 2.0 ** -6                          # smallest normal
    assert v[126] == 448.0                            # largest finite
    assert v[56] == 1.0 and v[57] == 1.125            # step 1/8 in [1, 2)
    assert np.all(np.diff(v) > 0)


def test_every_code_round_trips():
    codes = np.concatenate([np.arange(127), np.arange(128, 255)]).astype(np.uint8)
    assert np.array_equal(fp8.encode(fp8.decode(codes)), codes)


def test_ties_go_to_the_even_code():
    # 1.0625 lies halfway between 1.0 (code 56) and 1.125 (57): even -> 56;
    # 1.1875 between 1.125 (57) and 1.25 (58): even -> 58; 2^-10 between 0 and 2^-9: -> 0
    assert fp8.encode([1.0625, 1.1875, 2.0 ** -10]).tolist() == [56, 58, 0]
    assert fp8.encode([464.0, 1000.0, -1000.0]).tolist() == [126, 126, 254]  # satfinite


def test_matches_torch_conversion_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(scale=0.01, size=20000),
                        rng.normal(scale=1.0, size=20000)]).astype(np.float32)
    assert np.array_equal(fp8.encode(x), torch_e4m3(x))


def test_quantize_rows_scales_and_error():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(8, 256)).astype(np.float32)
    x[3] = 0.0
    q, s = fp8.quantize_rows(x)
    assert s.dtype == np.float32 and s[3] == 1.0
    amax = np.max(np.abs(x), axis=1)
    assert np.allclose(s[np.arange(8) != 3], amax[np.arange(8) != 3] / 448, rtol=1e-6)
    back = fp8.decode(q) * s[:, None]
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normal values
    big = np.abs(x) >= s[:, None] * 2.0 ** -6
    assert np.all(np.abs(back - x)[big] <= np.abs(x)[big] * 2.0 ** -4 + 1e-12)
    assert np.all(np.max(np.abs(fp8.decode(q)), axis=1)[np.arange(8) != 3] == 448.0)


def test_unembed_logits_equal_the_dequantised_product():
    rng = np.random.default_rng(2)
    h = rng.normal(size=(5, 64)).astype(np.float32)
    w = (rng.normal(size=(32, 64)) * 0.02).astype(np.float32)
    hq, hs = fp8.quantize_rows(h)
    wq, ws = fp8.quantize_tensor(w)
    got = fp8.unembed_logits(hq, hs, wq, ws)
    want = (fp8.decode(hq) * hs[:, None].astype(np.float64)) @ (fp8.decode(wq) * np.float64(ws)).T
    assert np.allclose(got, want, rtol=1e-6, atol=1e-7)
    # and close to the unquantised product (3 mantissa bits on each side)
    assert np.linalg.norm(got - h @ w.T) <= 0.08 * np.linalg.norm(h @ w.T)


def test_unembed_e4m3_one_hot_hidden_state():
    """hn = c e_j: its codes are 448 at j (scale c/448), so logit v is exactly c times
    the e4m3-rounded w[v, j] (the weight's own scale times its decoded code)."""
    from oracle import model as M
    rng = np.random.default_rng(3)
    w = rng.normal(scale=0.05, size=(64, 32))
    c, j = 1.5, 7
    hn = np.zeros((1, 32))
    hn[0, j] = c
    wq, ws = fp8.quantize_tensor(w)
    q_w = np.float64(ws) * fp8.decode(wq)
    got = M.unembed_e4m3(hn, w)
    np.testing.assert_array_equal(got[0], (c * q_w[:, j]).astype(np.float32))
    # a transposed or mis-scaled operand breaks it
    assert not np.allclose(got[0], c * w[:, j] * 2)


def test_unembed_e4m3_within_the_format_error_bound():
    """Each e4m3 operand of a normal-range value carries a relative error of at most
    2^-4 (half a step of a 3-bit mantissa); below 2^-6 scale units the error is at
    most 2^-10 absolute.  So |fp8 - exact| <= sum_k (2^-4 + 2^-4 + 2^-8) |h_k w_k| plus
    the subnormal slack, and the error is not zero (the path does quantise)."""
    from oracle import model as M
    rng = np.random.default_rng(4)
    h = rng.normal(size=(16, 128))
    w = rng.normal(scale=0.02, size=(96, 128))
    got = M.unembed_e4m3(h, w)
    exact = h @ w.T
    hs = np.abs(h).max(axis=1) / 448.0
    ws = np.abs(w).max() / 448.0
    rel = 2.0 ** -4 * 2 + 2.0 ** -8
    sub = 2.0 ** -10 * (hs[:, None] * (np.abs(w).sum(axis=1)[None, :])
                        + ws * np.abs(h).sum(axis=1)[:, None])
    bound = rel * (np.abs(h) @ np.abs(w).T) + sub + 1e-6 * np.abs(exact)
    assert np.all(np.abs(got - exact) <= bound)
    assert np.abs(got - exact).max() > 0


# ---------------------------------------------------------------- FP8 attention

def _codes(vals):
    return fp8.encode(np.asarray(vals, dtype=np.float64))


def test_attention_e4m3_two_keys_closed_form():
    # scores (ln(1/0.3), 0): p = (1, 0.3); e4m3(0.3) = 1.25 * 2^-2 = 0.3125 enters
    # the value sum, the exact 0.3 the normaliser
    q = _codes([[1.0]])
    k = _codes([[1.0], [0.0]])
    v = _codes([[2.0], [-4.0]])
    mask = np.ones((1, 2), dtype=bool)
    out = fp8.attention_head_e4m3(q, [1.0], k, v, 1.0, 0.5, mask, -np.log(0.3))
    assert np.isclose(out[0, 0], 0.5 * (2.0 - 4.0 * 0.3125) / 1.3, rtol=1e-12, atol=0)


def test_attention_e4m3_exact_probabilities_match_sdpa():
    # integer dot products times ln 2: every probability is a power of two no
    # smaller than 2^-6 (a normal e4m3 value), so only the dequantisation is left
    # and the result is softmax attention of the decoded values (library routine)
    rng = np.random.default_rng(3)
    lq, lp, hq, hkv, hd = 6, 9, 4, 2, 16
    qv = np.zeros((lq, hq, hd))
    for i in range(lq):
        for h in range(hq):
            dims = rng.choice(hd, size=3, replace=False)
            qv[i, h, dims] = rng.choice([-1.0, 1.0], size=3)
    kn = rng.choice([-1.0, 1.0], size=(lq, hkv, hd))
    kp = rng.choice([-1.0, 1.0], size=(hkv, lp, hd))
    vn = rng.normal(size=(lq, hkv, hd))
    vp = rng.normal(size=(hkv, lp, hd))
    qc = _codes(qv)                                     # codes of +-1 and 0
    vnc, vpc = _codes(vn * 16), _codes(vp * 16)
    for causal in (False, True):
        got = fp8.gqa_attention_e4m3(qc, np.ones(lq), _codes(kn), vnc, _codes(kp), vpc,
                                     1.0, 1.0 / 16, causal, np.log(2.0))
        mask = np.concatenate([np.ones((lq, lp), dtype=bool),
                               np.tril(np.ones((lq, lq), dtype=bool)) if causal
                               else np.ones((lq, lq), dtype=bool)], axis=1)
        for h in range(hq):
            g = h // (hq // hkv)
            k = torch.from_numpy(np.concatenate([kp[g], kn[:, g]], axis=0))
            v = torch.from_numpy(fp8.decode(np.concatenate([vpc[g], vnc[:, g]], axis=0)) / 16)
            want = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qv[:, h])[None], k[None], v[None],
                attn_mask=torch.from_numpy(mask)[None], scale=float(np.log(2.0)))[0].numpy()
            assert np.allclose(got[:, h], want, rtol=1e-12, atol=1e-14), (causal, h)


def test_attention_e4m3_integer_reference_shift_changes_nothing_in_the_normal_range():
    rng = np.random.default_rng(4)
    q = _codes(rng.normal(size=(8, 32)))
    k = _codes(rng.normal(size=(40, 32)))
    v = _codes(rng.normal(size=(40, 32)))
    qs = np.full(8, 0.05)
    mask = np.ones((8, 40), dtype=bool)
    # small scores: every p lies in [2^-5, 1], well inside the normal range
    base = fp8.attention_head_e4m3(q, qs, k, v, 1.0, 1.0, mask, 0.3)
    s = (fp8.decode(q) * qs[:, None]) @ fp8.decode(k).T * 0.3
    assert np.min(np.exp(s - s.max(axis=1, keepdims=True))) > 2.0 ** -5
    for c in (1, 3, 8):
        assert np.array_equal(fp8.attention_head_e4m3(q, qs, k, v, 1.0, 1.0, mask, 0.3, c), base)
    moved = fp8.attention_head_e4m3(q, qs, k, v, 1.0, 1.0, mask, 0.3, 0.5)
    assert not np.array_equal(moved, base)


def test_attention_e4m3_within_the_rounding_bound_of_exact_attention():
    # the only rounding after dequantisation is e4m3(p): relative 2^-4 for normal
    # values, absolute 2^-10 below 2^-6
    rng = np.random.default_rng(5)
    lq, lk, hd = 16, 300, 64
    q = _codes(rng.normal(size=(lq, hd)) * 20)
    qs = rng.uniform(0.02, 0.06, lq)
    k = _codes(rng.normal(size=(lk, hd)) * 20)
    v = _codes(rng.normal(size=(lk, hd)) * 20)
    mask = np.ones((lq, lk), dtype=bool)
    mask[3, 100:] = False
    got = fp8.attention_head_e4m3(q, qs, k, v, 0.05, 0.05, mask, 1 / np.sqrt(hd))
    qd = fp8.decode(q) * qs[:, None]
    s = (qd @ fp8.decode(k).T) * 0.05 / np.sqrt(hd)
    s = np.where(mask, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    vd = fp8.decode(v) * 0.05
    exact = (p @ vd) / p.sum(axis=1, keepdims=True)
    bound = ((np.maximum(p * 2.0 ** -4, 2.0 ** -10)) @ np.abs(vd)) / p.sum(axis=1, keepdims=True)
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-9))
    assert np.max(np.abs(got - exact)) > 0                # the rounding is there
