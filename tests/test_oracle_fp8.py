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
