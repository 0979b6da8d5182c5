"""FP8 (e4m3) quantisation and the FP8 unembedding of the oracle.

TEST INFRASTRUCTURE ONLY: only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path.

Format (the OCP 8-bit floating point specification's E4M3): 1 sign bit, 4
exponent bits with bias 7, 3 mantissa bits; normal values (1 + m/8) 2^(e-7)
for e = 1..15 (e = 15 with m = 7 is NaN, so the largest finite value is 448);
subnormal values (m/8) 2^-6 for e = 0.  Encoding rounds to the nearest
representable value, ties to the even code (the even mantissa), and clamps
finite values beyond 448 to 448 (saturating conversion).

Scaling (a reading: the pages quote FP8 checkpoints but fix no recipe):
  per row r of an activation matrix, s_r = max_k |x[r, k]| / 448 (fp32) and
  q[r, k] = e4m3(x[r, k] / s_r) (fp32 division); a weight matrix takes one
  scale for the whole tensor the same way.  An all-zero row takes s = 1.
"""
import numpy as np

MAX = 448.0


def _table():
    """Non-negative finite e4m3 values by code 0..126 (increasing)."""
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


VALUES = _table()


def encode(x):
    """e4m3 codes (uint8) of float values: nearest value, ties to the even code, satfinite."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), MAX)
    hi = np.searchsorted(VALUES, a, side="left")          # first value >= a
    hi = np.clip(hi, 0, len(VALUES) - 1)
    lo = np.clip(hi - 1, 0, len(VALUES) - 1)
    d_lo = a - VALUES[lo]
    d_hi = VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def decode(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    mag = VALUES[np.minimum(codes & 0x7F, 126)]
    return np.where(codes & 0x80, -mag, mag)


def _scale(amax):
    amax = np.float32(amax)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(MAX))


def quantize_rows(x):
    """Per-row e4m3: (codes [R, C] uint8, scales [R] float32)."""
    x = np.asarray(x, dtype=np.float32)
    scales = np.array([_scale(np.max(np.abs(row))) for row in x], dtype=np.float32)
    q = encode((x / scales[:, None]).astype(np.float32))
    return q, scales


def quantize_tensor(x):
    """One e4m3 scale for the whole tensor: (codes, scale float32)."""
    x = np.asarray(x, dtype=np.float32)
    s = _scale(np.max(np.abs(x)))
    return encode((x / s).astype(np.float32)), s


def unembed_logits(h_codes, h_scales, w_codes, w_scale, row_scale=None):
    """Logits of e4m3 operands: rs[t] s_h[t] s_w sum_k dec(h_q[t, k]) dec(w_q[v, k]), fp64
    (every product of two e4m3 values is exact), rounded to fp32 as the GPU keeps them.
    row_scale: the final RMSNorm's per-token scale (None: 1)."""
    acc = decode(h_codes) @ decode(w_codes).T
    s = np.asarray(h_scales, dtype=np.float64) * np.float64(w_scale)
    if row_scale is not None:
        s = s * np.asarray(row_scale, dtype=np.float64)
    return (acc * s[:, None]).astype(np.float32)


def attention_head_e4m3(q_codes, q_scales, k_codes, v_codes, k_scale, v_scale, mask, scale,
                        shift=0.0):
    """FP8 attention of one query head over its keys (a reading: the pages quote FP8
    serving but fix no recipe for attention).

    q_codes [Lq, hd] e4m3 codes with per-row (per-token) scales q_scales [Lq];
    k_codes, v_codes [Lk, hd] codes with one scale each; mask [Lq, Lk] boolean.
      s[i, j] = scale q_scales[i] k_scale sum_d dec(q)[i, d] dec(k)[j, d]
      p[i, j] = exp(s[i, j] - max_j s[i, j])            (masked keys: p = 0)
      out[i]  = v_scale sum_j e4m3(p[i, j]) dec(v)[j] / sum_j p[i, j]
    The probabilities enter the value product as e4m3 values (the operand type of
    an 8-bit product) and the normaliser as exact ones.  They are rounded relative
    to the row maximum (p <= 1); `shift` rounds 2^shift p instead and divides the
    result back, which is how a kernel whose running maximum lags the row's by a
    factor 2^shift rounds them.  An integer shift changes nothing while p stays in
    the normal range (e4m3 rounding commutes with powers of two there).
    """
    qd = decode(q_codes) * np.asarray(q_scales, dtype=np.float64)[:, None]
    kd = decode(k_codes)
    s = (qd @ kd.T) * (np.float64(k_scale) * scale)
    s = np.where(mask, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    p = np.exp(s - m)
    c = 2.0 ** shift
    pq = decode(encode(p * c)) / c
    return np.float64(v_scale) * (pq @ decode(v_codes)) / np.sum(p, axis=1, keepdims=True)


def gqa_attention_e4m3(q_codes, q_scales, kn_codes, vn_codes, kp_codes, vp_codes, k_scale,
                       v_scale, causal, scale, shift=0.0):
    """Grouped-query FP8 attention of one sequence: q_codes [Lq, Hq, hd] with per-token
    scales [Lq]; new rows' codes kn/vn [Lq, Hkv, hd]; cached prefix kp/vp [Hkv, L, hd];
    one K scale and one V scale for prefix and new rows together.  The key set and the
    mask are those of the bf16 attention (the prefix, then the new rows: full for a
    canvas, lower-triangular for a causal pass).  Returns [Lq, Hq, hd] fp64."""
    lq, hq, hd = q_codes.shape
    hkv = kn_codes.shape[1]
    group = hq // hkv
    lp = kp_codes.shape[1]
    pre = np.ones((lq, lp), dtype=bool)
    own = np.tril(np.ones((lq, lq), dtype=bool)) if causal else np.ones((lq, lq), dtype=bool)
    mask = np.concatenate([pre, own], axis=1)
    out = np.empty((lq, hq, hd), dtype=np.float64)
    for h in range(hq):
        g = h // group
        k = np.concatenate([kp_codes[g], kn_codes[:, g, :]], axis=0)
        v = np.concatenate([vp_codes[g], vn_codes[:, g, :]], axis=0)
        out[:, h, :] = attention_head_e4m3(q_codes[:, h, :], q_scales, k, v, k_scale, v_scale,
                                           mask, scale, shift)
    return out
