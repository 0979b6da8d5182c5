"""Argument checking of the C ABI, on the host: every entry point rejects bad
arguments with its documented status before it touches device memory, so
these run without a GPU (the pointers below are never dereferenced).  Also
the workspace-size queries and the sampler defaults against the pages'
settings."""
import ctypes
import os

import pytest

from conftest import ROOT

OK, INVALID, SHAPE, ALIGN, WS = 0, 1, 2, 3, 4
P = ctypes.c_void_p(0x100000)       # a 16-byte aligned stand-in for a device pointer
MIS = ctypes.c_void_p(0x100008)     # 8-byte aligned only
NULL = None


@pytest.fixture(scope="module")
def lib():
    from canvas_denoising_denoise_b200 import _lib
    return _lib.load()


@pytest.fixture(scope="module")
def L():
    from canvas_denoising_denoise_b200 import _lib
    return _lib


def settings():
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", "sampler_settings.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()[:2]
                out[k] = float(v)
    return out


def defaults(lib, L):
    c = L.SamplerCfg()
    lib.dg_sampler_defaults(ctypes.byref(c))
    return c


def test_sampler_defaults_are_the_pages_settings(lib, L):
    c, g = defaults(lib, L), settings()
    assert c.max_steps == g["max_steps"]
    assert c.t_start == pytest.approx(g["t_start"]) and c.t_end == pytest.approx(g["t_end"])
    assert c.stop_entropy == pytest.approx(g["stop_entropy"])
    assert c.entropy_bound == pytest.approx(g["select_entropy"])
    assert g["commit_min"] <= c.commit_k <= g["commit_max"]
    assert c.selection == 0 and c.unselected_policy == 0


def test_unembed_rejects_bad_arguments(lib):
    assert lib.dg_unembed(NULL, P, P, 256, 2048, 262144, None, 0, None) == INVALID
    assert lib.dg_unembed(P, P, P, 256, 2048, 1000, None, 0, None) == SHAPE       # V % 128
    assert lib.dg_unembed(P, P, P, 256, 100, 262144, None, 0, None) == SHAPE      # d % 64
    assert lib.dg_unembed(MIS, P, P, 256, 2048, 262144, None, 0, None) == ALIGN
    assert lib.dg_unembed(P, P, P, 0, 2048, 262144, None, 0, None) != OK


def test_linear_rejects_bad_arguments(lib):
    assert lib.dg_linear(P, P, P, 256, 2048, 2048, 7, None, 0, None) == INVALID   # epilogue
    assert lib.dg_linear(P, P, P, 256, 200, 2048, 1, None, 0, None) == SHAPE      # N % 128
    assert lib.dg_linear(P, P, P, 256, 256, 100, 1, None, 0, None) == SHAPE       # K % 64
    assert lib.dg_linear(P, MIS, P, 256, 256, 256, 1, None, 0, None) == ALIGN
    assert lib.dg_linear_e4m3(P, P, P, P, P, 256, 256, 192, 1, None) == SHAPE     # K % 128
    assert lib.dg_linear_e4m3(P, NULL, P, P, P, 256, 256, 256, 1, None) == INVALID


def test_quantize_and_fp8_unembedding_reject_bad_arguments(lib):
    assert lib.dg_quantize_e4m3(P, 4, 12, 1, P, P, None) == SHAPE                  # cols % 8
    assert lib.dg_quantize_e4m3(NULL, 4, 16, 1, P, P, None) == INVALID
    assert lib.dg_quantize_e4m3(P, 4, 16, 1, MIS, P, None) == ALIGN
    assert lib.dg_unembed_e4m3(P, P, P, P, P, 256, 2048, 1024 + 128, None) == SHAPE  # V % 256
    assert lib.dg_unembed_e4m3(P, P, P, P, P, 256, 2048 + 64, 1024, None) == SHAPE   # d % 128


def test_sample_commit_rejects_bad_arguments(lib, L):
    c = defaults(lib, L)
    ws = lib.dg_sample_commit_workspace_bytes(1, 256, 262144)
    args = lambda C, V, cfg, w, wn: lib.dg_sample_commit(  # noqa: E731
        P, P, P, P, P, ctypes.byref(cfg), 0, 0, 0, 1, C, V, None, w, wn, None)
    assert args(1025, 262144, c, P, ws) == SHAPE                                   # C > 1024
    assert args(256, 262146, c, P, ws) == SHAPE                                    # V % 4
    assert args(256, 262144, c, P, ws - 16) == WS
    assert args(256, 262144, c, NULL, ws) == WS
    bad = defaults(lib, L)
    bad.max_steps = 0
    assert args(256, 262144, bad, P, ws) == INVALID
    bad = defaults(lib, L)
    bad.selection = 2
    assert args(256, 262144, bad, P, ws) == INVALID
    bad = defaults(lib, L)
    bad.t_end = 0.0
    assert args(256, 262144, bad, P, ws) == INVALID


def test_canvas_attn_rejects_bad_arguments(lib):
    def call(hd=128, Hq=16, Hkv=8, mask=0, ld=16 * 128, ldkv=8 * 128, q=P, maxp=4096, lmax=4352):
        return lib.dg_canvas_attn(q, ld, P, P, ldkv, P, P, P, maxp, lmax, P, ld, None, 1, Hq,
                                  Hkv, 256, hd, 0.088, mask, P, 1 << 30, None)
    assert call(hd=96, ld=16 * 96, ldkv=8 * 96) == SHAPE
    assert call(Hq=12, Hkv=8) == INVALID          # Hq % Hkv
    assert call(mask=5) == INVALID
    assert call(maxp=5000) == INVALID             # prefix beyond the cache
    assert call(ld=16 * 128 - 8) == ALIGN         # leading dimension below Hq * hd
    assert call(q=MIS) == ALIGN
    assert call(q=NULL) == INVALID


def test_canvas_attn_e4m3_rejects_bad_arguments(lib):
    def call(hd=128, Hq=16, Hkv=8, mask=0, ldq=16 * 128, ldkv=8 * 128, ldvt=256, lmax=4352,
             q=P, qs=P, maxp=4096, ws_bytes=1 << 30):
        return lib.dg_canvas_attn_e4m3(q, ldq, qs, P, ldkv, P, ldvt, P, P, P, P, P, maxp, lmax,
                                       P, 16 * 128, None, 1, Hq, Hkv, 256, hd, 0.088, mask, P,
                                       ws_bytes, None)
    assert call(hd=64) == SHAPE                   # e4m3 attention is hd = 128 only
    assert call(Hq=12, Hkv=8) == INVALID          # Hq % Hkv
    assert call(mask=5) == INVALID
    assert call(maxp=5000) == INVALID             # prefix beyond the cache
    assert call(ldvt=200) == ALIGN                # ldvt below Lq
    assert call(ldvt=264) == ALIGN                # ldvt not a multiple of 16
    assert call(lmax=4360) == ALIGN               # lmax not a multiple of 16
    assert call(ldq=16 * 128 - 16) == ALIGN       # leading dimension below Hq * 128
    assert call(q=MIS) == ALIGN
    assert call(qs=NULL) == INVALID               # the per-token scales are required
    assert call(ws_bytes=16) == WS                # the split plan needs its partials


def test_workspace_queries(lib, L):
    assert lib.dg_sample_commit_workspace_bytes(0, 256, 512) == 0
    assert lib.dg_unembed_sample_commit_workspace_bytes(1, 256, 1000) == 0         # V % 256
    # the fused path's partials: tokens x 3 x (vocabulary segments per token
    # tile), and a wider batch spreads the pairs over more token tiles
    a = lib.dg_unembed_sample_commit_workspace_bytes(1, 256, 262144)
    b = lib.dg_unembed_sample_commit_workspace_bytes(8, 256, 262144)
    assert a > 0 and b > 0
    assert lib.dg_canvas_attn_workspace_bytes(1, 16, 8, 256, 128, 4096) > 0
    cfg = L.ModelCfg(2048, 24, 16, 8, 128, 8192, 262144, 1e-6)
    w1 = lib.dg_denoise_block_workspace_bytes(ctypes.byref(cfg), 1, 256, 4352)
    w8 = lib.dg_denoise_block_workspace_bytes(ctypes.byref(cfg), 8, 256, 4352)
    assert 0 < w1 < w8
    assert lib.dg_denoise_block_workspace_bytes(ctypes.byref(cfg), 0, 256, 4352) == 0


def test_model_checks_reject_bad_configurations(lib, L):
    layers = (L.LayerWeights * 2)(*[L.LayerWeights(P.value, P.value, P.value, P.value)] * 2)
    st = L.State()

    def model(**kw):
        c = dict(d=256, n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024, vocab=512,
                 eps=1e-6)
        c.update(kw)
        cfg = L.ModelCfg(c["d"], c["n_layers"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"],
                         c["ffn"], c["vocab"], c["eps"])
        return L.Model(cfg, P.value, P.value, ctypes.cast(layers, ctypes.POINTER(L.LayerWeights)),
                       None, None, None)

    scfg = defaults(lib, L)
    steps = ctypes.c_int(0)

    def run(m):
        return lib.dg_denoise_block(ctypes.byref(m), ctypes.byref(st), ctypes.byref(scfg), 0, 0,
                                    ctypes.byref(steps), P, 1 << 30, None)
    assert run(model(head_dim=96)) == SHAPE
    assert run(model(n_q_heads=3)) == INVALID      # Hq % Hkv
    assert run(model(ffn=1000)) == SHAPE           # not a multiple of 128
    m = model()
    m.unembed_e4m3 = P.value                       # an e4m3 unembedding without its scale
    assert run(m) == INVALID


def test_kv_block_commit_rejects_bad_arguments(lib):
    arr = ctypes.c_void_p * 2
    tab = arr(P.value, P.value)
    call = lambda hd, ld=8 * 128, nl=2: lib.dg_kv_block_commit(  # noqa: E731
        tab, tab, ld, tab, tab, P, nl, 1, 8, 256, hd, 4352, None)
    assert call(96, ld=8 * 96) == SHAPE            # head_dim not 64 or 128
    assert call(128, ld=8 * 128 - 8) == ALIGN      # leading dimension below Hkv * hd
    assert call(128, nl=65) == INVALID             # more layers than the tables hold
    assert lib.dg_kv_block_commit(tab, tab, 1024, tab, tab, NULL, 2, 1, 8, 256, 128, 4352,
                                  None) == INVALID


def test_projection_plans(lib):
    """One canvas takes the split-K GEMM; many tokens the CTA pairs (a full
    wave of 74 pairs of 256 x 256 tiles, or 48 tiles and more with 1536 tokens
    and more), when N is a multiple of 256 and K holds four 128-byte k-blocks."""
    SK, PR = 0, 1
    plan = lib.dg_linear_plan_of
    assert plan(256, 2048, 8192, 0) == SK          # one canvas, MLP down: 8 tiles
    assert plan(256, 262144, 2048, 0) == PR        # 1024 tiles
    assert plan(4096, 2048, 2048, 0) == PR         # 128 tiles
    assert plan(1024, 4096, 2048, 0) == SK         # 64 tiles, 1024 tokens
    assert plan(1536, 2048, 2048, 0) == PR         # 48 tiles, 1536 tokens
    assert plan(1535, 2048, 2048, 0) == SK         # 48 tiles, 1535 tokens
    assert plan(1600, 2048, 512, 0) == PR          # 56 tiles, ragged token tile
    assert plan(4096, 2048 + 128, 2048, 0) == SK   # N not a multiple of 256
    assert plan(4096, 2048, 192, 0) == SK          # three bf16 k-blocks
    assert plan(4096, 2048, 384, 1) == SK          # three e4m3 k-blocks
    assert plan(4096, 2048, 512, 1) == PR
    assert plan(4096, 2048, 100, 0) == -1          # K % 64
    assert plan(4096, 2048, 192, 1) == -1          # K % 128 on e4m3 codes
    assert plan(0, 2048, 2048, 0) == -1


def test_residual_projections_share_one_plan(lib, L):
    """dg_model_residual_on_pairs: whether both residual projections (output
    and MLP down) run on CTA pairs; each picks its plan from its own shape."""
    tiny = L.ModelCfg(256, 2, 4, 2, 64, 1024, 512, 1e-6)
    full = L.ModelCfg(2048, 24, 16, 8, 128, 8192, 262144, 1e-6)

    def on_pairs(cfg, M, e4m3):
        return lib.dg_model_residual_on_pairs(ctypes.byref(cfg), M, e4m3)
    assert on_pairs(full, 256, 0) == 0             # one canvas
    assert on_pairs(full, 2048, 0) == 1            # eight canvases: 64 tiles
    assert on_pairs(full, 4096, 0) == 1            # a 4096-token prefill
    assert on_pairs(full, 2048, 1) == 1
    assert on_pairs(tiny, 48 * 256, 0) == 1        # d = 256: one tile per 256 tokens
    assert on_pairs(tiny, 47 * 256, 0) == 0
    # e4m3: Hq hd = 256 is two 128-wide k-blocks, so the output projection
    # stays on the split-K GEMM while the MLP down projection takes the pairs
    assert lib.dg_linear_plan_of(75 * 256, 256, 1024, 1) == 1
    assert lib.dg_linear_plan_of(75 * 256, 256, 256, 1) == 0
    assert on_pairs(tiny, 75 * 256, 1) == 0
    assert lib.dg_model_residual_on_pairs(None, 256, 0) == -1
    assert on_pairs(full, 0, 0) == -1


def test_wait_limit_and_self_test_arguments(lib):
    """The wait limit must lie in [1 us, 600 s] (0: the default), and the
    self-test kind must be 0 or 1; both are checked before any device work."""
    for bad in (1, 999, 600_000_000_001):
        assert lib.dg_set_wait_limit_ns(bad, None) == 1
        assert b"outside" in lib.dg_last_error()
    assert lib.dg_self_test_wait(2, None) == 1
    assert lib.dg_self_test_wait(-1, None) == 1
