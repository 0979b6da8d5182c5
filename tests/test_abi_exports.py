"""The C ABI library builds, loads without a GPU and exports every declared symbol."""
import ctypes
import os
import re

from conftest import ROOT


def declared_functions():
    with open(os.path.join(ROOT, "include", "dg.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for required in ("dg_canvas_attn", "dg_unembed", "dg_sample_commit", "dg_kv_block_commit",
                     "dg_denoise_block"):
        assert required in names


def test_library_loads_and_exports_every_symbol():
    from canvas_denoising_denoise_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_signatures_cover_the_header():
    from canvas_denoising_denoise_b200 import _lib
    assert set(_lib.SIGNATURES) == set(declared_functions())


def test_host_side_queries_without_a_gpu():
    from canvas_denoising_denoise_b200 import _lib
    lib = _lib.load()
    assert lib.dg_version() >= 1
    assert lib.dg_status_string(4) == b"DG_ERR_WORKSPACE_TOO_SMALL"
    c = _lib.SamplerCfg()
    lib.dg_sampler_defaults(ctypes.byref(c))
    assert (c.max_steps, c.commit_k) == (48, 16)
    assert abs(c.t_start - 0.8) < 1e-7 and abs(c.t_end - 0.4) < 1e-7
    assert abs(c.renoise_conf - 0.05) < 1e-9 and abs(c.stop_entropy - 0.005) < 1e-9
    # workspace queries are pure host arithmetic
    assert lib.dg_sample_commit_workspace_bytes(1, 256, 262144) > 0
    mc = _lib.ModelCfg(2048, 24, 16, 8, 128, 8192, 262144, 1e-6)
    assert lib.dg_denoise_block_workspace_bytes(ctypes.byref(mc), 1, 256, 4352) > 256 * 262144 * 4


def test_argument_errors_are_reported_before_any_launch():
    from canvas_denoising_denoise_b200 import _lib
    lib = _lib.load()
    st = lib.dg_unembed(None, None, None, 1, 64, 128, None, 0, None)
    assert st == 1 and b"null" in lib.dg_last_error()
    # misaligned pointer
    st = lib.dg_unembed(ctypes.c_void_p(8), ctypes.c_void_p(16), ctypes.c_void_p(32), 1, 64, 128,
                        None, 0, None)
    assert st == 3
    # unsupported head dim
    st = lib.dg_canvas_attn(ctypes.c_void_p(16), 96, ctypes.c_void_p(16), ctypes.c_void_p(16), 96,
                            ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 0, 1,
                            ctypes.c_void_p(16), 96, None, 1, 1, 1, 8, 96, 0.1, 0, None, 0, None)
    assert st == 2
