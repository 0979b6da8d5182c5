"""dg_sample_commit_noalloc: the sampler step for callers that cannot allocate.

Some callers cannot allocate device memory for a workspace - a plugin whose
host application owns every device allocation, or code enqueueing work while
a stream is being captured, where cudaMalloc is not permitted.  The no-alloc
entry point keeps its scratch in a fixed static device array instead.  These
tests call it through the C ABI and check that two consecutive calls give the
same results as the workspace entry point on the same inputs.

The file name sorts last so that a run stopping at the first failure has
already run every other test; the test also passes alone in a fresh process
(its first call performs the per-device set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import assert_close


def _canvas(B, C, V, seed):
    g = torch.Generator().manual_seed(seed)
    tok = torch.randint(0, V, (B, C), generator=g, dtype=torch.int64).to(torch.int32)
    committed = (torch.rand((B, C), generator=g) < 0.3).to(torch.uint8)
    return {"tok": tok.cuda(), "committed": committed.cuda(),
            "prev": torch.full((B, C), -1, dtype=torch.int32, device="cuda"),
            "status": torch.zeros(B, dtype=torch.int32, device="cuda")}


def _outs(B, C):
    return {"x_hat": torch.empty((B, C), dtype=torch.int32, device="cuda"),
            "argmax": torch.empty((B, C), dtype=torch.int32, device="cuda"),
            "logconf": torch.empty((B, C), dtype=torch.float32, device="cuda"),
            "entropy": torch.empty((B, C), dtype=torch.float32, device="cuda"),
            "flags": torch.empty((B, C), dtype=torch.uint8, device="cuda")}


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import canvas_denoising_denoise_b200 as dg
    from canvas_denoising_denoise_b200 import _lib, synth
    lib = _lib.load()
    B, C, V = 2, 256, 65536
    settings = dg.SamplerSettings()
    seed, block = 21, 3
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    states = {"ws": _canvas(B, C, V, 5), "noalloc": _canvas(B, C, V, 5)}
    need = lib.dg_sample_commit_workspace_bytes(B, C, V)
    work = torch.empty(need, dtype=torch.uint8, device="cuda")
    for step in (7, 8):
        logits = synth.make_sampler_logits(B, C, V, seed=seed, step=step).cuda()
        outs = {}
        for name, s in states.items():
            o = _outs(B, C)
            so = _lib.StepOut(*[o[k].data_ptr() for k in
                                ("x_hat", "argmax", "logconf", "entropy", "flags")])
            args = (ctypes.c_void_p(logits.data_ptr()), ctypes.c_void_p(s["tok"].data_ptr()),
                    ctypes.c_void_p(s["committed"].data_ptr()),
                    ctypes.c_void_p(s["prev"].data_ptr()), ctypes.c_void_p(s["status"].data_ptr()),
                    ctypes.byref(settings.c), seed, block, step, B, C, V, ctypes.byref(so))
            if name == "ws":
                rc = lib.dg_sample_commit(*args, ctypes.c_void_p(work.data_ptr()), need, stream)
            else:
                rc = lib.dg_sample_commit_noalloc(*args, stream)
            assert rc == 0, lib.dg_last_error()
            outs[name] = o
        torch.cuda.synchronize()
        dg.check_device_errors()
        for k in ("tok", "committed", "prev", "status"):
            assert torch.equal(states["ws"][k], states["noalloc"][k]), (step, k)
        for k in ("x_hat", "argmax", "flags"):
            assert torch.equal(outs["ws"][k], outs["noalloc"][k]), (step, k)
        for k in ("logconf", "entropy"):
            assert_close(outs["noalloc"][k].cpu(), outs["ws"][k].cpu().double().numpy(),
                         rel_l2=1e-6, max_abs=1e-5, what=f"{k} step {step}")
        # the step did real work: 16 commits per sequence
        assert int(((outs["noalloc"]["flags"] & 1) != 0).sum()) == 16 * B


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from canvas_denoising_denoise_b200 import _lib
    lib = _lib.load()
    cfg = _lib.SamplerCfg()
    lib.dg_sampler_defaults(ctypes.byref(cfg))
    # two 32-byte chunk partials per position at V = 262144 (131072-entry
    # chunks with this many rows): the fixed 4 MiB holds 256 canvases of 256
    # positions exactly
    assert lib.dg_sample_commit_workspace_bytes(256, 256, 262144) == 4 << 20
    B, C, V = 257, 256, 262144
    assert lib.dg_sample_commit_workspace_bytes(B, C, V) > (4 << 20)
    p = ctypes.c_void_p(256)
    rc = lib.dg_sample_commit_noalloc(p, p, p, p, p, ctypes.byref(cfg), 0, 0, 0, B, C, V, None,
                                      None)
    assert rc == 2
    assert b"scratch" in lib.dg_last_error()
