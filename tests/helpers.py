"""Shared test helpers: tolerances and comparisons (no method arithmetic)."""
import numpy as np
import pytest
import torch

# Floating-point parity bar for attention and logits (bf16 inputs, fp32
# accumulation): relative L2 error <= 1e-2 and max absolute error <= 3e-2.
REL_L2 = 1e-2
MAX_ABS = 3e-2


def assert_close_bf16(got, want, rel_l2=REL_L2, max_abs=MAX_ABS, what=""):
    """The bar for a tensor the product stores in bf16 (the KV cache): rel-L2
    as for logits, and elementwise max-abs plus one bf16 step at the value's
    magnitude (2^-7 relative), since a stored value may round to the
    neighbouring bf16 number when its unrounded value sits within rounding of
    the boundary."""
    got = to64(got)
    want = to64(want)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    excess = float(np.max(err - (max_abs + np.abs(want) * 2.0 ** -7))) if err.size else 0.0
    assert rel <= rel_l2 and excess <= 0, f"{what}: rel_l2={rel:.3e} max excess={excess:.3e}"
    return rel


def cuda_ok():
    return torch.cuda.is_available()


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def assert_close(got, want, rel_l2=REL_L2, max_abs=MAX_ABS, what=""):
    got = to64(got)
    want = to64(want)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = got - want
    rel = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)
    mx = float(np.max(np.abs(err))) if err.size else 0.0
    assert rel <= rel_l2 and mx <= max_abs, f"{what}: rel_l2={rel:.3e} max_abs={mx:.3e}"
    return rel, mx


def gpu_weights(w_cpu, device="cuda"):
    return {"embed": w_cpu["embed"].to(device), "unembed": w_cpu["unembed"].to(device),
            "layers": [{k: v.to(device) for k, v in lw.items()} for lw in w_cpu["layers"]]}
