"""Failure detection on the device, without faulting or hanging the GPU.

Every wait in the kernels is bounded by the device's wait limit; on expiry it
records DG_ERR_TIMEOUT in the error word and the kernel returns.  Here the
limit is set to 1 ms and a self-test kernel waits on an mbarrier that nothing
arrives at: the wait must run out, dg_check_device_errors must report the
timeout (and clear it), and the context must stay usable afterwards.
"""
import time

import pytest
import torch

from conftest import read_golden_table

pytestmark = pytest.mark.gpu

DG_ERR_TIMEOUT = 6


@pytest.mark.parametrize("kind,site", [(0, 0x7F1), (1, 0x7F2)])
def test_expired_wait_reports_timeout_and_the_context_survives(kind, site):
    import canvas_denoising_denoise_b200 as dg
    from canvas_denoising_denoise_b200 import _lib
    assert dg.check_device_errors() == 0
    dg.set_wait_limit_ns(1_000_000)
    try:
        t0 = time.perf_counter()
        dg.self_test_wait(kind)
        with pytest.raises(dg.DgError) as e:
            dg.check_device_errors()
        took = time.perf_counter() - t0
    finally:
        dg.set_wait_limit_ns(0)
    assert e.value.status == DG_ERR_TIMEOUT
    assert f"site 0x{site:x}" in str(e.value)
    assert took < 1.0  # the 1 ms limit, not the 2 s default
    # the word was cleared, and ordinary work runs and reports no error
    assert dg.check_device_errors() == 0
    inp = torch.zeros((4, 6), dtype=torch.int32, device="cuda")
    out = torch.empty((4, 4), dtype=torch.int32, device="cuda")
    dg.philox(inp, out)
    assert dg.check_device_errors() == 0
    # the published known answer for a zero counter and key
    want = [int(x, 16) for x in read_golden_table("philox4x32_10_kat.txt")[0][6:]]
    assert [v & 0xFFFFFFFF for v in out[0].tolist()] == want

