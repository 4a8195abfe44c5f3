"""Failure detection on the GPU without a GPU fault: a bounded device wait that runs out.

The tensor-core scan's waits on its pipeline barriers are bounded.  The test hook
ssd_test_stall_scan makes the scan withhold one chunk's B/C tile, so the CTAs waiting for it
give up after a short limit.  The call must then report SSD_ERR_TIMEOUT through
ssd_get_device_error(), and the device must stay usable: the CTAs left cleanly (loads
drained, MMAs complete, tensor memory released), so the same prefill run right after it
matches the oracle.
"""
import pytest

from tests.gpu_util import (assert_close, host, make_case, oracle_output, run_gpu_prefill,
                            run_oracle_prefill, small_cfg, tol_for)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stall_chunk", [0, 1, 2])
def test_scan_wait_timeout_is_reported_and_the_device_recovers(cuda_lib, oracle, stall_chunk):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=333)  # 3 chunks of 128 tokens (the last one ragged)
    inp = make_case(cfg)
    assert ssd.get_device_error() == 0
    ssd.test_stall_scan(stall_chunk, wait_limit_ms=20.0)
    try:
        run_gpu_prefill(cfg, inp, kernel=ssd.KERNEL_TENSOR)
        status = ssd.get_device_error()
    finally:
        ssd.test_stall_scan(-1)
    assert status == 5, f"expected SSD_ERR_TIMEOUT, got {ssd.STATUS.get(status, status)}"
    # the same call again: complete, correct, and no error latched
    y, hf, cso = run_gpu_prefill(cfg, inp, kernel=ssd.KERNEL_TENSOR)
    torch.cuda.synchronize()
    assert ssd.get_device_error() == 0
    ref = run_oracle_prefill(oracle, cfg, inp)
    assert_close(y.float().cpu().numpy(), oracle_output(ref, cfg), tol_for(cfg),
                 f"after stall {stall_chunk}: y", out_dtype="bf16")
    assert_close(host(hf), ref["h_final"], tol_for(cfg), f"after stall {stall_chunk}: h_final")
