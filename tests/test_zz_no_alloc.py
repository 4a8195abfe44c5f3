"""ssd_prefill_noalloc against ssd_prefill (GPU, through the C ABI).

The no-allocation entry point serves callers that may not create device allocations of their
own; it runs the same prefill with the library's fixed per-device scratch.  Its results must
match the regular entry point on the same inputs, on consecutive calls (the scratch keeps the
previous call's contents), and oversized requests must be refused.  This file is collected
last so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

from tests.gpu_util import TOL_BF16, assert_close, dev, host, make_case, small_cfg

pytestmark = pytest.mark.gpu


def _args(inp):
    return (dev(inp["xBC"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["D"]), dev(inp["dt_bias"]),
            dev(inp.get("conv_w")), dev(inp.get("conv_b")), dev(inp.get("z")), dev(inp.get("norm_w")),
            dev(inp.get("h0")), dev(inp.get("conv_state_in")))


def _poison_scratch(ssd, torch):
    """One no-allocation call near the size limit on NaN inputs, so that most of the shared
    scratch holds NaNs when the compared calls run: a read of scratch that a call did not
    write first would then show up in their outputs."""
    cfg = small_cfg(batch=1, nheads=32, ngroups=4, norm_groups=4)
    L = 128
    while ssd.workspace_size(cfg, seqlen=2 * L) <= ssd.NOALLOC_WORKSPACE_BYTES and L < (1 << 16):
        L *= 2
    cfg = dict(cfg, seqlen=L)
    assert ssd.workspace_size(cfg) > ssd.NOALLOC_WORKSPACE_BYTES // 4
    inp = make_case(cfg, seed_idx=9)
    a = list(_args(inp))
    for i in (0, 1, 7):  # xBC, dt, z
        a[i] = torch.full_like(a[i], float("nan"))
    ssd.prefill_noalloc(cfg, *a)
    torch.cuda.synchronize()


def test_noalloc_matches_prefill_on_consecutive_calls(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    _poison_scratch(ssd, torch)
    cases = [small_cfg(seqlen=333), small_cfg(seqlen=517, norm_groups=0)]
    for i, cfg in enumerate(cases):  # two calls in a row, different shapes and options
        assert ssd.workspace_size(cfg) <= ssd.NOALLOC_WORKSPACE_BYTES
        inp = make_case(cfg, seed_idx=1 + i)
        a = _args(inp)
        y0, h0, c0 = ssd.prefill(cfg, *a)
        y1, h1, c1 = ssd.prefill_noalloc(cfg, *a)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical results, and nothing stale read
        assert torch.isfinite(y1.float()).all() and torch.isfinite(h1).all(), f"call {i}"
        assert torch.equal(y1, y0), f"noalloc call {i}: y differs from ssd_prefill"
        assert torch.equal(h1, h0), f"noalloc call {i}: h_final differs from ssd_prefill"
        assert torch.equal(c1, c0)
        assert_close(y1.float().cpu().numpy(), y0.float().cpu().numpy(), TOL_BF16,
                     f"noalloc call {i} y", out_dtype="bf16", both_rounded=True)
        assert_close(host(h1), host(h0), TOL_BF16, f"noalloc call {i} h_final")
    assert ssd.get_device_error() == 0


def test_noalloc_refuses_requests_beyond_its_scratch(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import datagen, ssd
    cfg = dict(datagen.config(1), seqlen=4096, norm_groups=8)  # ~300 MB of scratch
    assert ssd.workspace_size(cfg) > ssd.NOALLOC_WORKSPACE_BYTES
    cd = datagen.conv_dim(cfg)
    x = torch.zeros((1, 4096, cd), dtype=torch.bfloat16, device="cuda")
    dt = torch.zeros((1, 4096, 128), dtype=torch.bfloat16, device="cuda")
    z = torch.zeros((1, 4096, 8192), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros(128, device="cuda")
    w = torch.zeros((cd, 4), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SsdError) as ei:
        ssd.prefill_noalloc(cfg, x, dt, p, p, p, w, None, z)
    assert ei.value.status == 7  # SSD_ERR_WORKSPACE
