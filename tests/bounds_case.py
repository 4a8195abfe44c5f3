"""One prefill through a given build of the library, its outputs saved to a file.

The GPU test of the debug build (test_debug_bounds_gpu.py) starts this in a subprocess per
build, since a process loads one build of the library:

    python tests/bounds_case.py <libssd.so path> <extent divisor> <norm groups> <out.npz>

The outputs are poisoned (NaN) before the call, so that the file shows which elements the
call wrote; the device error word after the call is saved with them."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main(lib, denom, norm_groups, out):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    from tests.gpu_util import dev, make_case, small_cfg
    ssd.load(lib)
    cfg = small_cfg(batch=1, seqlen=300, nheads=16, ngroups=2, norm_groups=norm_groups)
    inp = make_case(cfg, seed_idx=13)
    H, P, N, L = cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["seqlen"]
    y = torch.full((1, L, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    hf = torch.full((1, H, P, N), float("nan"), dtype=torch.float32, device="cuda")
    ssd.get_device_error()  # clear
    ssd.test_bounds_scale(denom)
    try:
        ssd.prefill(cfg, dev(inp["xBC"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["D"]), dev(inp["dt_bias"]),
                    dev(inp.get("conv_w")), dev(inp.get("conv_b")), dev(inp.get("z")), dev(inp.get("norm_w")),
                    dev(inp.get("h0")), dev(inp.get("conv_state_in")), y=y, h_final=hf, kernel=2)
        torch.cuda.synchronize()
    finally:
        ssd.test_bounds_scale(1)
    status = ssd.get_device_error()
    np.savez(out, y=y.float().cpu().numpy(), h_final=hf.cpu().numpy(), status=status,
             debug_build=int(ssd.debug_bounds_build()))


if __name__ == "__main__":
    main(sys.argv[1], int(sys.argv[2]), int(sys.argv[3]), sys.argv[4])
