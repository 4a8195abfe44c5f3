"""GPU parity of the normalise-first output norm, out = rmsnorm(y) * w * silu(z)
(norm_before_gate = 1), against the fp64 oracle: prefill on both kernel families, decode
and the mixer layer."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, assert_close, host, make_case, oracle_output,
                            run_gpu_prefill, run_oracle_prefill, small_cfg)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("norm_groups", [2, 1])
def test_prefill_norm_before_gate(cuda_lib, oracle, kernel, norm_groups):
    cfg = small_cfg(norm_before_gate=True, norm_groups=norm_groups)
    inp = make_case(cfg, seed_idx=6)
    y, hf, _ = run_gpu_prefill(cfg, inp, kernel=kernel)
    ref = run_oracle_prefill(oracle, cfg, inp)
    assert_close(y.float().cpu().numpy(), oracle_output(ref, cfg), TOL_BF16, "nbg y", out_dtype="bf16")
    assert_close(host(hf), ref["h_final"], TOL_BF16, "nbg h_final")


def test_prefill_gate_order_matters(cuda_lib):
    """The two orders give different outputs (the flag reaches the kernel)."""
    cfg = small_cfg()
    inp = make_case(cfg, seed_idx=6)
    y0, _, _ = run_gpu_prefill(cfg, inp)
    y1, _, _ = run_gpu_prefill(dict(cfg, norm_before_gate=True), inp)
    assert not np.allclose(y0.float().cpu().numpy(), y1.float().cpu().numpy(), rtol=1e-2, atol=1e-2)


def test_decode_norm_before_gate(cuda_lib, oracle):
    from tests.test_decode_gpu import _decode_cfg, _run_steps
    _run_steps(oracle, _decode_cfg(norm_before_gate=True), steps=5)


def test_mixer_norm_before_gate(cuda_lib, oracle):
    from tests.test_mixer_gpu import _mixer, check_mixer
    cfg = dict(datagen.config(4), batch=1, seqlen=200, d_model=256, nheads=8, ngroups=2,
               norm_groups=2, norm_before_gate=True)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    check_mixer(out.float().cpu().numpy(), oracle, cfg, inp, "mixer nbg")
