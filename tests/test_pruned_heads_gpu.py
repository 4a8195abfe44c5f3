"""GPU parity at the pruned head counts: 112 and 120 Mamba heads in 8 groups (14 or 15 heads
per group, not a power of two), which the compressed 9B model's Mamba layers search over
(neurohive.io article, section "Model compression"; hyper.ai summary, section "Method").
Exercises the group-to-head mapping, the norm groups of 896 / 960 channels, a decode group
of 14 heads and a ragged in_proj width."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, assert_close, dev, host, make_case, oracle_output,
                            run_gpu_prefill, run_oracle_prefill)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H", [112, 120])
@pytest.mark.parametrize("kernel", [1, 2])
def test_prefill_pruned_heads(cuda_lib, oracle, H, kernel):
    cfg = dict(datagen.config(1), batch=1, seqlen=300, nheads=H, ngroups=8, norm_groups=8)
    inp = make_case(cfg, seed_idx=5)
    y, hf, cso = run_gpu_prefill(cfg, inp, kernel=kernel)
    ref = run_oracle_prefill(oracle, cfg, inp)
    assert_close(y.float().cpu().numpy(), oracle_output(ref, cfg), TOL_BF16, f"H{H} y", out_dtype="bf16")
    assert_close(host(hf), ref["h_final"], TOL_BF16, f"H{H} h_final")
    assert np.array_equal(host(cso), ref["conv_state_out"])


def test_decode_pruned_heads(cuda_lib, oracle):
    from tests.test_decode_gpu import _run_steps
    cfg = dict(datagen.config(2), batch=2, nheads=112, ngroups=8, norm_groups=8)
    _run_steps(oracle, cfg, steps=4)


def test_mixer_pruned_width(cuda_lib, oracle):
    """The compressed model's width: d_model 4480 with 112 heads (in_proj width 16496)."""
    from tests.test_mixer_gpu import _mixer, check_mixer
    cfg = dict(datagen.config(4), batch=1, seqlen=160, d_model=4480, nheads=112, ngroups=8,
               norm_groups=8)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    check_mixer(out.float().cpu().numpy(), oracle, cfg, inp, "mixer d4480 H112")
