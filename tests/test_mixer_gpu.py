"""GPU parity of mamba2_mixer_forward (through the C ABI) against the fp64 oracle.

The layer is compared with the oracle with no rounding anywhere (fp64 end to end).  A bf16
layer stores activations between its steps in bf16, and the layer's output is sensitive to
that storage (the in_proj output sets dt, whose exponentials compound over the sequence), so
the bound is the bf16 tolerance plus how far that storage alone moves the output: the distance
between the unrounded oracle and the oracle that rounds the activations a plain bf16 layer
stores (RMSNorm output, in_proj output, gated-norm output).  This layer stores only the last
two (the RMSNorm is folded into the in_proj GEMM).  Every figure is printed."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import TOL_BF16, assert_close, dev, rel_err

pytestmark = pytest.mark.gpu


def _mixer(cfg, inp, **kw):
    from mamba_ssd_scan_02_b200 import ssd
    return ssd.mixer_forward(cfg, dev(inp["hidden"]), dev(inp["rms_w"]), dev(inp["W_in"]),
                             dev(inp["W_out"]), dev(inp["A"]), dev(inp["D"]), dev(inp["dt_bias"]),
                             dev(inp["conv_w"]), None, dev(inp["norm_w"]), **kw)


def _oracle(oracle, cfg, inp, rows=None, tokens=None, bf16_activations=True):
    return oracle.mixer_forward(cfg, inp["hidden"], inp["rms_w"], inp["W_in"], inp["W_out"],
                                inp["A"], inp["D"], inp["dt_bias"], inp["conv_w"], None,
                                inp["norm_w"], rows=rows, tokens=tokens,
                                bf16_activations=bf16_activations)


def check_mixer(got, oracle, cfg, inp, what, rows=None, tokens=None):
    """got against the unrounded oracle, within TOL_BF16 plus the bf16-storage gap (above)."""
    exact = _oracle(oracle, cfg, inp, rows=rows, tokens=tokens, bf16_activations=False)
    rounded = _oracle(oracle, cfg, inp, rows=rows, tokens=tokens)
    gap = rel_err(rounded, exact)
    print(f"[parity] {what}: bf16-activation oracle vs unrounded oracle: max|diff|/RMS = {gap:.3e}")
    assert_close(got, exact, TOL_BF16 + gap, f"{what} vs unrounded oracle", out_dtype="bf16")
    assert_close(got, rounded, TOL_BF16 + gap, f"{what} vs bf16-activation oracle", out_dtype="bf16")


def test_mixer_small(cuda_lib, oracle):
    cfg = dict(datagen.config(4), batch=2, seqlen=300, d_model=256, nheads=8, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    check_mixer(out.float().cpu().numpy(), oracle, cfg, inp, "mixer small")


def test_mixer_odd_tokens_and_width(cuda_lib, oracle):
    cfg = dict(datagen.config(4), batch=1, seqlen=131, d_model=320, nheads=10, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    check_mixer(out.float().cpu().numpy(), oracle, cfg, inp, "mixer odd")


def test_mixer_12b_width_full_size(cuda_lib, oracle):
    """Workload 4 (B8 L8192 d_model 5120, H160 G8): batch rows 0 and 7, first 1024 tokens
    (exact: rows are independent and the layer is causal)."""
    cfg = datagen.config(4)
    inp = datagen.make_inputs(4)
    out = _mixer(cfg, inp)
    got = out[[0, 7], :1024].float().cpu().numpy()
    check_mixer(got, oracle, cfg, inp, "mixer 12B width", rows=[0, 7], tokens=1024)
