"""GPU parity of mamba2_mixer_forward (through the C ABI) against the fp64 oracle."""
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


def test_mixer_small(cuda_lib, oracle):
    cfg = dict(datagen.config(4), batch=2, seqlen=300, d_model=256, nheads=8, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    assert_close(out.float().cpu().numpy(), _oracle(oracle, cfg, inp), TOL_BF16, "mixer small", out_dtype="bf16")


def test_mixer_odd_tokens_and_width(cuda_lib, oracle):
    cfg = dict(datagen.config(4), batch=1, seqlen=131, d_model=320, nheads=10, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    assert_close(out.float().cpu().numpy(), _oracle(oracle, cfg, inp), TOL_BF16, "mixer odd", out_dtype="bf16")


def test_mixer_12b_width_full_size(cuda_lib, oracle):
    """Workload 4 (B8 L8192 d_model 5120, H160 G8): batch rows 0 and 7, first 1024 tokens
    (exact: rows are independent and the layer is causal)."""
    cfg = datagen.config(4)
    inp = datagen.make_inputs(4)
    out = _mixer(cfg, inp)
    got = out[[0, 7], :1024].float().cpu().numpy()
    want = _oracle(oracle, cfg, inp, rows=[0, 7], tokens=1024)
    assert_close(got, want, TOL_BF16, "mixer 12B width", out_dtype="bf16")


def test_mixer_against_the_unrounded_oracle(cuda_lib, oracle):
    """The layer against the oracle with no rounding anywhere (fp64 end to end), beside the
    oracle that rounds the three activations the layer stores in bf16 (its definition: the
    layer runs in bf16).  All three figures are printed: GPU vs rounded oracle (the asserted
    parity bound), GPU vs unrounded oracle, and rounded vs unrounded oracle -- the part of the
    gap that the bf16 storage of the activations alone accounts for.  Measured on B200: the
    unrounded comparison exceeds 2e-2 by a little (about 2.2e-2 over the storage rounding),
    so it is held to the bound plus the rounding-only gap."""
    cfg = dict(datagen.config(4), batch=2, seqlen=300, d_model=256, nheads=8, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    got = _mixer(cfg, inp).float().cpu().numpy()
    rounded = _oracle(oracle, cfg, inp)
    exact = _oracle(oracle, cfg, inp, bf16_activations=False)
    assert_close(got, rounded, TOL_BF16, "mixer vs bf16-activation oracle", out_dtype="bf16")
    gap = rel_err(rounded, exact)
    print(f"[parity] bf16-activation oracle vs unrounded oracle: max|diff|/RMS = {gap:.3e}")
    assert_close(got, exact, TOL_BF16 + gap, "mixer vs unrounded fp64 oracle", out_dtype="bf16")
