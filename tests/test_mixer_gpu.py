"""GPU parity of mamba2_mixer_forward (through the C ABI) against the fp64 oracle.

The layer is held to the oracle with no rounding anywhere (fp64 end to end), at the bf16
bound.  The oracle that rounds the activations a plain bf16 layer stores between its steps
(RMSNorm output, in_proj output, gated-norm output) is reported beside it: this layer keeps
the RMSNorm output in fp32 (folded into the in_proj GEMM), so it sits between the two."""
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
    assert_close(out.float().cpu().numpy(), _oracle(oracle, cfg, inp, bf16_activations=False), TOL_BF16,
                 "mixer small", out_dtype="bf16")


def test_mixer_odd_tokens_and_width(cuda_lib, oracle):
    cfg = dict(datagen.config(4), batch=1, seqlen=131, d_model=320, nheads=10, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    out = _mixer(cfg, inp)
    assert_close(out.float().cpu().numpy(), _oracle(oracle, cfg, inp, bf16_activations=False), TOL_BF16,
                 "mixer odd", out_dtype="bf16")


def test_mixer_12b_width_full_size(cuda_lib, oracle):
    """Workload 4 (B8 L8192 d_model 5120, H160 G8): batch rows 0 and 7, first 1024 tokens
    (exact: rows are independent and the layer is causal)."""
    cfg = datagen.config(4)
    inp = datagen.make_inputs(4)
    out = _mixer(cfg, inp)
    got = out[[0, 7], :1024].float().cpu().numpy()
    want = _oracle(oracle, cfg, inp, rows=[0, 7], tokens=1024, bf16_activations=False)
    assert_close(got, want, TOL_BF16, "mixer 12B width", out_dtype="bf16")


def test_mixer_between_the_two_oracles(cuda_lib, oracle):
    """All three figures are printed: GPU vs the unrounded oracle (held to the bf16 bound), GPU
    vs the oracle of a plain bf16 layer (which rounds the RMSNorm output, the in_proj output and
    the gated-norm output), and the two oracles against each other -- how far the bf16 storage of
    those activations alone moves the output.  The layer rounds only the last two, so against
    the rounded oracle it is held to the bound plus that gap."""
    cfg = dict(datagen.config(4), batch=2, seqlen=300, d_model=256, nheads=8, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(4, cfg)
    got = _mixer(cfg, inp).float().cpu().numpy()
    rounded = _oracle(oracle, cfg, inp)
    exact = _oracle(oracle, cfg, inp, bf16_activations=False)
    assert_close(got, exact, TOL_BF16, "mixer vs unrounded fp64 oracle", out_dtype="bf16")
    gap = rel_err(rounded, exact)
    print(f"[parity] bf16-activation oracle vs unrounded oracle: max|diff|/RMS = {gap:.3e}")
    assert_close(got, rounded, TOL_BF16 + gap, "mixer vs bf16-activation oracle", out_dtype="bf16")
