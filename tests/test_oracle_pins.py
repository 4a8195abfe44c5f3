"""CPU pins of the fp64 oracle (no GPU)."""
import json
import os

import numpy as np
import pytest

import oracle as _oracle
from tests import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mamba2_layer_hparams.json")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(oracle, pin):
    ok, detail = pin(oracle)
    assert ok, detail


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("k", sorted(pins.MUTANTS), ids=lambda k: pins.MUTANTS[k].replace(" ", "_"))
def test_planted_mistake_is_caught(k, mutant_dir):
    """Each planted mistake in the oracle must fail at least one pin."""
    om = _oracle.mutant(k, mutant_dir)
    failed = [p.__name__ for p in pins.ALL_PINS if not p(om)[0]]
    assert failed, f"mutant {k} ({pins.MUTANTS[k]}) passed every pin"


def test_workload_shapes_follow_the_pages():
    """The workload shapes use the Mamba-2 hyper-parameters the pages print."""
    from mamba_ssd_scan_02_b200 import datagen
    g = json.load(open(GOLDEN))
    for i in range(5):
        c = datagen.config(i)
        assert c["headdim"] == g["mamba2_head_dim"] and c["dstate"] == g["mamba2_state_dim"]
        if i > 0:
            assert c["ngroups"] == g["mamba2_groups"] and c["conv_width"] == g["mamba2_conv_window"]
    c4 = datagen.config(4)
    assert c4["d_model"] == g["d_model_12b"]
    assert c4["nheads"] * c4["headdim"] == g["mamba2_expand"] * g["d_model_12b"]


def test_oracle_full_width_head_subset_is_exact(oracle):
    """Heads are independent: running a subset of heads gives the same numbers bit for bit
    (this is what the sampled full-size parity checks rely on)."""
    from mamba_ssd_scan_02_b200 import datagen
    cfg = dict(datagen.config(1), seqlen=40, nheads=16, ngroups=2, norm_groups=2)
    inp = datagen.make_inputs(1, cfg)
    z = datagen.normal(99, "z", (1, 40, 16 * 64))
    full = oracle.ssd_prefill(cfg, inp["xBC"], inp["dt"], inp["A"], inp["D"], inp["dt_bias"],
                              conv_w=inp["conv_w"], z=z, threads=2)
    part = oracle.ssd_prefill(cfg, inp["xBC"], inp["dt"], inp["A"], inp["D"], inp["dt_bias"],
                              conv_w=inp["conv_w"], z=z, heads=(8, 16), threads=2)
    assert np.array_equal(part["y"], full["y"][:, :, 8:16])
    assert np.array_equal(part["h_final"], full["h_final"][:, 8:16])
    assert np.array_equal(part["out"], full["out"][:, :, 512:])


def test_datagen_is_deterministic_and_thread_independent():
    from mamba_ssd_scan_02_b200 import datagen
    a = datagen.normal(5, "xBC", (3, 1 << 21), threads=1)
    b = datagen.normal(5, "xBC", (3, 1 << 21), threads=4)
    assert np.array_equal(a, b)
    v = datagen.bf16_value(a).astype(np.float64)
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1) < 5e-3
    # bf16 rounding: ties go to even, values representable in bf16 are unchanged
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-3], np.float32)
    bits = datagen.bf16_bits(x)
    assert datagen.bf16_value(bits)[0] == 1.0 and datagen.bf16_value(bits)[1] == 1.0
    assert datagen.bf16_value(bits)[2] == 1.0 + 2 ** -6 and datagen.bf16_value(bits)[3] == -2.5
    hp = datagen.head_params(7, 128)
    dt0 = np.log1p(np.exp(hp["dt_bias"].astype(np.float64)))
    assert np.all(dt0 > 0.99e-3) and np.all(dt0 < 1.01e-1)
    assert np.all(hp["A"] <= -1.0) and np.all(hp["A"] >= -16.0)
