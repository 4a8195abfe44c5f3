"""Helpers for the GPU parity tests: device transfer, tolerance checks, oracle calls."""
from __future__ import annotations

import os

import numpy as np

from mamba_ssd_scan_02_b200 import datagen

# acceptance bounds: max|err| <= tol * RMS(reference)
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol_for(cfg):
    return TOL_BF16 if cfg.get("dtype", "bf16") == "bf16" else TOL_F32


def rel_err(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rms = float(np.sqrt(np.mean(want * want)))
    return float(np.max(np.abs(got - want))) / max(rms, 1e-300)


# unit roundoff of the stored output: round-to-nearest into bf16 moves a value by at most
# 2^-8 of its magnitude (8 significant bits), fp32 by 2^-24
UNIT_ROUNDOFF = {"bf16": 2.0 ** -8, "f32": 2.0 ** -24}


def assert_close(got, want, tol, what, out_dtype="f32", both_rounded=False):
    """max|got - want| <= tol * RMS(want), applied on top of the rounding of the output into
    its storage dtype: |got - want| <= tol * RMS(want) + u * |want| elementwise (u = 2^-8 for
    bf16 outputs).  When `want` is itself a stored GPU result (two roundings), the allowance
    is 2u: the two values may round to neighbouring representable numbers.  Returns the plain
    max|err|/RMS."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = max(float(np.sqrt(np.mean(want * want))), 1e-300)
    excess = np.abs(got - want) - (2 if both_rounded else 1) * UNIT_ROUNDOFF[out_dtype] * np.abs(want)
    r_ex = float(np.max(excess)) / rms
    r = rel_err(got, want)
    # both figures: the plain one, and the one the bound applies to (the excess over the
    # storage rounding); pytest shows them with -s or -rA
    print(f"[parity] {what}: max|err|/RMS = {r:.3e}; max(|err| - {'2u' if both_rounded else 'u'}|ref|)/RMS"
          f" = {r_ex:.3e} (bound {tol:.1e}, u = {UNIT_ROUNDOFF[out_dtype]:.3g})")
    assert r_ex <= tol, (f"{what}: max(|err| - u|ref|)/RMS = {r_ex:.3e} > {tol:.1e} "
                         f"(plain max|err|/RMS = {r:.3e})")
    return r


def as_f64(a):
    """numpy array (uint16 bf16 bits or float) -> float64."""
    if a.dtype == np.uint16:
        return datagen.bf16_value(a).astype(np.float64)
    return a.astype(np.float64)


def dev(a):
    from mamba_ssd_scan_02_b200 import ssd
    return None if a is None else ssd.to_device(a)


def host(t):
    from mamba_ssd_scan_02_b200 import ssd
    return ssd.to_numpy(t)


def small_cfg(**kw):
    """A small bf16 workload: several 128-token chunks plus a ragged tail."""
    c = dict(datagen.config(1), batch=2, seqlen=333, nheads=16, ngroups=2, chunk=128,
             norm_groups=2)
    c.update(kw)
    return c


def make_case(cfg, seed_idx=1, with_h0=True, with_cache=True, with_bias=True):
    """Inputs for a (possibly reshaped) workload drawn from seed_idx's streams, plus
    optional initial state / conv cache / conv bias."""
    inp = datagen.make_inputs(seed_idx, cfg)
    H, P, N = cfg["nheads"], cfg["headdim"], cfg["dstate"]
    bf = cfg["dtype"] == "bf16"
    cd = datagen.conv_dim(cfg)
    seed = datagen.SEED_BASE + 100 + seed_idx
    if cfg["norm_groups"] and "z" not in inp:
        inp["z"] = datagen.normal(seed, "z", (cfg["batch"], cfg["seqlen"], H * P), bf16=bf)
    inp["h0"] = datagen.random_state(seed, (cfg["batch"], H, P, N)) if with_h0 else None
    W = cfg["conv_width"]
    inp["conv_state_in"] = (datagen.random_conv_state(seed, (cfg["batch"], W, cd), bf16=bf)
                            if (with_cache and W) else None)
    if with_bias and W:
        b = datagen.normal(seed, "D", (cd,), std=0.1, bf16=bf)
        inp["conv_b"] = b
    else:
        inp["conv_b"] = None
    if cfg["norm_groups"]:
        r = np.random.default_rng(seed)
        nw = r.uniform(0.5, 1.5, H * P).astype(np.float32)
        inp["norm_w"] = datagen.bf16_bits(nw) if bf else nw
    return inp


def run_gpu_prefill(cfg, inp, kernel=None, **kw):
    from mamba_ssd_scan_02_b200 import ssd
    y, hf, cso = ssd.prefill(cfg, dev(inp["xBC"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["D"]),
                             dev(inp["dt_bias"]), dev(inp.get("conv_w")), dev(inp.get("conv_b")),
                             dev(inp.get("z")), dev(inp.get("norm_w")), dev(inp.get("h0")),
                             dev(inp.get("conv_state_in")), kernel=kernel, **kw)
    return y, hf, cso


def run_oracle_prefill(oracle, cfg, inp, heads=None, threads=None):
    return oracle.ssd_prefill(cfg, inp["xBC"], inp["dt"], inp["A"], inp["D"], inp["dt_bias"],
                              conv_w=inp.get("conv_w"), conv_b=inp.get("conv_b"), h0=inp.get("h0"),
                              conv_state_in=inp.get("conv_state_in"), z=inp.get("z"),
                              norm_w=inp.get("norm_w"), heads=heads,
                              threads=threads or os.cpu_count())


def oracle_output(res, cfg):
    """The oracle's final output in the GPU's layout [B, L, nh*P]."""
    if cfg["norm_groups"]:
        return res["out"]
    y = res["y"]
    return y.reshape(y.shape[0], y.shape[1], -1)
