"""Seeded synthetic inputs for the five workloads of the Mamba-2 scan.

This module only draws random numbers and rounds them to the storage type
(bf16 by round-to-nearest-even); it holds none of the method's arithmetic.
Both the CUDA path (tests, benchmark) and the fp64 oracle take their inputs
from here.

Workloads (shapes are those of the Nemotron Nano 2 Mamba-2 layers: 8 groups,
state 128, head dim 64, conv window 4, d_model 5120 at the 12B width):

  0 tiny fp32 scan      B1 L256    H8   G1 Q64,  no conv, no gate
  1 prefill             B1 L8192   H128 G8 Q128, conv+SiLU, output + final state
  2 decode              B64        H128 G8, 16384 single-token steps, gated RMSNorm
  3 long-context        B1 L131072 (4 x 32768 with carry) H128 G8 Q256, conv + gated RMSNorm
  4 mixer layer         B8 L8192 d_model 5120, H160 G8 Q128, in/out projections

Distributions:
  x|B|C raw channels ~ N(0, 1) (config 0: B and C then scaled by 1/sqrt(128));
  dt_raw ~ N(0, 1); dt_bias_h = softplus^-1(dt0_h) with dt0_h ~ LogUniform[1e-3, 1e-1];
  the effective step is clamped to [1e-3, 1e-1];
  A_h = -exp(U(log 1, log 16)); D_h ~ U(0, 1); conv weights ~ N(0, 0.5^2); no conv bias;
  z ~ N(0, 1); norm weights 1; hidden ~ N(0, 1); W_in, W_out ~ N(0, 0.02^2).

Every tensor has its own PCG64 stream per block of 2^22 elements, keyed by
(20260 + workload index, tensor index, block index), so values do not depend on
how many threads draw them.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SEED_BASE = 20260
BLOCK = 1 << 22
# fixed tensor order: each name's index keys its random stream
TENSORS = ("xBC", "dt", "z", "conv_w", "A", "D", "dt_bias", "hidden", "W_in", "W_out", "h0",
           "conv_state", "decode_pool")


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns to float32 values (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tensor: str, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [seed, TENSORS.index(tensor), block])))


def normal(seed: int, tensor: str, shape, std: float = 1.0, bf16: bool = True,
           threads: int | None = None) -> np.ndarray:
    """N(0, std^2) draws of the given shape; bf16 bit patterns (uint16) or float32."""
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16 if bf16 else np.float32)
    nblk = max(1, math.ceil(n / BLOCK))

    def work(k):
        lo, hi = k * BLOCK, min(n, (k + 1) * BLOCK)
        v = _rng(seed, tensor, k).standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[lo:hi] = bf16_bits(v) if bf16 else v

    if nblk == 1:
        work(0)
    else:
        with ThreadPoolExecutor(threads or min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(nblk)))
    return out.reshape(shape)


def head_params(seed: int, H: int) -> dict:
    """A, D, dt_bias (float32, [H]) with the distributions stated in the module docstring."""
    A = -np.exp(_rng(seed, "A").uniform(math.log(1.0), math.log(16.0), H)).astype(np.float32)
    D = _rng(seed, "D").uniform(0.0, 1.0, H).astype(np.float32)
    dt0 = np.exp(_rng(seed, "dt_bias").uniform(math.log(1e-3), math.log(1e-1), H))
    # inverse of softplus, so that softplus(dt_bias) = dt0 (parameter initialisation)
    dt_bias = (dt0 + np.log(-np.expm1(-dt0))).astype(np.float32)
    return {"A": A, "D": D, "dt_bias": dt_bias}


def config(idx: int) -> dict:
    """Shape/numeric parameters of workload idx (see the module docstring)."""
    base = dict(headdim=64, dstate=128, conv_width=4, dt_softplus=True, dt_min=1e-3, dt_max=1e-1,
                norm_eps=1e-5, norm_groups=0, dtype="bf16")
    if idx == 0:
        return dict(base, name="tiny_fp32_scan", batch=1, seqlen=256, nheads=8, ngroups=1, chunk=64,
                    conv_width=0, dtype="f32")
    if idx == 1:
        return dict(base, name="prefill_8k", batch=1, seqlen=8192, nheads=128, ngroups=8, chunk=128)
    if idx == 2:
        return dict(base, name="decode_16k_steps", batch=64, seqlen=1, nheads=128, ngroups=8,
                    chunk=128, norm_groups=8, steps=16384, prefill_len=8192)
    if idx == 3:
        return dict(base, name="long_context_128k", batch=1, seqlen=131072, nheads=128, ngroups=8,
                    chunk=256, norm_groups=8, segments=4)
    if idx == 4:
        return dict(base, name="mixer_12b_width", batch=8, seqlen=8192, nheads=160, ngroups=8,
                    chunk=128, norm_groups=8, d_model=5120, rms_eps=1e-5)
    raise ValueError(idx)


def conv_dim(cfg: dict) -> int:
    return cfg["nheads"] * cfg["headdim"] + 2 * cfg["ngroups"] * cfg["dstate"]


def make_inputs(idx: int, cfg: dict | None = None, seqlen: int | None = None) -> dict:
    """Host (numpy) inputs of workload idx.  bf16 tensors are uint16 bit patterns.

    ``cfg`` may override shapes (smaller test cases drawn from the same distributions);
    ``seqlen`` overrides the sequence length only.
    """
    cfg = dict(config(idx) if cfg is None else cfg)
    if seqlen is not None:
        cfg["seqlen"] = seqlen
    seed = SEED_BASE + idx
    Bn, L, H, P, N, G = (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                         cfg["ngroups"])
    d_inner, cd = H * P, conv_dim(cfg)
    bf = cfg["dtype"] == "bf16"
    out = {"cfg": cfg}
    out.update(head_params(seed, H))
    if idx == 4:
        out["hidden"] = normal(seed, "hidden", (Bn, L, cfg["d_model"]))
        proj = 2 * d_inner + 2 * G * N + H
        out["W_in"] = normal(seed, "W_in", (proj, cfg["d_model"]), std=0.02)
        out["W_out"] = normal(seed, "W_out", (cfg["d_model"], d_inner), std=0.02)
        out["rms_w"] = bf16_bits(np.ones(cfg["d_model"], np.float32))
    else:
        xBC = normal(seed, "xBC", (Bn, L, cd), bf16=bf)
        if idx == 0:  # B and C scaled by 1/sqrt(N) (raw draws, no conv)
            xBC = xBC.astype(np.float32)
            xBC[..., d_inner:] *= np.float32(1.0 / math.sqrt(N))
        out["xBC"] = xBC
        out["dt"] = normal(seed, "dt", (Bn, L, H), bf16=bf)
        if cfg["norm_groups"]:
            out["z"] = normal(seed, "z", (Bn, L, d_inner), bf16=bf)
    if cfg["conv_width"]:
        out["conv_w"] = normal(seed, "conv_w", (cd, cfg["conv_width"]), std=0.5, bf16=bf)
    if cfg["norm_groups"]:
        out["norm_w"] = bf16_bits(np.ones(d_inner, np.float32)) if bf else np.ones(d_inner, np.float32)
    return out


def decode_pool(cfg: dict, pool: int = 64, seed_idx: int = 2) -> dict:
    """Per-step decode inputs: ``pool`` distinct token draws [pool, B, ...]; step s uses
    entry s % pool.  xBC_t [pool, B, conv_dim], dt_t [pool, B, H], z_t [pool, B, d_inner]."""
    seed = SEED_BASE + seed_idx
    Bn, H = cfg["batch"], cfg["nheads"]
    d_inner, cd = H * cfg["headdim"], conv_dim(cfg)
    flat = normal(seed, "decode_pool", (pool, Bn, cd + H + d_inner))
    return {"xBC": np.ascontiguousarray(flat[..., :cd]),
            "dt": np.ascontiguousarray(flat[..., cd:cd + H]),
            "z": np.ascontiguousarray(flat[..., cd + H:])}


def random_state(seed: int, shape, std: float = 0.1) -> np.ndarray:
    """A float32 initial SSM state (for the tests of the h0 path)."""
    return normal(seed, "h0", shape, std=std, bf16=False)


def random_conv_state(seed: int, shape, bf16: bool = True) -> np.ndarray:
    """A conv cache [B, W, conv_dim] of raw inputs (for the tests of the carry path)."""
    return normal(seed, "conv_state", shape, bf16=bf16)
