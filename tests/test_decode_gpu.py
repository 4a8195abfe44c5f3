"""GPU parity of ssd_decode_step (through the C ABI) against the fp64 oracle."""
import os

import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, dev, host, make_case,
                            run_gpu_prefill, run_oracle_prefill, small_cfg)

pytestmark = pytest.mark.gpu


def _decode_cfg(**kw):
    c = dict(datagen.config(2), batch=3, nheads=16, ngroups=2, norm_groups=2)
    c.update(kw)
    return c


def _run_steps(oracle, cfg, steps, seed=3):
    """Random state and cache, then `steps` decode steps on GPU and in the oracle."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    Bn, H, P, N = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    bf = cfg["dtype"] == "bf16"
    pcfg = dict(cfg, seqlen=steps)
    inp = make_case(pcfg, seed_idx=seed)  # per-token draws reused as the decode inputs
    state = torch.from_numpy(inp["h0"]).cuda()
    cache = dev(inp["conv_state_in"])
    cache2 = torch.empty_like(cache)
    ost = inp["h0"].astype(np.float64)
    ocache = inp["conv_state_in"]
    p = {k: dev(inp.get(k)) for k in ("A", "D", "dt_bias", "conv_w", "conv_b", "norm_w")}
    worst = 0.0
    for t in range(steps):
        xt = np.ascontiguousarray(inp["xBC"][:, t]); dtt = np.ascontiguousarray(inp["dt"][:, t])
        zt = np.ascontiguousarray(inp["z"][:, t]) if cfg["norm_groups"] else None
        y = ssd.decode_step(cfg, dev(xt), dev(dtt), p["A"], p["D"], p["dt_bias"], p["conv_w"],
                            p["conv_b"], state, cache, cache2, dev(zt), p["norm_w"])
        r = oracle.decode_step(cfg, xt, dtt, inp["A"], inp["D"], inp["dt_bias"], inp["conv_w"],
                               inp["conv_b"], ocache, ost, z_t=zt, norm_w=inp.get("norm_w"))
        want = r["out"] if cfg["norm_groups"] else r["y"].reshape(Bn, -1)
        tol = TOL_BF16 if bf else TOL_F32
        worst = max(worst, assert_close(y.float().cpu().numpy(), want, tol, f"step {t} y",
                                        out_dtype=cfg["dtype"]))
        # the carried cache is the oracle's shifted cache, bit for bit
        ocache = np.ascontiguousarray(np.concatenate([ocache[:, 1:], xt[:, None]], axis=1))
        assert np.array_equal(host(cache2), ocache), f"conv cache, step {t}"
        cache, cache2 = cache2, cache
    assert_close(host(state), ost, TOL_BF16 if bf else TOL_F32, "state after steps")
    return worst


def test_decode_steps_bf16(cuda_lib, oracle):
    _run_steps(oracle, _decode_cfg(), steps=12)


def test_decode_steps_fp32(cuda_lib, oracle):
    _run_steps(oracle, _decode_cfg(dtype="f32", norm_groups=4), steps=6)


def test_decode_no_norm(cuda_lib, oracle):
    _run_steps(oracle, _decode_cfg(norm_groups=0, nheads=24, ngroups=3), steps=5)


def test_decode_equals_prefill(cuda_lib):
    """k decode steps after a prefill of L0 tokens equal the prefill of L0 + k tokens."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    L0, k = 200, 7
    cfg = small_cfg(seqlen=L0 + k)
    inp = make_case(cfg)
    yfull, hfull, cfull = run_gpu_prefill(cfg, inp)
    a = dict(inp, xBC=inp["xBC"][:, :L0], dt=inp["dt"][:, :L0], z=inp["z"][:, :L0])
    y0, state, cache = run_gpu_prefill(dict(cfg, seqlen=L0), a)
    cache2 = torch.empty_like(cache)
    p = {n: dev(inp[n]) for n in ("A", "D", "dt_bias", "conv_w", "conv_b", "norm_w")}
    for j in range(k):
        t = L0 + j
        y = ssd.decode_step(cfg, dev(np.ascontiguousarray(inp["xBC"][:, t])),
                            dev(np.ascontiguousarray(inp["dt"][:, t])), p["A"], p["D"], p["dt_bias"],
                            p["conv_w"], p["conv_b"], state, cache, cache2,
                            dev(np.ascontiguousarray(inp["z"][:, t])), p["norm_w"])
        cache, cache2 = cache2, cache
        ref = yfull[:, t].float().cpu().numpy()
        assert_close(y.float().cpu().numpy(), ref, TOL_BF16, f"decode step {j}", out_dtype="bf16",
                     both_rounded=True)
    assert_close(host(state), host(hfull), TOL_BF16, "state")
    assert torch.equal(cache, cfull)


def test_decode_16k_steps_full_size(cuda_lib, oracle):
    """Workload 2: B64 H128 G8, 16384 steps.
    (a) rows 0 and 63 for all 16384 steps (y compared every 16th step, the state and cache
        at the end), starting from an 8192-token prefill computed independently on the GPU
        (all 64 rows) and by the oracle (those two rows);
    (b) all 64 rows for the first 64 steps from a seeded random state and conv cache."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg = datagen.config(2)
    Bn, H, P, N = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    pcfg = dict(cfg, seqlen=cfg["prefill_len"], norm_groups=0)
    pin = datagen.make_inputs(2, pcfg)
    _, state, cache = run_gpu_prefill(pcfg, pin)
    rows = [0, Bn - 1]
    pre = run_oracle_prefill(oracle, dict(pcfg, batch=2),
                             dict(pin, xBC=np.ascontiguousarray(pin["xBC"][rows]),
                                  dt=np.ascontiguousarray(pin["dt"][rows])))
    assert_close(host(state)[rows], pre["h_final"], TOL_BF16, "post-prefill state")
    pool = datagen.decode_pool(cfg)
    npool = pool["xBC"].shape[0]
    par = {k: pin[k] for k in ("A", "D", "dt_bias", "conv_w")}
    norm_w = datagen.bf16_bits(np.ones(H * P, np.float32))
    dp = {k: dev(v) for k, v in par.items()}
    dnw = dev(norm_w)
    dpool = {k: dev(v) for k, v in pool.items()}

    # (b) all rows, first 64 steps, from a seeded state and cache
    seed = datagen.SEED_BASE + 202
    st_b = datagen.random_state(seed, (Bn, H, P, N), std=0.5)
    cache_b = datagen.random_conv_state(seed, (Bn, cfg["conv_width"], datagen.conv_dim(cfg)))
    gst, gc, gc2 = torch.from_numpy(st_b).cuda(), dev(cache_b), torch.empty_like(dev(cache_b))
    ost_b = st_b.astype(np.float64)
    oc_b = cache_b
    for s in range(64):
        i = s % npool
        y = ssd.decode_step(cfg, dpool["xBC"][i], dpool["dt"][i], dp["A"], dp["D"], dp["dt_bias"],
                            dp["conv_w"], None, gst, gc, gc2, dpool["z"][i], dnw)
        gc, gc2 = gc2, gc
        r = oracle.decode_step(cfg, pool["xBC"][i], pool["dt"][i], par["A"], par["D"],
                               par["dt_bias"], par["conv_w"], None, oc_b, ost_b, z_t=pool["z"][i],
                               norm_w=norm_w)
        oc_b = np.ascontiguousarray(np.concatenate([oc_b[:, 1:], pool["xBC"][i][:, None]], axis=1))
        assert np.array_equal(host(gc), oc_b), f"conv cache, step {s}"
        assert_close(y.float().cpu().numpy(), r["out"], TOL_BF16, f"all rows, step {s}",
                     out_dtype="bf16")
    assert_close(host(gst), ost_b, TOL_BF16, "state after 64 steps (all rows)")
    del gst, gc, gc2

    # (a) rows 0 and 63 for every step, from the two independently computed prefill states
    ost = pre["h_final"].copy()
    ocache = np.ascontiguousarray(pin["xBC"][rows][:, -cfg["conv_width"]:])
    assert np.array_equal(host(cache)[rows], ocache)
    cache2 = torch.empty_like(cache)
    steps = cfg["steps"]
    for s in range(steps):
        i = s % npool
        y = ssd.decode_step(cfg, dpool["xBC"][i], dpool["dt"][i], dp["A"], dp["D"], dp["dt_bias"],
                            dp["conv_w"], None, state, cache, cache2, dpool["z"][i], dnw)
        cache, cache2 = cache2, cache
        r = oracle.decode_step(dict(cfg, batch=2), np.ascontiguousarray(pool["xBC"][i][rows]),
                               np.ascontiguousarray(pool["dt"][i][rows]), par["A"], par["D"],
                               par["dt_bias"], par["conv_w"], None, ocache, ost,
                               z_t=np.ascontiguousarray(pool["z"][i][rows]), norm_w=norm_w)
        ocache = np.ascontiguousarray(
            np.concatenate([ocache[:, 1:], pool["xBC"][i][rows][:, None]], axis=1))
        if s % 16 == 15:
            assert_close(y.float().cpu().numpy()[rows], r["out"], TOL_BF16, f"rows 0/63, step {s}",
                         out_dtype="bf16")
    assert_close(host(state)[rows], ost, TOL_BF16, "state after 16384 steps")
    assert np.array_equal(host(cache)[rows], ocache)


@pytest.mark.parametrize("W", [2, 3])
def test_decode_narrow_conv_windows(cuda_lib, oracle, W):
    _run_steps(oracle, _decode_cfg(conv_width=W), steps=4)
