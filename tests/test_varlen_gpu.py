"""Variable-length batched prefill (ssd_prefill_varlen): packed sequences, each starting
from its own state and conv cache, against the fp64 oracle run on every sequence alone, and
against separate ssd_prefill calls (the same kernels on the same rows: bit-exact)."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, dev, host, oracle_output, rel_err,
                            run_oracle_prefill)

pytestmark = pytest.mark.gpu

LENS = [0, 1, 3, 127, 128, 129, 300, 517]


def _case():
    cfg = dict(datagen.config(1), batch=1, nheads=16, ngroups=2, norm_groups=2)
    cu = np.concatenate([[0], np.cumsum(LENS)]).astype(int)
    T, nseq = int(cu[-1]), len(LENS)
    inp = datagen.make_inputs(1, dict(cfg, seqlen=T))
    H, P, N, W = cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["conv_width"]
    cd = datagen.conv_dim(cfg)
    seed = datagen.SEED_BASE + 300
    inp["z"] = datagen.normal(seed, "z", (1, T, H * P))
    inp["h0"] = datagen.random_state(seed, (nseq, H, P, N))
    inp["conv_state_in"] = datagen.random_conv_state(seed, (nseq, W, cd))
    inp["norm_w"] = datagen.bf16_bits(np.random.default_rng(seed).uniform(0.5, 1.5, H * P).astype(np.float32))
    return cfg, cu, inp


def _gpu(cfg, cu, inp, **kw):
    from mamba_ssd_scan_02_b200 import ssd
    return ssd.prefill_varlen(cfg, cu, dev(inp["xBC"][0]), dev(inp["dt"][0]), dev(inp["A"]), dev(inp["D"]),
                              dev(inp["dt_bias"]), dev(inp["conv_w"]), None, dev(inp["z"][0]),
                              dev(inp["norm_w"]), dev(inp["h0"]), dev(inp["conv_state_in"]), **kw)


def test_varlen_without_final_states(cuda_lib):
    """Without final states the pass that computes their last chunks does not run (no
    ssd_state_tail launch), and y and the conv caches are bit-identical to the full call's."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg, cu, inp = _case()
    y, hf, cso = _gpu(cfg, cu, inp)
    ssd.trace_enable(True)
    ssd.trace_read()
    try:
        y2, hf2, cso2 = _gpu(cfg, cu, inp, want_state=False)
        names = [n for n, _ in ssd.trace_read()]
    finally:
        ssd.trace_enable(False)
    assert hf2 is None and "ssd_state_tail" not in names, names
    assert torch.equal(y, y2) and torch.equal(cso, cso2)


def test_varlen_matches_oracle_per_sequence(cuda_lib, oracle):
    cfg, cu, inp = _case()
    y, hf, cso = _gpu(cfg, cu, inp)
    y, hf, cso = y.float().cpu().numpy(), host(hf), host(cso)
    for i, L in enumerate(LENS):
        a, b = cu[i], cu[i + 1]
        sub = {k: inp[k] for k in ("A", "D", "dt_bias", "conv_w", "norm_w")}
        sub.update(xBC=inp["xBC"][:, a:b], dt=inp["dt"][:, a:b], z=inp["z"][:, a:b],
                   h0=inp["h0"][i:i + 1], conv_state_in=inp["conv_state_in"][i:i + 1], conv_b=None)
        scfg = dict(cfg, seqlen=L)
        if L:
            ref = run_oracle_prefill(oracle, scfg, sub)
            assert_close(y[a:b], oracle_output(ref, scfg)[0], TOL_BF16, f"seq {i} y", out_dtype="bf16")
            assert_close(hf[i], ref["h_final"][0], TOL_BF16, f"seq {i} h_final")
            if L <= 256:  # all of its state comes from the tail pass: the fp32 bound holds
                r = rel_err(hf[i], ref["h_final"][0])
                assert r <= TOL_F32, f"seq {i} (L={L}) tail-only h_final max|err|/RMS = {r:.3e}"
            assert np.array_equal(cso[i], ref["conv_state_out"][0]), f"seq {i} conv cache"
        else:  # empty: the carries pass through
            assert np.array_equal(hf[i], inp["h0"][i])
            assert np.array_equal(cso[i], inp["conv_state_in"][i])


def test_varlen_equals_separate_calls(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg, cu, inp = _case()
    y, hf, cso = _gpu(cfg, cu, inp)
    for i, L in enumerate(LENS):
        if not L:
            continue
        a, b = cu[i], cu[i + 1]
        yi, hi, ci = ssd.prefill(dict(cfg, seqlen=L), dev(inp["xBC"][:, a:b]), dev(inp["dt"][:, a:b]),
                                 dev(inp["A"]), dev(inp["D"]), dev(inp["dt_bias"]), dev(inp["conv_w"]), None,
                                 dev(inp["z"][:, a:b]), dev(inp["norm_w"]), dev(inp["h0"][i:i + 1]),
                                 dev(inp["conv_state_in"][i:i + 1]))
        assert torch.equal(yi[0], y[a:b]) and torch.equal(hi[0], hf[i]) and torch.equal(ci[0], cso[i])


def test_varlen_is_one_pass(cuda_lib):
    """On the tensor path the packed batch is one front end, one scan, one tail pass and one
    norm launch, whatever the number of sequences."""
    from mamba_ssd_scan_02_b200 import ssd
    cfg, cu, inp = _case()
    ssd.trace_enable(True)
    ssd.trace_read()
    try:
        _gpu(cfg, cu, inp)
        names = [n for n, _ in ssd.trace_read()]
    finally:
        ssd.trace_enable(False)
    for k in ("ssd_front", "ssd_scan_tc", "ssd_state_tail", "ssd_gated_norm"):
        assert names.count(k) == 1, names


def test_many_short_sequences_at_full_width(cuda_lib, oracle):
    """64 packed sequences of 1 to 700 tokens at the 8k layer's width (128 heads, 8 groups):
    bit-exact against one ssd_prefill call per sequence, and the oracle on three of them."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    rng = np.random.default_rng(datagen.SEED_BASE + 64)
    lens = rng.integers(1, 701, 64)
    lens[5], lens[17] = 1, 128
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    T, nseq = int(cu[-1]), len(lens)
    cfg = dict(datagen.config(1), batch=1, seqlen=T)
    inp = datagen.make_inputs(1, cfg)
    H, P, N, W = cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["conv_width"]
    seed = datagen.SEED_BASE + 301
    h0 = datagen.random_state(seed, (nseq, H, P, N))
    csi = datagen.random_conv_state(seed, (nseq, W, datagen.conv_dim(cfg)))
    d = {k: dev(inp[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    x, dtt = dev(inp["xBC"][0]), dev(inp["dt"][0])
    y, hf, cso = ssd.prefill_varlen(cfg, cu, x, dtt, d["A"], d["D"], d["dt_bias"], d["conv_w"], None,
                                    None, None, dev(h0), dev(csi))
    for i in range(nseq):
        a, b = int(cu[i]), int(cu[i + 1])
        yi, hi, ci = ssd.prefill(dict(cfg, seqlen=b - a), x[None, a:b], dtt[None, a:b], d["A"], d["D"],
                                 d["dt_bias"], d["conv_w"], None, None, None, dev(h0[i:i + 1]),
                                 dev(csi[i:i + 1]))
        assert torch.equal(yi[0], y[a:b]), f"seq {i} y"
        assert torch.equal(hi[0], hf[i]) and torch.equal(ci[0], cso[i]), f"seq {i} carries"
    yh = y.float().cpu().numpy()
    for i in (0, 5, 40):
        a, b = int(cu[i]), int(cu[i + 1])
        sub = {k: inp[k] for k in ("A", "D", "dt_bias", "conv_w")}
        sub.update(xBC=inp["xBC"][:, a:b], dt=inp["dt"][:, a:b], h0=h0[i:i + 1],
                   conv_state_in=csi[i:i + 1], conv_b=None)
        scfg = dict(cfg, seqlen=b - a)
        ref = run_oracle_prefill(oracle, scfg, sub, heads=(0, 16))
        assert_close(yh[a:b, :16 * P], oracle_output(ref, scfg)[0], TOL_BF16, f"seq {i} y", out_dtype="bf16")
        assert_close(host(hf)[i, :16], ref["h_final"][0], TOL_BF16, f"seq {i} h_final")
