"""GPU parity of the sequence-parallel steps (through the C ABI) against the fp64 oracle.

ssd_prefill_span_state is checked against the oracle's state from a zero state over the span
and the span's total decay (the oracle's own recurrence with no input and a state of ones);
ssd_span_prefix against the span recurrence written out; and the whole scheme, with the spans
of one sequence run one after another on one GPU (what each rank would run; the all-gather is
then a stack), against the oracle's single pass over the sequence."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, assert_close, dev, host, make_case, oracle_output, rel_err,
                            run_oracle_prefill, small_cfg, tol_for)

pytestmark = pytest.mark.gpu

KERNELS = [pytest.param(1, id="simt"), pytest.param(2, id="tc")]


def _oracle_span(oracle, cfg, inp, sl, halo):
    """The oracle's (state from zero, total decay) over tokens `sl` with conv history `halo`."""
    H, P = cfg["nheads"], cfg["headdim"]
    c = dict(cfg, seqlen=sl.stop - sl.start, norm_groups=0)
    xs, ds = np.ascontiguousarray(inp["xBC"][:, sl]), np.ascontiguousarray(inp["dt"][:, sl])
    s = oracle.ssd_prefill(c, xs, ds, inp["A"], inp["D"], inp["dt_bias"], conv_w=inp.get("conv_w"),
                           conv_b=inp.get("conv_b"), conv_state_in=halo)["h_final"]
    x0 = xs.copy()
    x0[..., :H * P] = 0
    h0 = None if halo is None else halo.copy()
    if h0 is not None:
        h0[..., :H * P] = 0
    ones = np.ones((xs.shape[0], H, P, cfg["dstate"]))
    lam = oracle.ssd_prefill(c, x0, ds, inp["A"], inp["D"], inp["dt_bias"], conv_w=inp.get("conv_w"),
                             h0=ones, conv_state_in=h0)["h_final"][:, :, 0, 0]
    return s, lam


def _halo(oracle, cfg, inp, t0):
    raw = inp["xBC"][:, :, :datagen.conv_dim(cfg)]
    return oracle.conv_state_after(raw[:, :t0], inp.get("conv_state_in"), cfg["conv_width"])


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("t0,t1,nseg", [(0, 333, 0), (100, 333, 0), (37, 1200, 3), (5, 5, 0)])
def test_span_state_matches_the_oracle(cuda_lib, oracle, kernel, t0, t1, nseg):
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=1200, n_segments=nseg)
    if kernel == 1:
        cfg = dict(cfg, dtype="bf16")
    inp = make_case(cfg)
    sl = slice(t0, t1)
    halo = _halo(oracle, cfg, inp, t0)
    c = dict(cfg, seqlen=t1 - t0)
    s, lam = ssd.prefill_span_state(c, dev(np.ascontiguousarray(inp["xBC"][:, sl])),
                                    dev(np.ascontiguousarray(inp["dt"][:, sl])), dev(inp["A"]),
                                    dev(inp["dt_bias"]), dev(inp["conv_w"]), dev(inp.get("conv_b")),
                                    dev(halo), kernel=kernel)
    if t1 == t0:
        assert np.all(host(s) == 0) and np.all(host(lam) == 1)
        return
    ws, wl = _oracle_span(oracle, cfg, inp, sl, halo)
    assert_close(host(s), ws, tol_for(cfg), f"span state [{t0},{t1})")
    # the decay is exp of a sum over the span: compare its logarithm, relative to that sum
    gl = host(lam).astype(np.float64)
    live = wl > 1e-30
    assert np.all(gl[~live] < 1e-29)
    lg, lw = np.log(gl[live]), np.log(wl[live])
    bad = np.abs(lg - lw) > 2e-6 * np.maximum(1.0, np.abs(lw))
    assert not bad.any(), f"span decay [{t0},{t1}): log error {np.max(np.abs(lg - lw)):.3e}"


def test_span_prefix_is_the_span_recurrence(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    rng = np.random.default_rng(11)
    S, Bn, H, P, N = 5, 2, 3, 64, 128
    st = rng.standard_normal((S, Bn, H, P, N)).astype(np.float32)
    de = rng.uniform(0.2, 1.0, (S, Bn, H)).astype(np.float32)
    h0 = rng.standard_normal((Bn, H, P, N)).astype(np.float32)
    want_in = np.empty((S, Bn, H, P, N))
    h = h0.astype(np.float64)
    for k in range(S):
        want_in[k] = h
        h = de[k].astype(np.float64)[:, :, None, None] * h + st[k]
    ds, dd, dh0 = (torch.from_numpy(a).cuda() for a in (st, de, h0))
    h_in, hf = ssd.span_prefix(ds, dd, dh0)
    assert rel_err(host(h_in), want_in) <= 1e-6 and rel_err(host(hf), h) <= 1e-6
    # in place, and without h0 (zero)
    _, hf0 = ssd.span_prefix(ds, dd, None, h_in=ds)
    want0 = np.zeros_like(h)
    for k in range(S):
        want0 = de[k].astype(np.float64)[:, :, None, None] * want0 + st[k]
    assert rel_err(host(hf0), want0) <= 1e-6
    assert rel_err(host(ds)[0], np.zeros_like(h)) == 0.0  # h_in[0] = zero state, in place
    with pytest.raises(ssd.SsdError):
        ssd.span_prefix(dd.new_empty((S, Bn, H, P, N)), dd, None, want_h_in=False, want_h_final=False)


def _run_spans(ssd, cfg, inp, cuts, oracle, kernel=None, with_norm=True):
    """Every span's (state, decay), stacked as the all-gather would leave them; the prefix; then
    each span's prefill from its h_in.  Returns (y of all spans, prefix h_final, last cache)."""
    import torch
    halos, states, decays = [], [], []
    for t0, t1 in zip(cuts[:-1], cuts[1:]):
        sl = slice(t0, t1)
        halo = _halo(oracle, cfg, inp, t0)
        halos.append(halo)
        s, lam = ssd.prefill_span_state(dict(cfg, seqlen=t1 - t0), dev(np.ascontiguousarray(inp["xBC"][:, sl])),
                                        dev(np.ascontiguousarray(inp["dt"][:, sl])), dev(inp["A"]),
                                        dev(inp["dt_bias"]), dev(inp["conv_w"]), dev(inp.get("conv_b")),
                                        dev(halo), kernel=kernel)
        states.append(s)
        decays.append(lam)
    h_in, hf = ssd.span_prefix(torch.stack(states), torch.stack(decays), dev(inp.get("h0")))
    ys, cso = [], None
    for k, (t0, t1) in enumerate(zip(cuts[:-1], cuts[1:])):
        sl = slice(t0, t1)
        z = dev(np.ascontiguousarray(inp["z"][:, sl])) if with_norm else None
        y, _, c = ssd.prefill(dict(cfg, seqlen=t1 - t0), dev(np.ascontiguousarray(inp["xBC"][:, sl])),
                              dev(np.ascontiguousarray(inp["dt"][:, sl])), dev(inp["A"]), dev(inp["D"]),
                              dev(inp["dt_bias"]), dev(inp["conv_w"]), dev(inp.get("conv_b")), z,
                              dev(inp.get("norm_w")) if with_norm else None, h_in[k].contiguous(),
                              dev(halos[k]), kernel=kernel)
        ys.append(y.float().cpu().numpy())
        cso = c
    return np.concatenate(ys, axis=1), hf, cso


@pytest.mark.parametrize("kernel", KERNELS)
def test_spans_on_one_gpu_reproduce_the_single_pass(cuda_lib, oracle, kernel):
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=900)
    inp = make_case(cfg)
    cuts = [0, 129, 130, 511, 900]  # unequal spans, one of a single token
    y, hf, cso = _run_spans(ssd, cfg, inp, cuts, oracle, kernel=kernel)
    ref = run_oracle_prefill(oracle, cfg, inp)
    assert_close(y, oracle_output(ref, cfg), tol_for(cfg), "spans y", out_dtype="bf16")
    assert_close(host(hf), ref["h_final"], tol_for(cfg), "spans h_final")
    assert np.array_equal(host(cso), ref["conv_state_out"])


def test_long_context_as_four_spans(cuda_lib, oracle):
    """Workload 3 (131072 tokens, gated norm) as four 32768-token spans, each started from the
    prefix of the gathered span states, against the oracle's single pass on the heads of
    group 0 (heads and groups are independent)."""
    from mamba_ssd_scan_02_b200 import ssd
    cfg = datagen.config(3)
    inp = datagen.make_inputs(3)
    L, S = cfg["seqlen"], cfg["seqlen"] // cfg["segments"]
    cuts = [k * S for k in range(cfg["segments"] + 1)]
    y, hf, cso = _run_spans(ssd, cfg, inp, cuts, oracle)
    ref = run_oracle_prefill(oracle, cfg, inp, heads=(0, 16))
    P = cfg["headdim"]
    assert_close(y[:, :, :16 * P], ref["out"], TOL_BF16, "cfg3 spans y group 0", out_dtype="bf16")
    assert_close(host(hf)[:, :16], ref["h_final"], TOL_BF16, "cfg3 spans h_final group 0")
    assert np.array_equal(host(cso), ref["conv_state_out"])
