"""GPU parity of ssd_prefill (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, host, make_case, oracle_output,
                            rel_err, run_gpu_prefill, run_oracle_prefill, small_cfg, tol_for)

pytestmark = pytest.mark.gpu

# 1 = CUDA-core scan, 2 = tcgen05 tensor-core scan (bf16 only)
KERNELS = [pytest.param(1, id="simt"), pytest.param(2, id="tc")]


def _check(oracle, cfg, inp, kernel, heads=None, check_cache=True, tag=""):
    y, hf, cso = run_gpu_prefill(cfg, inp, kernel=kernel)
    ref = run_oracle_prefill(oracle, cfg, inp, heads=heads)
    lo, hi = heads or (0, cfg["nheads"])
    P = cfg["headdim"]
    tol = tol_for(cfg)
    e1 = assert_close(y.float().cpu().numpy()[:, :, lo * P:hi * P], oracle_output(ref, cfg), tol,
                      f"{tag} y", out_dtype=cfg["dtype"])
    e2 = assert_close(host(hf)[:, lo:hi], ref["h_final"], tol, f"{tag} h_final")
    if check_cache and cfg["conv_width"]:
        assert np.array_equal(host(cso), ref["conv_state_out"]), f"{tag} conv_state_out not bit-exact"
    return e1, e2


def test_tiny_fp32_scan(cuda_lib, oracle):
    """Workload 0 at full size: fp32, no conv, no gate, zero initial state (1e-4 * RMS)."""
    cfg = datagen.config(0)
    inp = datagen.make_inputs(0)
    _check(oracle, cfg, inp, kernel=1, tag="cfg0")


@pytest.mark.parametrize("kernel", KERNELS)
def test_bf16_all_options(cuda_lib, oracle, kernel):
    """conv bias, incoming state and conv cache, z-gated norm, ragged last chunk."""
    cfg = small_cfg()
    _check(oracle, cfg, make_case(cfg), kernel, tag="small")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunk_sizes(cuda_lib, oracle, kernel, chunk):
    cfg = small_cfg(chunk=chunk, seqlen=517, batch=1, norm_groups=0)
    _check(oracle, cfg, make_case(cfg, with_bias=False), kernel, tag=f"Q{chunk}")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("nseg", [2, 3, 5])
def test_internal_segments(cuda_lib, oracle, kernel, nseg):
    """The segmented scan (local states, inter-segment pass, output pass) matches."""
    cfg = small_cfg(seqlen=1200, n_segments=nseg)
    _check(oracle, cfg, make_case(cfg), kernel, tag=f"seg{nseg}")


def test_fp32_with_conv_and_norm(cuda_lib, oracle):
    cfg = small_cfg(dtype="f32", seqlen=190, norm_groups=4)
    _check(oracle, cfg, make_case(cfg), 1, tag="f32 conv+norm")


@pytest.mark.parametrize("kernel", KERNELS)
def test_full_width_norm_group(cuda_lib, oracle, kernel):
    cfg = small_cfg(norm_groups=1, seqlen=150)
    _check(oracle, cfg, make_case(cfg), kernel, tag="norm_groups=1")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("L", [1, 2, 3, 5])
def test_short_sequences(cuda_lib, oracle, kernel, L):
    """Fewer tokens than the conv window: history comes from the incoming cache."""
    cfg = small_cfg(seqlen=L)
    _check(oracle, cfg, make_case(cfg), kernel, tag=f"L={L}")


@pytest.mark.parametrize("L,W", [(1, 4), (100, 4), (129, 1), (256, 4), (200, 0)])
def test_tail_covered_final_state_is_fp32_accurate(cuda_lib, oracle, L, W):
    """With at most two 128-token chunks, the tensor path's final state comes from the tail
    pass alone: the scan leaves h0 unchanged in fp32 and the fold adds what the tail computes
    from the raw inputs (the fp32 conv + SiLU, then three fp16 products of hi/lo parts,
    |v - hi - lo| <= 2^-22 |v|).  So it must meet the fp32 bound against the fp64 oracle, far
    inside the bf16 one that the scan's fp16 products need."""
    cfg = small_cfg(seqlen=L, conv_width=W, norm_groups=0)
    inp = make_case(cfg, seed_idx=9)
    _, hf, _ = run_gpu_prefill(cfg, inp, kernel=2)
    ref = run_oracle_prefill(oracle, cfg, inp)
    r = rel_err(host(hf), ref["h_final"])
    print(f"[parity] tail-only h_final L={L} W={W}: max|err|/RMS = {r:.3e} (bound {TOL_F32:.1e})")
    assert r <= TOL_F32, f"L={L} W={W}: tail-only h_final max|err|/RMS = {r:.3e} > {TOL_F32:.1e}"


def test_tail_after_the_scan_when_no_sms_are_free(cuda_lib, oracle):
    """A uniform batch whose scan takes more CTAs than the GPU has SMs (3 rows x 64 heads): the
    tail pass runs after the scan and folds into h_final itself (no fold pass).  y and h_final
    meet the same bounds against the oracle as on the side-stream path."""
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(batch=3, nheads=64, ngroups=4, seqlen=300, norm_groups=4)
    inp = make_case(cfg, seed_idx=11)
    ssd.trace_enable(True)
    ssd.trace_read()
    try:
        e1, e2 = _check(oracle, cfg, inp, 2, tag="tail after the scan")
        names = [n for n, _ in ssd.trace_read()]
    finally:
        ssd.trace_enable(False)
    assert "ssd_state_tail" in names and "ssd_tail_fold" not in names, names


def test_tensor_kernel_rejects_fp32(cuda_lib):
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(dtype="f32", seqlen=64)
    with pytest.raises(ssd.SsdError) as ei:
        run_gpu_prefill(cfg, make_case(cfg), kernel=2)
    assert ei.value.status == 2


def test_seqlen_zero_carries_through(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=0)
    inp = make_case(small_cfg(seqlen=4))
    h0 = torch.from_numpy(inp["h0"]).cuda()
    csi = ssd.to_device(inp["conv_state_in"])
    xBC = torch.empty((2, 0, datagen.conv_dim(cfg)), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((2, 0, 16), dtype=torch.bfloat16, device="cuda")
    z = torch.empty((2, 0, 1024), dtype=torch.bfloat16, device="cuda")
    p = {k: ssd.to_device(inp[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    y, hf, cso = ssd.prefill(cfg, xBC, dt, p["A"], p["D"], p["dt_bias"], p["conv_w"], None, z, None,
                             h0, csi)
    torch.cuda.synchronize()
    assert torch.equal(hf, h0) and torch.equal(cso, csi)


@pytest.mark.parametrize("kernel", KERNELS)
def test_split_with_carry_equals_unsplit(cuda_lib, oracle, kernel):
    """Consecutive calls fed each other's final state and conv cache equal one call; the
    carried conv cache is bit-exact."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=700)
    inp = make_case(cfg)
    yfull, hfull, cfull = run_gpu_prefill(cfg, inp, kernel=kernel)
    for L1 in (1, 3, 130, 256):
        a = dict(inp, xBC=inp["xBC"][:, :L1], dt=inp["dt"][:, :L1], z=inp["z"][:, :L1])
        y1, h1, c1 = run_gpu_prefill(dict(cfg, seqlen=L1), a, kernel=kernel)
        b = dict(inp, xBC=np.ascontiguousarray(inp["xBC"][:, L1:]),
                 dt=np.ascontiguousarray(inp["dt"][:, L1:]), z=np.ascontiguousarray(inp["z"][:, L1:]),
                 h0=host(h1), conv_state_in=host(c1))
        y2, h2, c2 = run_gpu_prefill(dict(cfg, seqlen=700 - L1), b, kernel=kernel)
        ycat = torch.cat([y1, y2], dim=1).float().cpu().numpy()
        assert_close(ycat, yfull.float().cpu().numpy(), TOL_BF16, f"split at {L1}", out_dtype="bf16",
                     both_rounded=True)
        assert rel_err(host(h2), host(hfull)) <= TOL_BF16
        assert torch.equal(c2, cfull), f"conv cache differs after split at {L1}"
    ref = run_oracle_prefill(oracle, cfg, inp)
    assert_close(host(hfull), ref["h_final"], TOL_BF16, "h_final")
    assert_close(yfull.float().cpu().numpy(), ref["out"], TOL_BF16, "unsplit y", out_dtype="bf16")


def test_every_output_element_written(cuda_lib):
    """Outputs pre-filled with NaN come back finite everywhere (nothing left unwritten)."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    from tests.gpu_util import dev
    cfg = small_cfg(seqlen=259)
    inp = make_case(cfg)
    y = torch.full((2, 259, 1024), float("nan"), dtype=torch.bfloat16, device="cuda")
    hf = torch.full((2, 16, 64, 128), float("nan"), device="cuda")
    cso = torch.full((2, 4, datagen.conv_dim(cfg)), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = ssd.workspace_size(cfg)
    ws = torch.full((nbytes // 4,), float("nan"), device="cuda").view(torch.uint8)
    run_gpu_prefill(cfg, inp, y=y, h_final=hf, conv_state_out=cso, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all() and torch.isfinite(hf).all()
    assert torch.isfinite(cso.float()).all()


def test_prefill_8k_full_size(cuda_lib, oracle):
    """Workload 1 at full size (B1 L8192 H128 G8 Q128, conv+SiLU), all heads."""
    cfg = datagen.config(1)
    inp = datagen.make_inputs(1)
    _check(oracle, cfg, inp, kernel=None, tag="cfg1")


@pytest.mark.parametrize("nseg", [3])
def test_prefill_8k_full_size_internal_segments(cuda_lib, oracle, nseg):
    """Workload 1 at full size with the sequence forced into internal segments (state-only
    pass, inter-segment pass, output pass), all heads."""
    cfg = dict(datagen.config(1), n_segments=nseg)
    inp = datagen.make_inputs(1)
    _check(oracle, cfg, inp, kernel=None, tag=f"cfg1 seg{nseg}")


def test_long_context_split_equals_unsplit(cuda_lib, oracle):
    """Workload 3: 131072 tokens as 4 x 32768 with state + conv-cache carry equals one pass;
    the oracle checks the heads of groups 0 and 7 (heads and groups are independent)."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    from tests.gpu_util import dev
    cfg = datagen.config(3)
    inp = datagen.make_inputs(3)
    L, S = cfg["seqlen"], cfg["seqlen"] // cfg["segments"]
    full_y, full_h, full_c = run_gpu_prefill(cfg, inp)
    h, c = None, None
    ys = []
    for k in range(cfg["segments"]):
        sl = slice(k * S, (k + 1) * S)
        seg = dict(inp, xBC=np.ascontiguousarray(inp["xBC"][:, sl]),
                   dt=np.ascontiguousarray(inp["dt"][:, sl]), z=np.ascontiguousarray(inp["z"][:, sl]))
        y, hf, cso = ssd.prefill(dict(cfg, seqlen=S), dev(seg["xBC"]), dev(seg["dt"]), dev(seg["A"]),
                                 dev(seg["D"]), dev(seg["dt_bias"]), dev(seg["conv_w"]), None,
                                 dev(seg["z"]), dev(seg["norm_w"]), h, c)
        h, c = hf, cso
        ys.append(y.float().cpu().numpy())
    ysplit = np.concatenate(ys, axis=1)
    yfull = full_y.float().cpu().numpy()
    assert_close(ysplit, yfull, TOL_BF16, "cfg3 split vs unsplit", out_dtype="bf16",
                 both_rounded=True)
    assert rel_err(host(h), host(full_h)) <= TOL_BF16
    assert torch.equal(c, full_c)
    P = cfg["headdim"]
    for g in (0, 7):
        lo, hi = g * 16, (g + 1) * 16
        ref = run_oracle_prefill(oracle, cfg, inp, heads=(lo, hi))
        assert_close(ysplit[:, :, lo * P:hi * P], ref["out"], TOL_BF16, f"cfg3 split y group {g}",
                     out_dtype="bf16")
        assert_close(host(h)[:, lo:hi], ref["h_final"], TOL_BF16, f"cfg3 h_final group {g}")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("W", [0, 1, 2, 3])
def test_narrow_conv_windows(cuda_lib, oracle, kernel, W):
    """Conv windows below 4 (0 = no conv and no activation), with cache and gated norm."""
    cfg = small_cfg(conv_width=W, seqlen=261)
    _check(oracle, cfg, make_case(cfg, seed_idx=7), kernel, tag=f"W{W}")


def test_tc_prefill_graph_capture_and_reuse(cuda_lib):
    """The tensor-core prefill runs its fp32 final-state pass on a side stream forked from the
    caller's stream and joined before the fold.  Captured into a CUDA graph, the fork and join
    land in the graph, so replays reproduce the eager outputs bit for bit; and back-to-back
    calls with different inputs (the side stream and its events reused) each match their own
    single eager call."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    cfg = small_cfg(seqlen=333)
    names = ["xBC", "dt", "A", "D", "dt_bias", "conv_w", "conv_b", "z", "norm_w", "h0", "conv_state_in"]
    cases = [make_case(cfg, seed_idx=s) for s in (11, 12)]
    devs = [[(None if c.get(k) is None else ssd.to_device(c[k])) for k in names] for c in cases]
    torch.cuda.synchronize()
    eager = []
    for d in devs:
        y, hf, cso = ssd.prefill(cfg, *d, kernel=2)
        torch.cuda.synchronize()
        eager.append((y.clone(), hf.clone(), cso.clone()))
    # back to back on one stream, no synchronisation in between
    outs = [ssd.prefill(cfg, *d, kernel=2) for d in devs for _ in range(2)]
    torch.cuda.synchronize()
    for i, (y, hf, cso) in enumerate(outs):
        ye, he, ce = eager[i // 2]
        assert torch.equal(y, ye) and torch.equal(hf, he) and torch.equal(cso, ce), f"call {i}"
    # graph capture on a side stream, then replays
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ssd.prefill(cfg, *devs[0], kernel=2)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        yg, hg, cg = ssd.prefill(cfg, *devs[0], kernel=2)
    for _ in range(3):
        hg.zero_()
        yg.zero_()
        g.replay()
        torch.cuda.synchronize()
        ye, he, ce = eager[0]
        assert torch.equal(yg, ye) and torch.equal(hg, he) and torch.equal(cg, ce)
