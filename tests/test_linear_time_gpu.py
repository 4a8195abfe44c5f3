"""Linear time in the sequence length (the pages' claim for the Mamba-2 layer; hyper.ai summary
"NVIDIA Nemotron Nano 2", section "Method"): the tensor-core prefill at 8k, 32k and 128k tokens
of the 8k layer's width, timed with CUDA events, costs the same per token within a factor of
two (the chunked scan does the same work per chunk whatever the length; a quadratic term would
grow the per-token cost 16-fold between 8k and 128k)."""
import statistics

import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen

pytestmark = pytest.mark.gpu


def _time_prefill(ssd, torch, L, reps=5):
    cfg = dict(datagen.config(1), batch=1, seqlen=L)
    H, P, G, N, W = cfg["nheads"], cfg["headdim"], cfg["ngroups"], cfg["dstate"], cfg["conv_width"]
    conv_dim = H * P + 2 * G * N
    g = torch.Generator(device="cuda").manual_seed(datagen.SEED_BASE + L)
    xBC = torch.randn((1, L, conv_dim), generator=g, device="cuda").to(torch.bfloat16)
    dt = torch.randn((1, L, H), generator=g, device="cuda").to(torch.bfloat16)
    A = -torch.rand((H,), generator=g, device="cuda") * 8 - 0.5
    D = torch.rand((H,), generator=g, device="cuda")
    dt_bias = torch.rand((H,), generator=g, device="cuda") * 0.1 - 3.0
    conv_w = (torch.randn((conv_dim, W), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    ws = ssd.alloc_workspace(ssd.workspace_size(cfg))

    def run():
        ssd.prefill(cfg, xBC, dt, A, D, dt_bias, conv_w, None, None, None, workspace=ws)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    assert ssd.get_device_error() == 0
    return statistics.median(ms)


def test_prefill_time_is_linear_in_length(cuda_lib):
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    per_tok = {L: _time_prefill(ssd, torch, L) / L for L in (8192, 32768, 131072)}
    print("[linear] ns per token: " + ", ".join(f"{L}: {1e6 * t:.1f}" for L, t in per_tok.items()))
    base = per_tok[8192]
    for L, t in per_tok.items():
        assert 0.5 * base <= t <= 2.0 * base, f"L={L}: {1e6 * t:.1f} ns/token against {1e6 * base:.1f} at 8k"
