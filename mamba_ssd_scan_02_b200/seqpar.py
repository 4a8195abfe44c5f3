"""Sequence-parallel prefill: one span of a long sequence per rank, one exchange.

The scan's state recurrence is linear, so a sequence split into spans of consecutive tokens
(span k on rank k) needs one exchange.  Each rank scans its span from a zero state, giving
s_k and its total decay lambda_k = exp(sum over the span of dt*A) per (batch row, head); the
ranks all-gather (s_k, lambda_k); every rank forms the state entering its span,
h_in[k] = lambda_{k-1} h_in[k-1] + s_{k-1} with h_in[0] = h0, and runs the ordinary prefill on
its span from h_in[k].  The state after the last span is the sequence's final state.  The
pages fix the fp32 state this carries (neurohive.io article on Nemotron Nano 2, section
"Deployment and usage") and the 128k-token contexts that make the split worth having (the
English abstract on the shd-paper.top page).

The conv of a span's first W-1 tokens reads the previous span's last W raw rows.  Each rank is
given them as `halo` (a W-row overlap of its input, the way a sequence-parallel loader hands out
spans), so the exchange carries only the states and decays: n_spans * (B*H*P*N + B*H) floats.

This module is host orchestration only: the three compute steps are the library's kernels
(`ssd.prefill_span_state`, `ssd.span_prefix`, `ssd.prefill`) and the exchange is the process
group's all-gather (NCCL between GPUs).
"""
from __future__ import annotations


class LibraryOps:
    """The compute steps, as the library runs them on the GPU."""

    def __init__(self, workspace=None):
        self.workspace = workspace

    def span_state(self, cfg, xBC, dt, A, dt_bias, conv_w, conv_b, halo):
        from . import ssd
        return ssd.prefill_span_state(cfg, xBC, dt, A, dt_bias, conv_w, conv_b, halo,
                                      workspace=self.workspace)

    def span_prefix(self, states, decays, h0):
        from . import ssd
        return ssd.span_prefix(states, decays, h0)

    def prefill(self, cfg, xBC, dt, A, D, dt_bias, conv_w, conv_b, z, norm_w, h_in, halo, last):
        from . import ssd
        y, _, cso = ssd.prefill(cfg, xBC, dt, A, D, dt_bias, conv_w, conv_b, z, norm_w, h_in, halo,
                                workspace=self.workspace, want_state=last)
        return y, cso


def seqpar_prefill(cfg: dict, xBC, dt, A, D, dt_bias, conv_w=None, conv_b=None, z=None,
                   norm_w=None, h0=None, halo=None, *, group=None, ops=None):
    """Prefill of this rank's span of a sequence split across the ranks of `group`.

    xBC, dt, z: this rank's span ([B, L_span, ...]; spans may differ in length).  halo: the
    previous span's last W raw xBC rows as a conv cache [B, W, conv_dim] (on rank 0, the
    sequence's incoming conv cache, or None).  h0: the sequence's initial state, the same on
    every rank (None = zero).  Returns (y of the span, the sequence's final state, the
    sequence's outgoing conv cache on the last rank and None elsewhere)."""
    import torch
    import torch.distributed as dist
    ops = ops or LibraryOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    s_loc, d_loc = ops.span_state(cfg, xBC, dt, A, dt_bias, conv_w, conv_b, halo)
    # the one exchange (both gathers in flight together), into span-major buffers: gathered
    # along the batch axis and viewed as [world, B, ...] without a copy
    states = torch.empty((world * s_loc.shape[0],) + tuple(s_loc.shape[1:]), dtype=s_loc.dtype,
                         device=s_loc.device)
    decays = torch.empty((world * d_loc.shape[0],) + tuple(d_loc.shape[1:]), dtype=d_loc.dtype,
                         device=d_loc.device)
    w1 = dist.all_gather_into_tensor(states, s_loc.contiguous(), group=group, async_op=True)
    w2 = dist.all_gather_into_tensor(decays, d_loc.contiguous(), group=group, async_op=True)
    w1.wait()
    w2.wait()
    states = states.view((world,) + tuple(s_loc.shape))
    decays = decays.view((world,) + tuple(d_loc.shape))
    h_in, h_final = ops.span_prefix(states, decays, h0)
    y, cso = ops.prefill(cfg, xBC, dt, A, D, dt_bias, conv_w, conv_b, z, norm_w,
                         h_in[rank].contiguous(), halo, rank == world - 1)
    return y, h_final, (cso if rank == world - 1 else None)
