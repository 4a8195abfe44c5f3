"""Sequence-parallel prefill on CPU: the exchange logic of `seqpar.seqpar_prefill` with gloo
ranks, the compute steps supplied by the oracle.

Each rank holds one span of a sequence (spans of unequal length) plus the previous span's last
W raw rows as its conv halo.  The span states and decays are all-gathered, every rank forms the
state entering its span, and runs its span from there.  The spans' outputs, concatenated, and
the final state must equal the oracle's single pass over the whole sequence.  What this checks
is the host side: the rank-to-span order of the gather, the prefix indexing, the halo and the
last rank's conv cache.  The kernels behind the same three steps are checked on the GPU
(tests/test_seqpar_gpu.py)."""
import os
import socket

import numpy as np
import pytest

from mamba_ssd_scan_02_b200 import datagen


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(lens):
    cfg = dict(datagen.config(1), batch=2, seqlen=int(sum(lens)), nheads=4, ngroups=2,
               norm_groups=2)
    inp = datagen.make_inputs(5, cfg)
    seed = datagen.SEED_BASE + 321
    H, P, N = cfg["nheads"], cfg["headdim"], cfg["dstate"]
    inp["z"] = datagen.normal(seed, "z", (cfg["batch"], cfg["seqlen"], H * P))
    inp["h0"] = datagen.random_state(seed, (cfg["batch"], H, P, N))
    inp["conv_state_in"] = datagen.random_conv_state(seed, (cfg["batch"], 4, datagen.conv_dim(cfg)))
    return cfg, inp


class OracleOps:
    """The three compute steps from the oracle (fp64), on torch CPU tensors."""

    def __init__(self, oracle, inp):
        self.o, self.inp = oracle, inp

    def _run(self, cfg, xBC, dt, h0, halo, z=None, norm=False, conv_b=True):
        import torch
        c = dict(cfg, batch=xBC.shape[0], seqlen=xBC.shape[1])
        if not norm:
            c["norm_groups"] = 0
        return self.o.ssd_prefill(c, xBC, dt, self.inp["A"], self.inp["D"], self.inp["dt_bias"],
                                  conv_w=self.inp["conv_w"],
                                  conv_b=self.inp.get("conv_b") if conv_b else None,
                                  h0=None if h0 is None else (h0.numpy() if isinstance(h0, torch.Tensor) else h0),
                                  conv_state_in=halo, z=z, norm_w=self.inp.get("norm_w"))

    def span_state(self, cfg, xBC, dt, A, dt_bias, conv_w, conv_b, halo):
        import torch
        s = self._run(cfg, xBC, dt, None, halo)["h_final"]
        # the span's total decay, from the same recurrence: no input (raw x and its halo zeroed,
        # no conv bias, so SiLU(conv) = 0) and a state of ones
        x0 = xBC.copy()
        H, P = cfg["nheads"], cfg["headdim"]
        x0[..., :H * P] = 0
        h0 = None if halo is None else halo.copy()
        if h0 is not None:
            h0[..., :H * P] = 0
        ones = np.ones((xBC.shape[0], H, P, cfg["dstate"]))
        lam = self._run(cfg, x0, dt, ones, h0, conv_b=False)["h_final"][:, :, 0, 0]
        return torch.from_numpy(s), torch.from_numpy(np.ascontiguousarray(lam))

    def span_prefix(self, states, decays, h0):
        import torch
        S = states.shape[0]
        h = np.zeros(states.shape[1:]) if h0 is None else np.asarray(h0, np.float64)
        h_in = np.empty(states.shape)
        for k in range(S):
            h_in[k] = h
            h = decays[k].numpy()[:, :, None, None] * h + states[k].numpy()
        return torch.from_numpy(h_in), torch.from_numpy(h)

    def prefill(self, cfg, xBC, dt, A, D, dt_bias, conv_w, conv_b, z, norm_w, h_in, halo, last):
        r = self._run(cfg, xBC, dt, h_in, halo, z=z, norm=True)
        return r["out"], r.get("conv_state_out") if last else None


def _rank_main(rank, world, port, lens, errs):
    import torch
    import torch.distributed as dist
    import oracle as oracle_mod
    from mamba_ssd_scan_02_b200 import seqpar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = oracle_mod.get()
        cfg, inp = _case(lens)
        cu = np.concatenate([[0], np.cumsum(lens)])
        t0, t1 = int(cu[rank]), int(cu[rank + 1])
        W = cfg["conv_width"]
        raw = inp["xBC"][:, :, :datagen.conv_dim(cfg)]
        # this rank's conv halo: the last W raw rows before its span (the sequence's cache first)
        halo = o.conv_state_after(raw[:, :t0], inp["conv_state_in"], W)
        sl = slice(t0, t1)
        ops = OracleOps(o, inp)
        y, hf, cso = seqpar.seqpar_prefill(
            cfg, np.ascontiguousarray(inp["xBC"][:, sl]), np.ascontiguousarray(inp["dt"][:, sl]),
            inp["A"], inp["D"], inp["dt_bias"], inp["conv_w"], inp.get("conv_b"),
            np.ascontiguousarray(inp["z"][:, sl]), inp.get("norm_w"), inp["h0"], halo, ops=ops)
        full = o.ssd_prefill(cfg, inp["xBC"], inp["dt"], inp["A"], inp["D"], inp["dt_bias"],
                             conv_w=inp["conv_w"], conv_b=inp.get("conv_b"), h0=inp["h0"],
                             conv_state_in=inp["conv_state_in"], z=inp["z"], norm_w=inp.get("norm_w"))
        want_y = full["out"][:, sl]
        ry = np.max(np.abs(y - want_y)) / np.sqrt(np.mean(want_y ** 2))
        hfw = full["h_final"]
        rh = np.max(np.abs(hf.numpy() - hfw)) / np.sqrt(np.mean(hfw ** 2))
        msgs = []
        if not ry < 1e-9:
            msgs.append(f"rank {rank}: y rel err {ry:.3e}")
        if not rh < 1e-9:
            msgs.append(f"rank {rank}: h_final rel err {rh:.3e}")
        if rank == world - 1 and not np.array_equal(cso, full["conv_state_out"]):
            msgs.append(f"rank {rank}: conv cache differs")
        if rank < world - 1 and cso is not None:
            msgs.append(f"rank {rank}: only the last rank returns the conv cache")
        errs[rank] = msgs
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [(150, 183), (64, 1, 200)])
def test_gloo_ranks_reproduce_the_single_pass(lens):
    import torch.multiprocessing as mp
    world = len(lens)
    with mp.Manager() as mgr:
        errs = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), lens, errs), nprocs=world, join=True)
        res = dict(errs)
    assert sorted(res) == list(range(world))
    assert all(not m for m in res.values()), res
