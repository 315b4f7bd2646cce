"""Sequence-parallel prefill across ranks, on CPU: two `gloo` ranks each hold
half of one sequence and run prefill_sequence_parallel (the product's
ordering of the steps and its one all-gather), with the compute steps
supplied by the fp64 oracle instead of the CUDA library.  Each rank's
outputs and the last rank's final state must equal the oracle's single pass
over the whole sequence: this pins the record layout, the rank order of the
gathered records, the composition and the hand-over of the initial state."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads as wl


class OracleOps:
    """The three compute steps of the sequence-parallel prefill, in fp64 on
    the CPU (the oracle's recurrence), on torch CPU tensors."""

    def empty(self, n, like):
        return torch.empty(n, dtype=torch.float64)

    def segment_record(self, seg, record, BH, F, dv, flags):
        per_feature = bool(flags & 2)
        nl = BH * F if per_feature else BH
        off_S = (nl + 3) // 4 * 4
        off_z = off_S + BH * F * dv
        np_ = {k: v.numpy() for k, v in seg.items() if isinstance(v, torch.Tensor)}
        _, S, z = oracle.scan_fwd(np_["q"], np_["k"], np_["v"], np_["W_q"], np_["W_k"], dt=np_["dt"],
                                  A_log=np_["A_log"], dt_scaled_input=bool(flags & 1), return_state=True)
        if per_feature:
            lam = oracle.log_decay_per_feature(np_["dt"], np_["A_log"]).sum(axis=1)   # [B, H, F]
        else:
            lam = oracle.log_decay(np_["dt"], np_["A_log"]).sum(axis=1)               # [B, H]
        record[:nl] = torch.from_numpy(lam.reshape(-1))
        record[off_S:off_z] = torch.from_numpy(S.reshape(-1))
        record[off_z:off_z + BH * F] = torch.from_numpy(z.reshape(-1))

    def start_state(self, gathered, n_parts, rank, BH, F, dv, flags, S0, z0, S_start, z_start):
        per_feature = bool(flags & 2)
        nl = BH * F if per_feature else BH
        n = (nl + 3) // 4 * 4 + BH * F * dv + BH * F
        off_S = (nl + 3) // 4 * 4
        S = np.zeros((BH, F, dv)) if S0 is None else S0.numpy().reshape(BH, F, dv).copy()
        z = np.zeros((BH, F)) if z0 is None else z0.numpy().reshape(BH, F).copy()
        g = gathered.numpy()
        for r in range(rank):
            rec = g[r * n:(r + 1) * n]
            lam = rec[:nl].reshape(BH, F) if per_feature else rec[:nl].reshape(BH, 1)
            S = np.exp(lam)[:, :, None] * S + rec[off_S:off_S + BH * F * dv].reshape(BH, F, dv)
            z = np.exp(lam) * z + rec[off_S + BH * F * dv:n].reshape(BH, F)
        S_start.copy_(torch.from_numpy(S.reshape(-1)))
        z_start.copy_(torch.from_numpy(z.reshape(-1)))

    def scan(self, seg, o, S0, z0, S_out, z_out, flags):
        np_ = {k: v.numpy() for k, v in seg.items() if isinstance(v, torch.Tensor)}
        res = oracle.scan_fwd(np_["q"], np_["k"], np_["v"], np_["W_q"], np_["W_k"], dt=np_["dt"],
                              A_log=np_["A_log"], S0=S0.numpy(), z0=z0.numpy(),
                              dt_scaled_input=bool(flags & 1), return_state=True)
        o.copy_(torch.from_numpy(res[0]))
        if S_out is not None:
            S_out.copy_(torch.from_numpy(res[1]))
            z_out.copy_(torch.from_numpy(res[2]))


def _inputs(flags):
    cfg = wl.TINY_F32
    L = 96
    inp = wl.scan_inputs(cfg, B=2, L=L, seed=91)
    inp["dt"] = wl.round_f32(wl.normal(91, "dt", (2, L, cfg.H)))
    if flags & 2:
        inp["A_log"] = wl.round_f32(wl.uniform(91, "A_log_f", (cfg.H, cfg.F), 0.0, 1.0))
    else:
        inp["A_log"] = wl.round_f32(wl.uniform(91, "A_log", (cfg.H,), 0.0, 1.0))
    S0 = np.abs(wl.normal(91, "S0", (2, cfg.H, cfg.F, cfg.dv), 0.1))
    z0 = np.abs(wl.normal(91, "z0", (2, cfg.H, cfg.F), 0.1)) + 0.01
    return cfg, inp, S0, z0


def _rank_main(rank, world, port, flags, out):
    import torch.distributed as dist
    from selective_ssm_sequence_b200 import sequence_parallel as sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, inp, S0, z0 = _inputs(flags)
        L = inp["q"].shape[1]
        t0, t1 = rank * L // world, (rank + 1) * L // world
        seg = {n: torch.from_numpy(np.ascontiguousarray(inp[n][:, t0:t1])) for n in ("q", "k", "v", "dt")}
        seg.update(W_q=torch.from_numpy(inp["W_q"]), W_k=torch.from_numpy(inp["W_k"]),
                   A_log=torch.from_numpy(inp["A_log"]))
        o = torch.empty(2, t1 - t0, cfg.H, cfg.dv, dtype=torch.float64)
        S_out = torch.empty(2, cfg.H, cfg.F, cfg.dv, dtype=torch.float64)
        z_out = torch.empty(2, cfg.H, cfg.F, dtype=torch.float64)
        sp.prefill_sequence_parallel(seg, o, cfg.F, flags=flags,
                                     S0=torch.from_numpy(S0) if rank == 0 else None,
                                     z0=torch.from_numpy(z0) if rank == 0 else None,
                                     S_out=S_out, z_out=z_out, ops=OracleOps())
        np.savez(os.path.join(out, "rank%d.npz" % rank), o=o.numpy(), S=S_out.numpy(), z=z_out.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("flags", [0, 1, 2])
def test_two_gloo_ranks_equal_one_pass(oracle_mod, tmp_path, flags):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), flags, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    cfg, inp, S0, z0 = _inputs(flags)
    o_ref, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                          A_log=inp["A_log"], S0=S0, z0=z0, dt_scaled_input=bool(flags & 1),
                                          return_state=True)
    L = inp["q"].shape[1]
    for r in range(world):
        d = np.load(tmp_path / ("rank%d.npz" % r))
        t0, t1 = r * L // world, (r + 1) * L // world
        np.testing.assert_allclose(d["o"], o_ref[:, t0:t1], rtol=1e-10, atol=1e-12)
    last = np.load(tmp_path / ("rank%d.npz" % (world - 1)))
    np.testing.assert_allclose(last["S"], S_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(last["z"], z_ref, rtol=1e-10, atol=1e-12)
