"""GPU parity of the pieces of the sequence-parallel prefill against the fp64
oracle: the state-only scan (o = NULL) with its summed log decay, the affine
composition of segment records (hm_scan_combine), a sequence cut into pieces
run one after another on this GPU exactly as ranks would run them, and
prefill_sequence_parallel itself on a one-rank NCCL group."""
import os
import socket

import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_common import TOL_BF16, TOL_F32, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def _dev_inputs(inp, io):
    t = {n: dev_tensor(inp[n], io) for n in ("q", "k", "v", "W_q", "W_k")}
    t["dt"] = dev_tensor(inp["dt"], "f32")
    t["A_log"] = dev_tensor(inp["A_log"], "f32")
    return t


@pytest.mark.parametrize("cfgname,io,L", [("prefill", "bf16", 1000), ("prefill", "bf16", 70), ("tiny", "f32", 130)])
def test_state_only_scan_and_log_decay(hm, cfgname, io, L):
    import torch
    cfg = wl.PREFILL_PYTHIA if cfgname == "prefill" else wl.TINY_F32
    inp = wl.scan_inputs(cfg, B=2, L=L, seed=101)
    if "dt" not in inp:
        inp["dt"] = wl.round_f32(wl.normal(101, "dt", (2, L, cfg.H)))
        inp["A_log"] = wl.round_f32(wl.uniform(101, "A_log", (cfg.H,), 0.0, 1.0))
    t = _dev_inputs(inp, io)
    S = torch.full((2, cfg.H, cfg.F, cfg.dv), float("nan"), device="cuda")
    z = torch.full((2, cfg.H, cfg.F), float("nan"), device="cuda")
    lam = torch.full((2, cfg.H), float("nan"), device="cuda")
    a = hm.scan_args(None, t["k"], t["v"], None, W_q=t["W_q"], W_k=t["W_k"], dt=t["dt"], A_log=t["A_log"],
                     S_out=S, z_out=z, log_decay_out=lam)
    ws = hm.alloc_workspace(hm.hm_scan_workspace_size(a))
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_scan_chunked_fwd(a)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    _, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                      A_log=inp["A_log"], return_state=True)
    lam_ref = oracle.log_decay(inp["dt"], inp["A_log"]).sum(axis=1)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert rel_err(to_np(S), S_ref) <= tol
    assert rel_err(to_np(z), z_ref) <= tol
    np.testing.assert_allclose(to_np(lam), lam_ref, rtol=1e-4)


@pytest.mark.parametrize("flags", [0, 1, 2])
def test_pieces_run_like_ranks_equal_one_pass(hm, flags):
    """A sequence of 4 x 512 tokens (bf16, F = dv = 256; the per-feature
    decay on the CUDA-core scan) cut into 4 pieces: state-only records of every
    piece, all start states from hm_scan_combine (only_part = -1), then each
    piece from its start; plus an initial state before piece 0."""
    import torch
    cfg = wl.PREFILL_PYTHIA
    n, Lp, B = 4, 512, 1
    L = n * Lp
    inp = wl.scan_inputs(cfg, B=B, L=L, seed=102)
    if flags & 2:
        inp["A_log"] = wl.round_f32(wl.uniform(102, "A_log_f", (cfg.H, cfg.F), 0.0, 1.0))
    S0 = wl.round_f32(np.abs(wl.normal(102, "S0", (B, cfg.H, cfg.F, cfg.dv), 0.05)))
    z0 = wl.round_f32(np.abs(wl.normal(102, "z0", (B, cfg.H, cfg.F), 0.05)) + 1e-3)
    t = _dev_inputs(inp, "bf16")
    BH, F, dv = B * cfg.H, cfg.F, cfg.dv
    per_feature = bool(flags & 2)
    reclen = hm.combine_record_len(BH, F, dv, per_feature)
    nl = BH * F if per_feature else BH
    off_S = (nl + 3) // 4 * 4
    recs = torch.zeros(n * reclen, device="cuda")
    for r in range(n):
        rec = recs[r * reclen:(r + 1) * reclen]
        sl = slice(r * Lp, (r + 1) * Lp)
        a = hm.scan_args(None, t["k"][:, sl], t["v"][:, sl], None, W_q=t["W_q"], W_k=t["W_k"],
                         dt=t["dt"][:, sl], A_log=t["A_log"], S_out=rec[off_S:off_S + BH * F * dv],
                         z_out=rec[off_S + BH * F * dv:off_S + BH * F * dv + BH * F], log_decay_out=rec[:nl],
                         flags=flags)
        ws = hm.alloc_workspace(hm.hm_scan_workspace_size(a))
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_scan_chunked_fwd(a)
    S_start = torch.empty(n, BH, F, dv, device="cuda")
    z_start = torch.empty(n, BH, F, device="cuda")
    S_end = torch.empty(BH, F, dv, device="cuda")
    z_end = torch.empty(BH, F, device="cuda")
    tS0, tz0 = dev_tensor(S0, "f32"), dev_tensor(z0, "f32")
    hm.hm_scan_combine(hm.combine_args(recs, n, BH, F, dv, reclen, S_start, z_start, per_feature=per_feature,
                                       S0=tS0, z0=tz0, S_end=S_end, z_end=z_end))
    o = torch.empty_like(t["v"])
    for r in range(n):
        sl = slice(r * Lp, (r + 1) * Lp)
        a = hm.scan_args(t["q"][:, sl], t["k"][:, sl], t["v"][:, sl], o[:, sl], W_q=t["W_q"], W_k=t["W_k"],
                         dt=t["dt"][:, sl], A_log=t["A_log"], S0=S_start[r].view(B, cfg.H, F, dv),
                         z0=z_start[r].view(B, cfg.H, F), flags=flags)
        ws = hm.alloc_workspace(hm.hm_scan_workspace_size(a))
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_scan_chunked_fwd(a)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    o_ref, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                          A_log=inp["A_log"], S0=S0, z0=z0, dt_scaled_input=bool(flags & 1),
                                          return_state=True)
    assert rel_err(to_np(o), o_ref) <= TOL_BF16
    assert rel_err(to_np(S_end).reshape(S_ref.shape), S_ref) <= TOL_BF16
    assert rel_err(to_np(z_end).reshape(z_ref.shape), z_ref) <= TOL_BF16


def test_combine_rejects_bad_records(hm):
    import torch
    recs = torch.zeros(100, device="cuda")
    S = torch.empty(4, device="cuda")
    a = hm.combine_args(recs, 2, 1, 4, 4, 20, S, S)    # a record needs 4 + 16 + 4 = 24 values
    with pytest.raises(hm.HMError):
        hm.hm_scan_combine(a)
    a = hm.combine_args(recs, 2, 1, 4, 4, 24, S, S, only_part=2)
    with pytest.raises(hm.HMError):
        hm.hm_scan_combine(a)


def test_prefill_sequence_parallel_one_rank_nccl(hm):
    """The orchestration with its real collectives on a one-rank NCCL group
    (this run has one GPU): equals the single call."""
    import torch
    import torch.distributed as dist
    from selective_ssm_sequence_b200 import sequence_parallel as sp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        cfg = wl.PREFILL_PYTHIA
        inp = wl.scan_inputs(cfg, B=2, L=300, seed=103)
        t = _dev_inputs(inp, "bf16")
        S0 = wl.round_f32(np.abs(wl.normal(103, "S0", (2, cfg.H, cfg.F, cfg.dv), 0.05)))
        z0 = wl.round_f32(np.abs(wl.normal(103, "z0", (2, cfg.H, cfg.F), 0.05)) + 1e-3)
        o = torch.empty_like(t["v"])
        S_out = torch.empty(2, cfg.H, cfg.F, cfg.dv, device="cuda")
        z_out = torch.empty(2, cfg.H, cfg.F, device="cuda")
        sp.prefill_sequence_parallel(t, o, cfg.F, S0=dev_tensor(S0, "f32"), z0=dev_tensor(z0, "f32"),
                                     S_out=S_out, z_out=z_out)
        torch.cuda.synchronize()
        assert hm.hm_get_device_error() == hm.HM_OK
        o_ref, S_ref, _ = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                          A_log=inp["A_log"], S0=S0, z0=z0, return_state=True)
        assert rel_err(to_np(o), o_ref) <= TOL_BF16
        assert rel_err(to_np(S_out), S_ref) <= TOL_BF16
    finally:
        dist.destroy_process_group()
