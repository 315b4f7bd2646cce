"""hm_step_decode_noalloc: the decode step for callers that cannot allocate
device memory (a plugin whose host application owns all device memory and
gives it no allocator, or a serving loop that must not allocate once it is
running).  Its per-token feature scratch is a fixed array inside the library
instead of a caller workspace.

Checked through the C ABI against hm_step_decode (which takes a workspace) on
consecutive calls: the two must give bit-identical o, S and z, since they run
the same launches, and both must match the fp64 oracle within the bf16 (or
fp32) tolerance of the other parity tests.  Also: a small call after a full-size
one reads nothing the earlier call left in the shared array, caller-supplied
features (W_q = NULL) need no scratch, and sizes beyond the array are refused
before anything is enqueued.

This file is collected last on purpose: it exercises a library-wide device
array shared by every call, and must pass both on its own in a fresh process
and after the rest of the suite."""
import ctypes

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


def _both_steps(hm, tq, tk, tv, S_ws, z_ws, S_na, z_na, **kw):
    """One step through each entry point on its own copy of the state;
    returns (o of hm_step_decode, o of hm_step_decode_noalloc)."""
    import torch
    o_ws = torch.full_like(tv, float("nan"))
    o_na = torch.full_like(tv, float("nan"))
    a_ws = hm.decode_args(tq, tk, tv, o_ws, S_ws, z_ws, **kw)
    ws = hm.alloc_workspace(hm.hm_decode_workspace_size(a_ws))
    a_ws.workspace, a_ws.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_step_decode(a_ws)
    a_na = hm.decode_args(tq, tk, tv, o_na, S_na, z_na, **kw)
    st = hm.lib.hm_step_decode_noalloc(ctypes.byref(a_na), torch.cuda.current_stream().cuda_stream)
    assert st == hm.HM_OK, hm.lib.hm_last_error_detail()
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return o_ws, o_na


def _oracle_step(tok, Wq, Wk, A_log, S, z, decay=True):
    phq = oracle.featmap(tok["q"], Wq)
    phk = oracle.featmap(tok["k"], Wk)
    la = oracle.log_decay(tok["dt"], A_log) if decay else None
    return oracle.decode_step(phq, phk, tok["v"], S, z, la)


def test_noalloc_decode_matches_workspace_decode_and_oracle_on_two_steps(hm):
    """256 sequences x 8 heads, F = 256 (exactly the array's limit), bf16 io,
    from a small seeded state so that the per-step increments dominate S."""
    import torch
    cfg = wl.DECODE
    w = wl.decode_weights(cfg)
    B, H, F, dv = cfg.B, cfg.H, cfg.F, cfg.dv
    S_ref = wl.round_f32(np.abs(wl.normal(cfg.seed, "S_na", (B, H, F, dv), 0.01)))
    z_ref = wl.round_f32(np.abs(wl.normal(cfg.seed, "z_na", (B, H, F), 0.01)) + 1e-3)
    S_ws, z_ws = dev_tensor(S_ref, "f32"), dev_tensor(z_ref, "f32")
    S_na, z_na = S_ws.clone(), z_ws.clone()
    tWq, tWk = dev_tensor(w["W_q"], "bf16"), dev_tensor(w["W_k"], "bf16")
    tA = dev_tensor(w["A_log"], "f32")
    for step in range(2):
        tok = wl.decode_step_tokens(cfg, 100 + step)
        tq, tk, tv = (dev_tensor(tok[n], "bf16") for n in ("q", "k", "v"))
        o_ws, o_na = _both_steps(hm, tq, tk, tv, S_ws, z_ws, S_na, z_na, W_q=tWq, W_k=tWk,
                                 dt=dev_tensor(tok["dt"], "f32"), A_log=tA)
        assert torch.equal(o_na, o_ws)
        assert torch.equal(S_na, S_ws)
        assert torch.equal(z_na, z_ws)
        o_ref, S_ref, z_ref = _oracle_step(tok, w["W_q"], w["W_k"], w["A_log"], S_ref, z_ref)
        assert rel_err(to_np(o_na), o_ref) <= TOL_BF16, step
    assert rel_err(to_np(S_na), S_ref) <= TOL_BF16
    assert rel_err(to_np(z_na), z_ref) <= TOL_BF16


def test_noalloc_small_fp32_call_after_a_full_size_call(hm):
    """A full-size call fills the shared array; the small fp32 call that
    follows (CUDA-core feature map, B=2 H=2 d=32 p=32 dv=32) must read only
    what it wrote itself: equal to hm_step_decode and to the oracle at 1e-4."""
    import torch
    cfg = wl.DECODE
    w = wl.decode_weights(cfg)
    tok = wl.decode_step_tokens(cfg, 200)
    big = [dev_tensor(tok[n], "bf16") for n in ("q", "k", "v")]
    Sb = torch.zeros(cfg.B, cfg.H, cfg.F, cfg.dv, device="cuda")
    zb = torch.full((cfg.B, cfg.H, cfg.F), 1e-3, device="cuda")
    ob = torch.empty_like(big[2])
    ab = hm.decode_args(*big, ob, Sb, zb, W_q=dev_tensor(w["W_q"], "bf16"), W_k=dev_tensor(w["W_k"], "bf16"))
    assert hm.lib.hm_step_decode_noalloc(ctypes.byref(ab), torch.cuda.current_stream().cuda_stream) == hm.HM_OK
    torch.cuda.synchronize()
    del Sb, zb

    B, H, d, p, dv = 2, 2, 32, 32, 32
    Wq = wl.round_f32(wl.normal(61, "W_q", (p, d), (1.0 / d) ** 0.5))
    Wk = wl.round_f32(wl.normal(61, "W_k", (p, d), (1.0 / d) ** 0.5))
    S0 = wl.round_f32(np.abs(wl.normal(61, "S0", (B, H, 2 * p, dv), 0.05)))
    z0 = wl.round_f32(np.abs(wl.normal(61, "z0", (B, H, 2 * p), 0.05)) + 1e-2)
    S_ws, z_ws = dev_tensor(S0, "f32"), dev_tensor(z0, "f32")
    S_na, z_na = S_ws.clone(), z_ws.clone()
    S_ref, z_ref = S0, z0
    for step in range(2):
        t = {n: wl.round_f32(wl.normal(62 + step, n, shp)) for n, shp in
             (("q", (B, H, d)), ("k", (B, H, d)), ("v", (B, H, dv)), ("dt", (B, H)))}
        tq, tk, tv = (dev_tensor(t[n], "f32") for n in ("q", "k", "v"))
        A = np.zeros(H)
        o_ws, o_na = _both_steps(hm, tq, tk, tv, S_ws, z_ws, S_na, z_na, W_q=dev_tensor(Wq, "f32"),
                                 W_k=dev_tensor(Wk, "f32"), dt=dev_tensor(t["dt"], "f32"),
                                 A_log=dev_tensor(A, "f32"))
        assert torch.equal(o_na, o_ws) and torch.equal(S_na, S_ws) and torch.equal(z_na, z_ws)
        o_ref, S_ref, z_ref = _oracle_step(t, Wq, Wk, A, S_ref, z_ref)
        assert rel_err(to_np(o_na), o_ref) <= TOL_F32, step
    assert rel_err(to_np(S_na), S_ref) <= TOL_F32
    assert rel_err(to_np(z_na), z_ref) <= TOL_F32


def test_noalloc_with_caller_features(hm):
    """W_q = W_k = NULL: q and k are the feature vectors; no scratch is used."""
    import torch
    B, H, F, dv = 4, 8, 256, 256
    phq = np.abs(wl.normal(71, "phq", (B, H, F))) + 1e-3
    phk = np.abs(wl.normal(71, "phk", (B, H, F))) + 1e-3
    phq, phk = wl.round_bf16(phq / phq.sum(-1, keepdims=True)), wl.round_bf16(phk / phk.sum(-1, keepdims=True))
    v = wl.round_bf16(wl.normal(71, "v", (B, H, dv)))
    dt = wl.round_f32(wl.normal(71, "dt", (B, H)))
    A = wl.round_f32(np.linspace(0.0, 2.0, H))
    S0 = wl.round_f32(np.abs(wl.normal(71, "S0", (B, H, F, dv), 0.01)))
    z0 = wl.round_f32(np.abs(wl.normal(71, "z0", (B, H, F), 0.01)) + 1e-3)
    S_ws, z_ws = dev_tensor(S0, "f32"), dev_tensor(z0, "f32")
    S_na, z_na = S_ws.clone(), z_ws.clone()
    o_ws, o_na = _both_steps(hm, dev_tensor(phq, "bf16"), dev_tensor(phk, "bf16"), dev_tensor(v, "bf16"),
                             S_ws, z_ws, S_na, z_na, dt=dev_tensor(dt, "f32"), A_log=dev_tensor(A, "f32"))
    assert torch.equal(o_na, o_ws) and torch.equal(S_na, S_ws) and torch.equal(z_na, z_ws)
    o_ref, S_ref, z_ref = oracle.decode_step(phq, phk, v, S0, z0, oracle.log_decay(dt, A))
    assert rel_err(to_np(o_na), o_ref) <= TOL_BF16
    assert rel_err(to_np(S_na), S_ref) <= TOL_BF16


def test_noalloc_decode_rejects_sizes_beyond_its_scratch(hm):
    import torch
    B, H, d, p, dv = 257, 8, 256, 128, 256   # B * H * F = 526,336 > 524,288
    tq = torch.zeros(B, H, d, dtype=torch.bfloat16, device="cuda")
    tv = torch.zeros(B, H, dv, dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(tv, 7.0)
    S = torch.zeros(B, H, 2 * p, dv, device="cuda")
    z = torch.ones(B, H, 2 * p, device="cuda")
    W = torch.zeros(p, d, dtype=torch.bfloat16, device="cuda")
    a = hm.decode_args(tq, tq, tv, o, S, z, W_q=W, W_k=W)
    st = hm.lib.hm_step_decode_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream)
    assert st == hm.HM_ERR_INVALID_ARG
    assert b"scratch" in hm.lib.hm_last_error_detail()
    torch.cuda.synchronize()
    assert (o == 7.0).all()          # nothing was enqueued
