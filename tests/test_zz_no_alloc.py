"""hm_step_decode_noalloc: the decode step for callers that cannot allocate
device memory (its feature-vector scratch is a fixed array inside the
library).  Checked through the C ABI against hm_step_decode, which takes a
caller-provided workspace, on two consecutive steps; plus the size limit.

This file is collected last on purpose: it exercises a library-wide device
array shared by every call, and must pass both on its own in a fresh process
and after the rest of the suite."""
import ctypes

import numpy as np
import pytest

import workloads as wl
from gpu_common import TOL_BF16, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def test_noalloc_decode_matches_workspace_decode_on_two_steps(hm):
    import torch
    cfg = wl.DECODE                       # 256 sequences x 8 heads, F = 256: exactly the limit
    w = wl.decode_weights(cfg)
    B, H, F, dv = cfg.B, cfg.H, cfg.F, cfg.dv
    S_init = wl.round_f32(np.abs(wl.normal(cfg.seed, "S_na", (B, H, F, dv), 0.01)))
    z_init = wl.round_f32(np.abs(wl.normal(cfg.seed, "z_na", (B, H, F), 0.01)) + 1e-3)
    S_ref, z_ref = dev_tensor(S_init, "f32"), dev_tensor(z_init, "f32")
    S_na, z_na = S_ref.clone(), z_ref.clone()
    tWq, tWk = dev_tensor(w["W_q"], "bf16"), dev_tensor(w["W_k"], "bf16")
    tA = dev_tensor(w["A_log"], "f32")
    for step in range(2):
        tok = wl.decode_step_tokens(cfg, 100 + step)
        tq, tk, tv = (dev_tensor(tok[n], "bf16") for n in ("q", "k", "v"))
        tdt = dev_tensor(tok["dt"], "f32")
        o_ref = torch.empty_like(tv)
        o_na = torch.full_like(tv, float("nan"))
        a_ref = hm.decode_args(tq, tk, tv, o_ref, S_ref, z_ref, W_q=tWq, W_k=tWk, dt=tdt, A_log=tA)
        ws = hm.alloc_workspace(hm.hm_decode_workspace_size(a_ref))
        a_ref.workspace, a_ref.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_step_decode(a_ref)
        a_na = hm.decode_args(tq, tk, tv, o_na, S_na, z_na, W_q=tWq, W_k=tWk, dt=tdt, A_log=tA)
        st = hm.lib.hm_step_decode_noalloc(ctypes.byref(a_na), torch.cuda.current_stream().cuda_stream)
        assert st == hm.HM_OK, hm.lib.hm_last_error_detail()
        torch.cuda.synchronize()
        assert hm.hm_get_device_error() == hm.HM_OK
        assert rel_err(to_np(o_na), to_np(o_ref)) <= TOL_BF16
        assert rel_err(to_np(S_na), to_np(S_ref)) <= TOL_BF16
        assert rel_err(to_np(z_na), to_np(z_ref)) <= TOL_BF16


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
