"""GPU parity of the Hedgehog feature map (hm_featmap) and the recurrent
decode step (hm_step_decode) against the fp64 oracle."""
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


def _featmap_gpu(hm, x, W, io, out_dtype, H=1, bias=None, w_head_stride=0):
    import torch
    tx = dev_tensor(x, io)
    tW = dev_tensor(W, io)
    p = W.shape[-2]
    phi = torch.empty(x.shape[:-1] + (2 * p,), device="cuda",
                      dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32)
    tb = dev_tensor(bias, "f32") if bias is not None else None
    hm.hm_featmap(tx, tW, phi, H=H, bias=tb, w_head_stride=w_head_stride)
    torch.cuda.synchronize()
    return to_np(phi)


@pytest.mark.parametrize("rows", [1, 127, 128, 129, 1000, 5000])
@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_featmap_bf16_pythia_shape(hm, rows, out_dtype):
    x = wl.round_bf16(wl.normal(rows, "x", (rows, 256)))
    W = wl.round_bf16(wl.normal(rows, "W", (128, 256), 1 / 16))
    phi = _featmap_gpu(hm, x, W, "bf16", out_dtype)
    ref = oracle.featmap(x, W)
    assert rel_err(phi, ref) <= TOL_BF16
    assert (phi >= 0).all()
    np.testing.assert_allclose(phi.sum(-1), 1.0, rtol=2e-2)


def test_featmap_fp32_tiny_config(hm):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg)
    phi = _featmap_gpu(hm, inp["q"], inp["W_q"], "f32", "f32", H=cfg.H)
    ref = oracle.featmap(inp["q"], inp["W_q"], H=cfg.H)
    assert rel_err(phi, ref) <= TOL_F32


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_featmap_per_head_weights_and_bias(hm, out_dtype):
    H, d, p, rows = 4, 256, 128, 4 * 300
    x = wl.round_bf16(wl.normal(3, "x", (rows, d)))
    W = wl.round_bf16(wl.normal(3, "W", (H, p, d), 1 / 16))
    b = wl.round_f32(wl.normal(3, "b", (H, p), 0.5))
    phi = _featmap_gpu(hm, x, W, "bf16", out_dtype, H=H, bias=b, w_head_stride=p * d)
    ref = oracle.featmap(x, W, bias=b, H=H, w_head_stride=p * d, b_head_stride=p)
    assert rel_err(phi, ref) <= TOL_BF16


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_featmap_large_logits_stay_finite(hm, out_dtype):
    # |u| up to ~60: the max subtraction keeps exp in range
    x = wl.round_bf16(wl.normal(4, "x", (300, 256), 4.0))
    W = wl.round_bf16(wl.normal(4, "W", (128, 256), 1.0))
    phi = _featmap_gpu(hm, x, W, "bf16", out_dtype)
    assert np.isfinite(phi).all()
    assert rel_err(phi, oracle.featmap(x, W)) <= TOL_BF16


# ------------------------------------------------------------------ decode

def _decode_gpu(hm, q, k, v, S, z, Wq, Wk, dt, A_log, io="bf16"):
    import torch
    tq, tk, tv = dev_tensor(q, io), dev_tensor(k, io), dev_tensor(v, io)
    tS, tz = dev_tensor(S, "f32"), dev_tensor(z, "f32")
    o = torch.empty_like(tv)
    tWq, tWk = dev_tensor(Wq, io), dev_tensor(Wk, io)
    tdt = dev_tensor(dt, "f32") if dt is not None else None
    tA = dev_tensor(A_log, "f32")
    args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=tWq, W_k=tWk, dt=tdt, A_log=tA)
    ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_step_decode(args)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(o), to_np(tS), to_np(tz)


def _oracle_prefill_state(cfg, w, heads):
    """fp64 state after the seeded 1024-token prefill, for the (b, h) pairs in `heads`."""
    S = {}
    for b, h in heads:
        pre = wl.decode_prefill(cfg, index=(slice(b, b + 1), slice(None), slice(h, h + 1)))
        _, Sbh, zbh = oracle.scan_fwd(pre["q"], pre["k"], pre["v"], w["W_q"], w["W_k"],
                                      dt=pre["dt"], A_log=w["A_log"][h:h + 1], return_state=True)
        S[(b, h)] = (Sbh[0, 0], zbh[0, 0])
    return S


def test_decode_steps_full_size_sampled_heads(hm):
    """256 sequences x 8 heads.  Every head starts from a seeded synthetic
    state except the sampled heads, which start from the oracle's 1024-token
    prefill (cast to fp32); 8 decode steps then run on all heads and the
    sampled heads are compared with the oracle's own decode steps."""
    import torch
    cfg = wl.DECODE
    steps = 8
    w = wl.decode_weights(cfg)
    F, B, H = cfg.F, cfg.B, cfg.H
    heads = [(0, 0), (17, 3), (255, 7)]
    base = _oracle_prefill_state(cfg, w, heads)
    S = wl.round_f32(np.abs(wl.normal(cfg.seed, "S_init", (B, H, F, cfg.dv), 0.01)))
    z = wl.round_f32(np.abs(wl.normal(cfg.seed, "z_init", (B, H, F), 0.01)) + 1e-3)
    for (b, h), (Sb, zb) in base.items():
        S[b, h] = wl.round_f32(Sb)
        z[b, h] = wl.round_f32(zb)
    tS, tz = dev_tensor(S, "f32"), dev_tensor(z, "f32")
    ref_state = {bh: (S[bh].copy(), z[bh].copy()) for bh in base}
    tWq, tWk = dev_tensor(w["W_q"], "bf16"), dev_tensor(w["W_k"], "bf16")
    tA = dev_tensor(w["A_log"], "f32")
    for t in range(steps):
        tok = wl.decode_step_tokens(cfg, t)
        tq, tk, tv = (dev_tensor(tok[n], "bf16") for n in ("q", "k", "v"))
        o = torch.empty_like(tv)
        args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=tWq, W_k=tWk,
                              dt=dev_tensor(tok["dt"], "f32"), A_log=tA)
        ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_step_decode(args)
        og = to_np(o)
        for (b, h) in heads:
            Sr, zr = ref_state[(b, h)]
            phq = oracle.featmap(tok["q"][b:b + 1, h:h + 1], w["W_q"])
            phk = oracle.featmap(tok["k"][b:b + 1, h:h + 1], w["W_k"])
            la = oracle.log_decay(tok["dt"][b:b + 1, h:h + 1], w["A_log"][h:h + 1])
            o_ref, Sn, zn = oracle.decode_step(phq, phk, tok["v"][b:b + 1, h:h + 1],
                                               Sr[None, None], zr[None, None], la)
            ref_state[(b, h)] = (Sn[0, 0], zn[0, 0])
            assert rel_err(og[b, h], o_ref[0, 0]) <= TOL_BF16, (t, b, h)
    Sg, zg = to_np(tS), to_np(tz)
    for (b, h) in heads:
        assert rel_err(Sg[b, h], ref_state[(b, h)][0]) <= TOL_BF16
        assert rel_err(zg[b, h], ref_state[(b, h)][1]) <= TOL_BF16
    assert hm.hm_get_device_error() == hm.HM_OK


def test_decode_all_heads_16_steps_against_oracle(hm):
    """Every one of the 256 x 8 heads, 16 consecutive hm_step_decode calls,
    from a small seeded state (so that the per-step increments phi(k) v^T,
    not the initial state, make up S): o at every step and the final S and z
    against the oracle's own decode steps."""
    import torch
    cfg = wl.DECODE
    steps = 16
    w = wl.decode_weights(cfg)
    B, H, F, dv = cfg.B, cfg.H, cfg.F, cfg.dv
    S_ref = wl.round_f32(np.abs(wl.normal(cfg.seed, "S_all", (B, H, F, dv), 0.01)))
    z_ref = wl.round_f32(np.abs(wl.normal(cfg.seed, "z_all", (B, H, F), 0.01)) + 1e-3)
    tS, tz = dev_tensor(S_ref, "f32"), dev_tensor(z_ref, "f32")
    tWq, tWk = dev_tensor(w["W_q"], "bf16"), dev_tensor(w["W_k"], "bf16")
    tA = dev_tensor(w["A_log"], "f32")
    for t in range(steps):
        tok = wl.decode_step_tokens(cfg, 300 + t)
        tq, tk, tv = (dev_tensor(tok[n], "bf16") for n in ("q", "k", "v"))
        o = torch.empty_like(tv)
        args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=tWq, W_k=tWk,
                              dt=dev_tensor(tok["dt"], "f32"), A_log=tA)
        ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_step_decode(args)
        phq = oracle.featmap(tok["q"], w["W_q"])
        phk = oracle.featmap(tok["k"], w["W_k"])
        la = oracle.log_decay(tok["dt"], w["A_log"])
        o_ref, S_ref, z_ref = oracle.decode_step(phq, phk, tok["v"], S_ref, z_ref, la)
        assert rel_err(to_np(o), o_ref) <= TOL_BF16, t
    assert hm.hm_get_device_error() == hm.HM_OK
    assert rel_err(to_np(tS), S_ref) <= TOL_BF16
    assert rel_err(to_np(tz), z_ref) <= TOL_BF16


def test_decode_continues_gpu_prefill(hm):
    """prefill(L) then n decode steps = prefill(L + n) (both on the GPU and
    compared with the oracle's single prefill)."""
    import torch
    from gpu_common import run_scan
    cfg = wl.PREFILL_PYTHIA
    L, n = 257, 5
    inp = wl.scan_inputs(cfg, B=2, L=L + n, seed=41)
    pre = {k: (v[:, :L] if k in ("q", "k", "v", "dt") else v) for k, v in inp.items()}
    _, S, z = run_scan(hm, pre, "bf16", want_state=True)
    o_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                            A_log=inp["A_log"])
    for t in range(L, L + n):
        o, S, z = _decode_gpu(hm, inp["q"][:, t], inp["k"][:, t], inp["v"][:, t], S, z,
                              inp["W_q"], inp["W_k"], inp["dt"][:, t], inp["A_log"])
        assert rel_err(o, o_ref[:, t]) <= TOL_BF16


def test_decode_fp32_no_decay(hm):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, B=3, L=40, seed=42)
    o_ref, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"],
                                          return_state=True)
    _, S, z = oracle.scan_fwd(inp["q"][:, :39], inp["k"][:, :39], inp["v"][:, :39], inp["W_q"],
                              inp["W_k"], return_state=True)
    import torch
    S32, z32 = wl.round_f32(S), wl.round_f32(z)
    tq, tk, tv = (dev_tensor(inp[n][:, 39], "f32") for n in ("q", "k", "v"))
    tS, tz = dev_tensor(S32, "f32"), dev_tensor(z32, "f32")
    o = torch.empty_like(tv)
    tWq, tWk = dev_tensor(inp["W_q"], "f32"), dev_tensor(inp["W_k"], "f32")
    args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=tWq, W_k=tWk)
    ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_step_decode(args)
    torch.cuda.synchronize()
    assert rel_err(to_np(o), o_ref[:, 39]) <= TOL_F32
    assert rel_err(to_np(tS), S_ref) <= TOL_F32
