"""GPU parity of the scan's variant flags against the fp64 oracle:

* HM_FLAG_DT_SCALED_INPUT (Mamba's discretised input B-bar = Delta B with
  Delta = softplus(dt); HedgeMamba explainer sec. 5.2, SSM article sec. 3.2)
  on the tensor-core scan (bf16, F = dv = 256: ragged tails, several segments,
  returned states, an initial state) and on the CUDA-core scan (fp32 tiny);
* HM_FLAG_PER_FEATURE_DECAY (one rate per (head, feature), A_log [H, F];
  linear-attention tutorial sec. 4.4) on the CUDA-core scan;
* both flags in the decode step;
* HM_FLAG_ROPE (rotary embedding of phi(Q), phi(K), HedgeMamba explainer sec.
  5.2) on the tensor-core and CUDA-core scans, with a position offset, on
  caller-supplied features, and in the decode step at per-sequence positions."""
import math

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


def _scan(hm, inp, io, flags, A_log=None, S0=None, z0=None, want_state=False):
    import torch
    q, k, v = (dev_tensor(inp[n], io) for n in ("q", "k", "v"))
    Wq, Wk = dev_tensor(inp["W_q"], io), dev_tensor(inp["W_k"], io)
    A = dev_tensor(inp["A_log"] if A_log is None else A_log, "f32")
    o = torch.empty_like(v)
    B, L, H, d = inp["q"].shape
    F, dv = 2 * inp["W_q"].shape[-2], inp["v"].shape[-1]
    S = z = None
    if want_state:
        S = torch.full((B, H, F, dv), float("nan"), device="cuda")
        z = torch.full((B, H, F), float("nan"), device="cuda")
    args = hm.scan_args(q, k, v, o, W_q=Wq, W_k=Wk, dt=dev_tensor(inp["dt"], "f32"), A_log=A,
                        S0=None if S0 is None else dev_tensor(S0, "f32"),
                        z0=None if z0 is None else dev_tensor(z0, "f32"), S_out=S, z_out=z, flags=flags)
    ws = hm.alloc_workspace(hm.hm_scan_workspace_size(args))
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_scan_chunked_fwd(args)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(o), (to_np(S) if want_state else None), (to_np(z) if want_state else None)


def _per_feature_rates(seed, H, F):
    return wl.round_f32(wl.uniform(seed, "A_log_f", (H, F), 0.0, math.log(16.0)))


@pytest.mark.parametrize("L,want_state", [(300, False), (300, True), (1000, True), (4096, False)])
def test_dt_scaled_input_tensor_cores(hm, L, want_state):
    inp = wl.scan_inputs(wl.PREFILL_PYTHIA, B=2, L=L, seed=81 + L)
    o, S, z = _scan(hm, inp, "bf16", hm.HM_FLAG_DT_SCALED_INPUT, want_state=want_state)
    ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                          A_log=inp["A_log"], dt_scaled_input=True, return_state=want_state)
    if want_state:
        ref, S_ref, z_ref = ref
        assert rel_err(S, S_ref) <= TOL_BF16
        assert rel_err(z, z_ref) <= TOL_BF16
    assert rel_err(o, ref) <= TOL_BF16


def test_dt_scaled_input_from_an_initial_state(hm):
    inp = wl.scan_inputs(wl.PREFILL_PYTHIA, B=1, L=700, seed=85)
    B, H, F, dv = 1, wl.PREFILL_PYTHIA.H, wl.PREFILL_PYTHIA.F, wl.PREFILL_PYTHIA.dv
    S0 = wl.round_f32(np.abs(wl.normal(85, "S0", (B, H, F, dv), 0.05)))
    z0 = wl.round_f32(np.abs(wl.normal(85, "z0", (B, H, F), 0.05)) + 1e-3)
    o, S, _ = _scan(hm, inp, "bf16", hm.HM_FLAG_DT_SCALED_INPUT, S0=S0, z0=z0, want_state=True)
    ref, S_ref, _ = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                    A_log=inp["A_log"], dt_scaled_input=True, S0=S0, z0=z0,
                                    return_state=True)
    assert rel_err(o, ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_variants_fp32_tiny(hm, flags):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, L=130, seed=86)
    inp["dt"] = wl.round_f32(wl.normal(86, "dt", (cfg.B, 130, cfg.H)))
    inp["A_log"] = wl.round_f32(wl.uniform(86, "A_log", (cfg.H,), 0.0, math.log(4.0)))
    A = _per_feature_rates(86, cfg.H, cfg.F) if flags & 2 else None
    o, S, _ = _scan(hm, inp, "f32", flags, A_log=A, want_state=True)
    ref, S_ref, _ = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                    A_log=inp["A_log"] if A is None else A, dt_scaled_input=bool(flags & 1),
                                    return_state=True)
    assert rel_err(o, ref) <= TOL_F32
    assert rel_err(S, S_ref) <= TOL_F32


@pytest.mark.parametrize("flags", [2, 3])
def test_per_feature_decay_bf16(hm, flags):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=2, L=200, seed=87)
    A = _per_feature_rates(87, cfg.H, cfg.F)
    o, S, z = _scan(hm, inp, "bf16", flags, A_log=A, want_state=True)
    ref, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                        A_log=A, dt_scaled_input=bool(flags & 1), return_state=True)
    assert rel_err(o, ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16
    assert rel_err(z, z_ref) <= TOL_BF16


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_decode_variants(hm, flags):
    import torch
    cfg = wl.DECODE
    B, H, F, dv = 16, cfg.H, cfg.F, cfg.dv
    w = wl.decode_weights(cfg)
    A = _per_feature_rates(88, H, F) if flags & 2 else w["A_log"]
    S = wl.round_f32(np.abs(wl.normal(88, "S", (B, H, F, dv), 0.01)))
    z = wl.round_f32(np.abs(wl.normal(88, "z", (B, H, F), 0.01)) + 1e-3)
    tS, tz = dev_tensor(S, "f32"), dev_tensor(z, "f32")
    tWq, tWk, tA = dev_tensor(w["W_q"], "bf16"), dev_tensor(w["W_k"], "bf16"), dev_tensor(A, "f32")
    for step in range(3):
        t = {n: wl.round_bf16(wl.normal(89 + step, n, shp)) for n, shp in
             (("q", (B, H, cfg.d)), ("k", (B, H, cfg.d)), ("v", (B, H, dv)))}
        t["dt"] = wl.round_f32(wl.normal(89 + step, "dt", (B, H)))
        tq, tk, tv = (dev_tensor(t[n], "bf16") for n in ("q", "k", "v"))
        o = torch.empty_like(tv)
        args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=tWq, W_k=tWk, dt=dev_tensor(t["dt"], "f32"),
                              A_log=tA, flags=flags)
        ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_step_decode(args)
        torch.cuda.synchronize()
        assert hm.hm_get_device_error() == hm.HM_OK
        phq = oracle.featmap(t["q"], w["W_q"])[:, None]
        phk = oracle.featmap(t["k"], w["W_k"])[:, None]
        dt1 = t["dt"][:, None]
        laf = oracle.log_decay_per_feature(dt1, A) if flags & 2 else None
        la = None if flags & 2 else oracle.log_decay(dt1, A)
        sc = oracle.step_size(dt1) if flags & 1 else None
        o_ref, S, z = oracle.scan_recurrent_ext(phq, phk, t["v"][:, None], log_a=la, log_a_f=laf, in_scale=sc,
                                                S0=S, z0=z, return_state=True)
        assert rel_err(to_np(o), o_ref[:, 0]) <= TOL_BF16, step
    assert rel_err(to_np(tS), S) <= TOL_BF16
    assert rel_err(to_np(tz), z) <= TOL_BF16


# ---------------------------------------------------------------- rotary embedding (HM_FLAG_ROPE)

def _scan_rope(hm, inp, io, pos0=0, S0=None, z0=None, want_state=False, with_W=True, base=10000.0):
    import torch
    q, k, v = (dev_tensor(inp[n], io) for n in ("q", "k", "v"))
    Wq = dev_tensor(inp["W_q"], io) if with_W else None
    Wk = dev_tensor(inp["W_k"], io) if with_W else None
    o = torch.empty_like(v)
    B, L, H, d = inp["q"].shape
    F = 2 * inp["W_q"].shape[-2] if with_W else d
    dv = inp["v"].shape[-1]
    S = z = None
    if want_state:
        S = torch.full((B, H, F, dv), float("nan"), device="cuda")
        z = torch.full((B, H, F), float("nan"), device="cuda")
    args = hm.scan_args(q, k, v, o, W_q=Wq, W_k=Wk, dt=dev_tensor(inp["dt"], "f32"),
                        A_log=dev_tensor(inp["A_log"], "f32"),
                        S0=None if S0 is None else dev_tensor(S0, "f32"),
                        z0=None if z0 is None else dev_tensor(z0, "f32"), S_out=S, z_out=z,
                        flags=hm.HM_FLAG_ROPE, rope_base=base, pos0=pos0)
    ws = hm.alloc_workspace(hm.hm_scan_workspace_size(args))
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_scan_chunked_fwd(args)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(o), (to_np(S) if want_state else None), (to_np(z) if want_state else None)


@pytest.mark.parametrize("L", [300, 1000])
def test_rope_tensor_cores(hm, L):
    inp = wl.scan_inputs(wl.PREFILL_PYTHIA, B=2, L=L, seed=111)
    o, S, _ = _scan_rope(hm, inp, "bf16", want_state=True)
    ref, S_ref, _ = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                    A_log=inp["A_log"], rope_base=10000.0, return_state=True)
    assert rel_err(o, ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16


def test_rope_split_with_position_offset(hm):
    """[0, 600) then [600, 1300) from the carried state at positions 600..:
    the outputs equal the oracle's single pass."""
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=1300, seed=112)
    L1 = 600
    first = {n: (a[:, :L1] if n in ("q", "k", "v", "dt") else a) for n, a in inp.items()}
    second = {n: (a[:, L1:] if n in ("q", "k", "v", "dt") else a) for n, a in inp.items()}
    o1, S1, z1 = _scan_rope(hm, first, "bf16", want_state=True)
    o2, _, _ = _scan_rope(hm, second, "bf16", pos0=L1, S0=S1, z0=z1)
    ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"], A_log=inp["A_log"],
                          rope_base=10000.0)
    assert rel_err(np.concatenate([o1, o2], axis=1), ref) <= TOL_BF16


def test_rope_fp32_tiny(hm):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, L=130, seed=113)
    inp["dt"] = wl.round_f32(wl.normal(113, "dt", (cfg.B, 130, cfg.H)))
    inp["A_log"] = wl.round_f32(wl.uniform(113, "A_log", (cfg.H,), 0.0, math.log(4.0)))
    o, S, _ = _scan_rope(hm, inp, "f32", want_state=True)
    ref, S_ref, _ = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                                    A_log=inp["A_log"], rope_base=10000.0, return_state=True)
    assert rel_err(o, ref) <= TOL_F32
    assert rel_err(S, S_ref) <= TOL_F32


def test_rope_caller_features(hm):
    """W_q = NULL: the caller's (positive) features are rotated into the
    workspace, and the caller's buffers are left as they were."""
    import torch
    cfg = wl.PREFILL_PYTHIA
    B, L, H, F = 1, 400, cfg.H, cfg.F
    inp = wl.scan_inputs(cfg, B=B, L=L, seed=114)
    phq = oracle.featmap(inp["q"], inp["W_q"])
    phk = oracle.featmap(inp["k"], inp["W_k"])
    feat = dict(inp, q=wl.round_bf16(phq), k=wl.round_bf16(phk))
    tq = dev_tensor(feat["q"], "bf16")
    before = tq.clone()
    o, _, _ = _scan_rope(hm, feat, "bf16", with_W=False)
    ref = oracle.scan_fwd(feat["q"], feat["k"], inp["v"], dt=inp["dt"], A_log=inp["A_log"], rope_base=10000.0)
    assert rel_err(o, ref) <= TOL_BF16
    assert torch.equal(tq, before)


def test_rope_decode(hm):
    import torch
    cfg = wl.DECODE
    B, H, F, dv = 16, cfg.H, cfg.F, cfg.dv
    w = wl.decode_weights(cfg)
    S = wl.round_f32(np.abs(wl.normal(115, "S", (B, H, F, dv), 0.01)))
    z = wl.round_f32(np.abs(wl.normal(115, "z", (B, H, F), 0.01)) + 1e-3)
    pos = np.arange(B, dtype=np.int64) * 997 + 5
    tS, tz = dev_tensor(S, "f32"), dev_tensor(z, "f32")
    tpos = torch.from_numpy(pos).cuda()
    for step in range(2):
        t = {n: wl.round_bf16(wl.normal(116 + step, n, shp)) for n, shp in
             (("q", (B, H, cfg.d)), ("k", (B, H, cfg.d)), ("v", (B, H, dv)))}
        t["dt"] = wl.round_f32(wl.normal(116 + step, "dt", (B, H)))
        tq, tk, tv = (dev_tensor(t[n], "bf16") for n in ("q", "k", "v"))
        o = torch.empty_like(tv)
        args = hm.decode_args(tq, tk, tv, o, tS, tz, W_q=dev_tensor(w["W_q"], "bf16"), W_k=dev_tensor(w["W_k"], "bf16"),
                              dt=dev_tensor(t["dt"], "f32"), A_log=dev_tensor(w["A_log"], "f32"),
                              flags=hm.HM_FLAG_ROPE, rope_base=10000.0, positions=tpos + step)
        ws = hm.alloc_workspace(hm.hm_decode_workspace_size(args))
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_step_decode(args)
        torch.cuda.synchronize()
        assert hm.hm_get_device_error() == hm.HM_OK
        p = (pos + step)[:, None]
        phq = oracle.rope(oracle.featmap(t["q"], w["W_q"]), p)[:, None]
        phk = oracle.rope(oracle.featmap(t["k"], w["W_k"]), p)[:, None]
        o_ref, S, z = oracle.scan_recurrent(phq, phk, t["v"][:, None], oracle.log_decay(t["dt"][:, None], w["A_log"]),
                                            S0=S, z0=z, return_state=True)
        assert rel_err(to_np(o), o_ref[:, 0]) <= TOL_BF16, step
    assert rel_err(to_np(tS), S) <= TOL_BF16
