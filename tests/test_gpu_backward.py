"""GPU parity of the backward pass (hm_scan_bwd) against the oracle's
backward (chain-rule derivative of the forward definition, pinned by finite
differences and an independent autograd of the masked form): gradients of
sum(dout * o) with respect to q, k, v, the Hedgehog weights, dt and A_log,
and the initial state."""
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


def _bwd_gpu(hm, inp, dout, io, with_W=True, S0=None, z0=None):
    import torch
    q, k, v = (dev_tensor(inp[n], io) for n in ("q", "k", "v"))
    B, L, H, d = inp["q"].shape
    dv = inp["v"].shape[-1]
    F = 2 * inp["W_q"].shape[0] if with_W else d
    f32 = lambda *shape: torch.full(shape, float("nan"), device="cuda")
    g = dict(grad_q=f32(B, L, H, d), grad_k=f32(B, L, H, d), grad_v=f32(B, L, H, dv))
    kw = {}
    if with_W:
        p = inp["W_q"].shape[0]
        kw.update(W_q=dev_tensor(inp["W_q"], io), W_k=dev_tensor(inp["W_k"], io))
        g.update(grad_W_q=f32(p, d), grad_W_k=f32(p, d))
    if "dt" in inp:
        kw.update(dt=dev_tensor(inp["dt"], "f32"), A_log=dev_tensor(inp["A_log"], "f32"))
        g.update(grad_dt=f32(B, L, H), grad_A_log=f32(H))
    if S0 is not None:
        kw.update(S0=dev_tensor(S0, "f32"), z0=dev_tensor(z0, "f32"))
        g.update(grad_S0=f32(B, H, F, dv), grad_z0=f32(B, H, F))
    a = hm.scan_bwd_args(q, k, v, dev_tensor(dout, io), **kw, **g)
    ws = hm.alloc_workspace(hm.hm_scan_bwd_workspace_size(a))
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_scan_bwd(a)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return {n: to_np(t) for n, t in g.items()}


def _check(got, ref, tol):
    for name, r in ref.items():
        assert name in got, name
        assert np.isfinite(got[name]).all(), name
        err = rel_err(got[name], r)
        assert err <= tol, (name, err)


@pytest.mark.parametrize("L", [64, 131])
def test_backward_fp32_tiny(hm, L):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, L=L, seed=121)
    inp["dt"] = wl.round_f32(wl.normal(121, "dt", (cfg.B, L, cfg.H)))
    inp["A_log"] = wl.round_f32(wl.uniform(121, "A_log", (cfg.H,), 0.0, math.log(4.0)))
    dout = wl.round_f32(wl.normal(121, "dout", inp["v"].shape))
    got = _bwd_gpu(hm, inp, dout, "f32")
    r = oracle.scan_bwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dout, dt=inp["dt"],
                        A_log=inp["A_log"])
    _check(got, {"grad_q": r["dq"], "grad_k": r["dk"], "grad_v": r["dv"], "grad_W_q": r["dW_q"],
                 "grad_W_k": r["dW_k"], "grad_dt": r["ddt"], "grad_A_log": r["dA_log"]}, TOL_F32)


def test_backward_bf16_pythia_shape(hm):
    """d = dv = 256, p = 128 (F = 256), bf16 inputs, several token blocks and a ragged tail."""
    inp = wl.scan_inputs(wl.PREFILL_PYTHIA, B=1, L=150, seed=122)
    inp = {k: (v[:, :, :2] if k in ("q", "k", "v", "dt") else (v[:2] if k == "A_log" else v)) for k, v in inp.items()}
    dout = wl.round_bf16(wl.normal(122, "dout", inp["v"].shape))
    got = _bwd_gpu(hm, inp, dout, "bf16")
    r = oracle.scan_bwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dout, dt=inp["dt"],
                        A_log=inp["A_log"])
    _check(got, {"grad_q": r["dq"], "grad_k": r["dk"], "grad_v": r["dv"], "grad_W_q": r["dW_q"],
                 "grad_W_k": r["dW_k"], "grad_dt": r["ddt"], "grad_A_log": r["dA_log"]}, TOL_BF16)


def test_backward_initial_state_and_caller_features(hm):
    """q, k given as features (W = NULL) and an initial state: the gradients of
    the features, v, dt, A_log and of S0, z0."""
    cfg = wl.TINY_F32
    B, L, H, F, dv = 2, 90, cfg.H, 16, 8
    rng = np.random.default_rng(123)
    phq = rng.random((B, L, H, F)) + 0.05
    phk = rng.random((B, L, H, F)) + 0.05
    phq, phk = phq / phq.sum(-1, keepdims=True), phk / phk.sum(-1, keepdims=True)
    inp = {"q": wl.round_f32(phq), "k": wl.round_f32(phk), "v": wl.round_f32(rng.normal(size=(B, L, H, dv))),
           "dt": wl.round_f32(rng.normal(size=(B, L, H))), "A_log": wl.round_f32(np.array([0.2, 0.9]))}
    S0 = wl.round_f32(np.abs(rng.normal(size=(B, H, F, dv))) * 0.1)
    z0 = wl.round_f32(np.abs(rng.normal(size=(B, H, F))) * 0.1 + 0.01)
    dout = wl.round_f32(rng.normal(size=(B, L, H, dv)))
    got = _bwd_gpu(hm, inp, dout, "f32", with_W=False, S0=S0, z0=z0)
    la = oracle.log_decay(inp["dt"], inp["A_log"])
    dphq, dphk, dvv, dla, dS0, dz0 = oracle.scan_recurrent_bwd(inp["q"], inp["k"], inp["v"], dout, la, S0, z0)
    ddt, dA = oracle.log_decay_bwd(inp["dt"], inp["A_log"], dla)
    _check(got, {"grad_q": dphq, "grad_k": dphk, "grad_v": dvv, "grad_dt": ddt, "grad_A_log": dA,
                 "grad_S0": dS0, "grad_z0": dz0}, TOL_F32)


@pytest.mark.parametrize("d,p", [(10, 5), (260, 64), (64, 64)])
def test_backward_feature_map_products_shapes(hm, d, p):
    """The feature map's gradient products (dx = du W, dW = du^T x, the latter
    split over tokens) at sizes off the 128 x 128 tiles: d = 10, p = 5 (no
    vector loads; 582 rows over five row tiles, dW over 37 token splits),
    d = 260 (a column tile with 4 columns) and d = p = 64, where dx runs on
    the tensor cores as three bf16 segments of fp32 du and W (K = 192, 582
    rows: a ragged last row tile)."""
    cfg = wl.ScanConfig("ragged_featmap", 2, 97, 3, d, p, 8, "f32", True, 131, math.sqrt(1.0 / d))
    inp = wl.scan_inputs(cfg)
    dout = wl.round_f32(wl.normal(131, "dout", inp["v"].shape))
    got = _bwd_gpu(hm, inp, dout, "f32")
    r = oracle.scan_bwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dout, dt=inp["dt"],
                        A_log=inp["A_log"])
    _check(got, {"grad_q": r["dq"], "grad_k": r["dk"], "grad_v": r["dv"], "grad_W_q": r["dW_q"],
                 "grad_W_k": r["dW_k"], "grad_dt": r["ddt"]}, TOL_F32)
    # grad_A_log[h] = sum over tokens of dlog a_t * log a_t, whose terms cancel
    # (sum |terms| / |sum| reaches 36 here): an fp32 sum is accurate relative
    # to the sum of the terms' magnitudes, so that is the scale of the bar
    la = oracle.log_decay(inp["dt"], inp["A_log"])
    phq, phk = oracle.featmap(inp["q"], inp["W_q"]), oracle.featmap(inp["k"], inp["W_k"])
    dla = oracle.scan_recurrent_bwd(phq, phk, inp["v"], dout, la)[3]
    scale = np.abs(dla * la).sum(axis=(0, 1))
    assert np.allclose(r["dA_log"], (dla * la).sum(axis=(0, 1)), rtol=1e-12)
    assert (np.abs(got["grad_A_log"] - r["dA_log"]) <= TOL_F32 * scale).all()


def test_backward_empty_sequence_zeroes_parameter_gradients(hm):
    """L = 0: no token reaches an output, so the gradients of W_q, W_k, A_log
    and of the initial state are exactly zero (the buffers start as NaN)."""
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, B=2, L=0, seed=132)
    inp["dt"] = np.zeros((2, 0, cfg.H))
    inp["A_log"] = wl.round_f32(np.array([0.3, 1.1]))
    F = 2 * cfg.p
    S0 = np.full((2, cfg.H, F, cfg.dv), 0.5)
    z0 = np.full((2, cfg.H, F), 0.25)
    got = _bwd_gpu(hm, inp, np.zeros(inp["v"].shape), "f32", S0=S0, z0=z0)
    for name in ("grad_W_q", "grad_W_k", "grad_A_log", "grad_S0", "grad_z0"):
        assert got[name].size > 0 and (got[name] == 0).all(), name


def test_backward_bf16_rows_off_16_bytes(hm):
    """bf16 inputs whose value rows are not a multiple of 16 bytes (dv = 12):
    the passes stage their token blocks with plain loads instead of cp.async;
    d = 24, p = 12 (F = 24), two heads, a ragged last block of tokens."""
    cfg = wl.ScanConfig("bf16_dv12", 2, 45, 2, 24, 12, 12, "bf16", True, 133, math.sqrt(1.0 / 24))
    inp = wl.scan_inputs(cfg)
    dout = wl.round_bf16(wl.normal(133, "dout", inp["v"].shape))
    got = _bwd_gpu(hm, inp, dout, "bf16")
    r = oracle.scan_bwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dout, dt=inp["dt"],
                        A_log=inp["A_log"])
    _check(got, {"grad_q": r["dq"], "grad_k": r["dk"], "grad_v": r["dv"], "grad_W_q": r["dW_q"],
                 "grad_W_k": r["dW_k"], "grad_dt": r["ddt"], "grad_A_log": r["dA_log"]}, TOL_BF16)
