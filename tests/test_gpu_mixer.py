"""GPU parity of the full HedgeMamba mixer forward (hm_mixer_fwd) against the
fp64 oracle: projections, causal conv, Hedgehog maps, decayed normalised
scan, SiLU gate and output projection."""
import math

import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_common import TOL_BF16, dev_tensor, rel_err, rel_err_norm, rel_err_rows, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def _run_mixer(hm, x, w, H, b_g=None, conv_b=None):
    import torch
    B, L, D = x.shape
    t = {k: dev_tensor(v, "f32" if k in ("conv_w", "A_log") else "bf16") for k, v in w.items()}
    tx = dev_tensor(x, "bf16")
    out = torch.empty(B, L, D, dtype=torch.bfloat16, device="cuda")
    tbg = dev_tensor(b_g, "f32") if b_g is not None else None
    tcb = dev_tensor(conv_b, "f32") if conv_b is not None else None
    args = hm.mixer_args(tx, out, t["W_q"], t["W_k"], t["W_v"], t["W_g"], t["W_dt"], t["conv_w"],
                         t["W_hq"], t["W_hk"], t["A_log"], t["W_o"], n_heads=H, b_g=tbg, conv_b=tcb)
    ws = hm.alloc_workspace(hm.hm_mixer_workspace_size(args))
    hm.hm_mixer_fwd(args, ws)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(out)


def _small_weights(seed, D, H, p, K=4):
    cfg = wl.MixerConfig("small", 2, 300, D, H, p, K, seed)
    return cfg, wl.mixer_weights(cfg)


def test_mixer_small_against_oracle(hm):
    cfg, w = _small_weights(51, 512, 2, 128)
    x = wl.mixer_x(cfg, B=2, L=300)
    out = _run_mixer(hm, x, w, cfg.H)
    ref = oracle.mixer_fwd(x, n_heads=cfg.H, **w)
    assert rel_err(out, ref) <= TOL_BF16


def test_mixer_with_biases(hm):
    cfg, w = _small_weights(52, 512, 2, 128)
    x = wl.mixer_x(cfg, B=1, L=200)
    E = cfg.H * cfg.d_head
    b_g = wl.round_f32(wl.normal(52, "b_g", (E,), 0.5))
    conv_b = wl.round_f32(wl.normal(52, "conv_b", (3, E), 0.2))
    out = _run_mixer(hm, x, w, cfg.H, b_g=b_g, conv_b=conv_b)
    ref = oracle.mixer_fwd(x, n_heads=cfg.H, b_g=b_g, conv_b=conv_b, **w)
    assert rel_err(out, ref) <= TOL_BF16


def test_mixer_stage1_conv_and_gate_identity(hm):
    """Stage-1 identity initialisation of the conv and the gate (HedgeMamba
    explainer sec. 3.1): conv kernel [0, 0, 0, 1] and gate weights 0 with bias
    SiLU^-1(1) make both identities, so the mixer reduces to
    out_proj(decayed linear attention(q, k, v)).  The decay stays on: with
    a = 1 as well, late outputs are long averages and the tensor's rms (the
    metric's floor) shrinks below the bf16 storage error of v and y on the
    first tokens (a known limit, recorded in the design notes); the a = 1 scan
    itself is covered by the scan tests."""
    cfg, w = _small_weights(53, 512, 2, 128)
    x = wl.mixer_x(cfg, B=2, L=257)
    E = cfg.H * cfg.d_head
    w["conv_w"] = np.zeros((3, E, 4))
    w["conv_w"][:, :, -1] = 1.0
    w["W_g"] = np.zeros_like(w["W_g"])
    # SiLU^-1(1), rounded to fp32 (the stored bias)
    b_g = np.full(E, wl.round_f32(1.2784645427610738))
    out = _run_mixer(hm, x, w, cfg.H, b_g=b_g)
    B, L, D = x.shape
    xf = x.reshape(B * L, D)
    q = (xf @ w["W_q"].T).reshape(B, L, cfg.H, cfg.d_head)
    k = (xf @ w["W_k"].T).reshape(B, L, cfg.H, cfg.d_head)
    v = (xf @ w["W_v"].T).reshape(B, L, cfg.H, cfg.d_head)
    dt = (xf @ w["W_dt"].T).reshape(B, L, cfg.H)
    o = oracle.scan_fwd(q, k, v, W_q=w["W_hq"], W_k=w["W_hk"], dt=dt, A_log=w["A_log"])
    gate = oracle.silu(b_g)
    ref = (o.reshape(B * L, E) * gate) @ w["W_o"].T
    assert rel_err(out, ref.reshape(B, L, D)) <= TOL_BF16


def test_mixer_stage1_identity_without_decay(hm):
    """The full stage-1 identity initialisation (HedgeMamba explainer sec.
    3.1): conv kernel [0, 0, 0, 1], gate weights 0 with bias SiLU^-1(1), and no
    decay (exp(A_log) = 0, so a = 1 whatever dt is).  The mixer then reduces to
    out_proj(Hedgehog linear attention(q, k, v)).

    With a = 1, output row t is a t-token average, so rows shrink like
    1/sqrt(t) and the whole tensor's rms falls far below the first rows' size.
    The checks, at the 2e-2 bar, are (1) the max relative error with each
    token row's own rms as the floor and (2) the normwise error, both against
    the fp64 reference.  The whole-tensor floor is not used here: the bf16
    storage of the output alone (half an ulp of the largest, first-row
    outputs) is ~2 % of that floor, so it measured 2.4 % even against a
    reference that mirrors the mixer's bf16 storage of q, k and v."""
    cfg, w = _small_weights(54, 512, 2, 128)
    x = wl.mixer_x(cfg, B=2, L=257)
    E = cfg.H * cfg.d_head
    w["conv_w"] = np.zeros((3, E, 4))
    w["conv_w"][:, :, -1] = 1.0
    w["W_g"] = np.zeros_like(w["W_g"])
    w["A_log"] = np.full(cfg.H, -np.inf)
    b_g = np.full(E, wl.round_f32(1.2784645427610738))
    out = _run_mixer(hm, x, w, cfg.H, b_g=b_g)
    B, L, D = x.shape
    xf = x.reshape(B * L, D)
    gate = oracle.silu(b_g)

    q, k, v = ((xf @ w[n].T).reshape(B, L, cfg.H, cfg.d_head) for n in ("W_q", "W_k", "W_v"))
    o = oracle.scan_fwd(q, k, v, W_q=w["W_hq"], W_k=w["W_hk"])   # a = 1
    ref = ((o.reshape(B * L, E) * gate) @ w["W_o"].T).reshape(B, L, D)
    assert rel_err_rows(out, ref) <= TOL_BF16
    assert rel_err_norm(out, ref) <= TOL_BF16


def test_mixer_full_size_sampled_batches(hm):
    """B=8, L=4096, d_model=2048, H=8: every output of batches 0 and 7."""
    cfg = wl.MIXER
    w = wl.mixer_weights(cfg)
    x = wl.mixer_x(cfg)
    out = _run_mixer(hm, x, w, cfg.H)
    ref = oracle.mixer_fwd(x, n_heads=cfg.H, batches=[0, 7], **w)
    assert rel_err(out[[0, 7]], ref) <= TOL_BF16
