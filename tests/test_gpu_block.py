"""GPU parity of the fused epilogues and of the parallel block (hm_block_fwd)
against the fp64 oracle (HedgeMamba explainer sec. 5.1: x + mixer(LN1 x) +
MLP(LN2 x); sec. 2.3 / 5.2 for the mixer).

The mixer's projections carry the causal conv in their GEMM epilogue, with M
tiles that overlap by conv width - 1 rows; the cases below put sequence starts
inside tiles (L not a multiple of the tile step), use every conv width from 1
to 8 (halo 0..7 rows, crossing the epilogue warps' 32-row boundaries) and both
scan paths (the tensor-core scan, which applies the gate as it stores o, and
the CUDA-core scan, after which a separate kernel applies it)."""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_common import TOL_BF16, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def _dev_mixer(w):
    return {k: dev_tensor(v, "f32" if k in ("conv_w", "A_log", "conv_b", "b_g") else "bf16")
            for k, v in w.items()}


def _run_mixer(hm, x, w, H):
    import torch
    B, L, D = x.shape
    tx = dev_tensor(x, "bf16")
    out = torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    args = hm.mixer_args(tx, out, n_heads=H, **_dev_mixer(w))
    ws = hm.alloc_workspace(hm.hm_mixer_workspace_size(args))
    hm.hm_mixer_fwd(args, ws)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(out)


def branch_err(out, ref, x):
    """Error of the branches' sum (out - x) against the oracle's (ref - x) with
    the metric's floor on the branches, after allowing for the bf16 rounding of
    the stored output itself (up to 2^-8 |ref| per element): the residual x
    usually dominates |out|, so that rounding alone can exceed 2 % of a small
    branch value."""
    b = ref - x
    floor = np.maximum(np.abs(b), np.sqrt(np.mean(b * b)))
    excess = np.maximum(np.abs(out.astype(np.float64) - ref) - 2.0 ** -8 * np.abs(ref), 0.0)
    return float(np.max(excess / floor))


def _run_block(hm, x, w, bw, H):
    import torch
    B, L, D = x.shape
    tx = dev_tensor(x, "bf16")
    out = torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    tb = {k: dev_tensor(v, "bf16" if k.startswith("W_") else "f32") for k, v in bw.items()}
    args = hm.block_args(tx, out, _dev_mixer(w), n_heads=H, **tb)
    ws = hm.alloc_workspace(hm.hm_block_workspace_size(args))
    hm.hm_block_fwd(args, ws)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(out)


@pytest.mark.parametrize("K", [1, 2, 8])
def test_mixer_conv_epilogue_widths(hm, K):
    cfg = wl.MixerConfig("small", 2, 300, 512, 2, 128, K, 60 + K)
    w = wl.mixer_weights(cfg)
    x = wl.mixer_x(cfg)
    out = _run_mixer(hm, x, w, cfg.H)
    assert np.isfinite(out).all()
    ref = oracle.mixer_fwd(x, n_heads=cfg.H, **w)
    assert rel_err(out, ref) <= TOL_BF16


def test_mixer_cuda_core_scan_with_separate_gate(hm):
    # d_head = 64 (F = 64): the scan runs on the CUDA cores and the gate is a kernel of its own
    cfg = wl.MixerConfig("small_simt", 2, 190, 512, 8, 32, 4, 67)
    w = wl.mixer_weights(cfg)
    x = wl.mixer_x(cfg)
    E = cfg.H * cfg.d_head
    w["b_g"] = wl.round_f32(wl.normal(67, "b_g", (E,), 0.5))
    out = _run_mixer(hm, x, w, cfg.H)
    ref = oracle.mixer_fwd(x, n_heads=cfg.H, **w)
    assert rel_err(out, ref) <= TOL_BF16


def test_block_against_oracle(hm):
    cfg = wl.MixerConfig("block_small", 2, 300, 512, 2, 128, 4, 71)
    w = wl.mixer_weights(cfg)
    bw = wl.block_weights(cfg)
    x = wl.mixer_x(cfg)
    out = _run_block(hm, x, w, bw, cfg.H)
    assert np.isfinite(out).all()
    ref = oracle.block_fwd(x, n_heads=cfg.H, mixer=w, **bw)
    assert rel_err(out, ref) <= TOL_BF16
    # the branches: what both branches add to x must match at the same bar
    assert branch_err(out, ref, x) <= TOL_BF16


def test_block_with_mlp_silenced_is_input_plus_mixer(hm):
    cfg = wl.MixerConfig("block_nomlp", 1, 260, 512, 2, 128, 4, 72)
    w = wl.mixer_weights(cfg)
    bw = wl.block_weights(cfg, d_ff=1024)
    bw["W_fc2"] = np.zeros_like(bw["W_fc2"])
    bw["b_fc2"] = np.zeros_like(bw["b_fc2"])
    x = wl.mixer_x(cfg)
    out = _run_block(hm, x, w, bw, cfg.H)
    h1 = oracle.layer_norm(x, bw["ln1_w"], bw["ln1_b"])
    ref = x + oracle.mixer_fwd(h1, n_heads=cfg.H, **w)
    assert rel_err(out, ref) <= TOL_BF16
    assert branch_err(out, ref, x) <= TOL_BF16
