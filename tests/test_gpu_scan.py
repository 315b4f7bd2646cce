"""GPU parity of the prefill scan (hm_scan_chunked_fwd) against the fp64 oracle.

Every case runs through the C ABI on the same seeded inputs as the oracle.
Sizes span several chunks and ragged tails; the full-size configurations
are compared element by element (Pythia-shaped prefill) or on whole sampled
heads (long-context prefill), with the tolerances of the parity bar."""
import math

import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_common import TOL_BF16, TOL_F32, rel_err, run_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hm():
    import torch
    assert torch.cuda.is_available()
    import selective_ssm_sequence_b200 as mod
    return mod


def _oracle(inp, decay=True, S0=None, z0=None):
    return oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"],
                           dt=inp.get("dt") if decay else None,
                           A_log=inp.get("A_log") if decay else None,
                           S0=S0, z0=z0, return_state=True)


# ------------------------------------------------------------------ fp32 tiny config

def test_tiny_fp32_config_full(hm):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg)
    o, S, z = run_scan(hm, inp, "f32", want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(S, S_ref) <= TOL_F32
    assert rel_err(z, z_ref) <= TOL_F32


@pytest.mark.parametrize("L", [1, 7, 63, 64, 65, 129])
def test_tiny_fp32_ragged_lengths(hm, L):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, L=L, seed=100 + L)
    o, _, _ = run_scan(hm, inp, "f32")
    o_ref, _, _ = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_F32


def test_fp32_with_decay_and_initial_state(hm):
    cfg = wl.TINY_F32
    inp = wl.scan_inputs(cfg, B=2, L=100, seed=5)
    inp["dt"] = wl.store(wl.normal(5, "dt", (2, 100, cfg.H)), "f32")
    inp["A_log"] = wl.store(wl.uniform(5, "A_log", (cfg.H,), 0.0, math.log(16)), "f32")
    F = 2 * cfg.p
    S0 = wl.round_f32(np.abs(wl.normal(5, "S0", (2, cfg.H, F, cfg.dv))))
    z0 = wl.round_f32(np.abs(wl.normal(5, "z0", (2, cfg.H, F))) + 0.1)
    o, S, z = run_scan(hm, inp, "f32", S0=S0, z0=z0, want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp, S0=S0, z0=z0)
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(S, S_ref) <= TOL_F32
    assert rel_err(z, z_ref) <= TOL_F32


# ------------------------------------------------------------------ bf16 Pythia-shaped

@pytest.mark.parametrize("L", [1, 100, 128, 129, 300, 1000])
def test_bf16_pythia_shape_small(hm, L):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=L, seed=200 + L)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16
    assert rel_err(z, z_ref) <= TOL_BF16


def test_bf16_no_decay(hm):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=2, L=520, seed=7)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True, decay=False)
    o_ref, S_ref, z_ref = _oracle(inp, decay=False)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16


def test_bf16_weak_decay_carries_state_across_chunks(hm):
    # A_log very negative -> a_t close to 1: contributions survive many chunks
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=700, seed=8)
    inp["A_log"] = np.full(cfg.H, -6.0)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16


def test_bf16_initial_state_and_split_invariance(hm):
    # running [0, s) then [s, L) from the carried state equals one pass
    cfg = wl.PREFILL_PYTHIA
    L, s = 600, 333
    inp = wl.scan_inputs(cfg, B=1, L=L, seed=9)
    inp["A_log"] = np.full(cfg.H, -3.0)
    first = {k: (v[:, :s] if k in ("q", "k", "v", "dt") else v) for k, v in inp.items()}
    second = {k: (v[:, s:] if k in ("q", "k", "v", "dt") else v) for k, v in inp.items()}
    o1, S1, z1 = run_scan(hm, first, "bf16", want_state=True)
    o2, S2, z2 = run_scan(hm, second, "bf16", S0=S1, z0=z1, want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(np.concatenate([o1, o2], 1), o_ref) <= TOL_BF16
    assert rel_err(S2, S_ref) <= TOL_BF16
    o_all, _, _ = run_scan(hm, inp, "bf16")
    assert rel_err(np.concatenate([o1, o2], 1), o_all) <= TOL_BF16


def test_bf16_pythia_full_size(hm):
    # with the final state returned (the state phase covers every part, with
    # hi / lo splits) and without it (the timed prefill call: the state phase
    # covers the first segment only)
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16
    assert rel_err(z, z_ref) <= TOL_BF16
    o2, _, _ = run_scan(hm, inp, "bf16")
    assert rel_err(o2, o_ref) <= TOL_BF16


@pytest.mark.parametrize("L", [512, 1000])
def test_bf16_two_segments_with_initial_state(hm, L):
    # 32 heads: two output segments; the initial state enters segment 0
    # directly and segment 1 through the state parts and the carry
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, L=L, seed=300 + L)
    B = inp["q"].shape[0]
    F = 2 * cfg.p
    S0 = wl.round_f32(wl.normal(300 + L, "S0", (B, cfg.H, F, cfg.dv)) * 0.5)
    z0 = wl.round_f32(np.abs(wl.normal(300 + L, "z0", (B, cfg.H, F))) + 0.1)
    o, _, _ = run_scan(hm, inp, "bf16", S0=S0, z0=z0)
    o_ref, _, _ = _oracle(inp, S0=S0, z0=z0)
    assert rel_err(o, o_ref) <= TOL_BF16


def test_bf16_long_context_full_size_sampled_heads(hm):
    # every output of two whole heads (all 32768 tokens) and their final states
    cfg = wl.PREFILL_LONG
    inp = wl.scan_inputs(cfg)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True)
    o2, _, _ = run_scan(hm, inp, "bf16")   # the timed call: no returned state
    for h in (0, 5):
        sub = {k: (v[:, :, h:h + 1] if k in ("q", "k", "v", "dt") else
                   (v[h:h + 1] if k == "A_log" else v)) for k, v in inp.items()}
        o_ref, S_ref, z_ref = _oracle(sub)
        assert rel_err(o[:, :, h:h + 1], o_ref) <= TOL_BF16
        assert rel_err(S[:, h:h + 1], S_ref) <= TOL_BF16
        assert rel_err(z[:, h:h + 1], z_ref) <= TOL_BF16
        assert rel_err(o2[:, :, h:h + 1], o_ref) <= TOL_BF16


# ------------------------------------------------------------------ closed forms and degenerate cases

def test_zero_weight_gives_prefix_mean(hm):
    cfg = wl.PREFILL_PYTHIA
    L = 300
    inp = wl.scan_inputs(cfg, B=1, L=L, seed=21)
    inp["W_q"] = np.zeros_like(inp["W_q"])
    inp["W_k"] = np.zeros_like(inp["W_k"])
    o, _, _ = run_scan(hm, inp, "bf16", decay=False)
    ref = np.cumsum(inp["v"], axis=1) / np.arange(1, L + 1)[None, :, None, None]
    assert rel_err(o, ref) <= TOL_BF16


def test_constant_v_is_returned_and_outputs_are_convex(hm):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=400, seed=22)
    c = wl.round_bf16(wl.normal(22, "c", (1, 1, cfg.H, cfg.dv)))
    inp["v"] = np.broadcast_to(c, inp["v"].shape).copy()
    o, _, _ = run_scan(hm, inp, "bf16")
    assert rel_err(o, inp["v"]) <= 1e-2
    inp2 = wl.scan_inputs(cfg, B=1, L=400, seed=23)
    o2, _, _ = run_scan(hm, inp2, "bf16")
    lo = np.minimum.accumulate(inp2["v"], axis=1)
    hi = np.maximum.accumulate(inp2["v"], axis=1)
    slack = 1e-2 * np.abs(inp2["v"]).max()
    assert (o2 >= lo - slack).all() and (o2 <= hi + slack).all()


def test_full_reset_returns_v(hm):
    # dt huge -> a = 0 at every token -> o_t = v_t
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=200, seed=24)
    inp["dt"] = np.full(inp["dt"].shape, 1e30)
    o, _, _ = run_scan(hm, inp, "bf16")
    assert rel_err(o, inp["v"]) <= TOL_BF16


def test_empty_sequence_copies_the_state(hm):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=2, L=0, seed=25)
    F = 2 * cfg.p
    S0 = wl.round_f32(np.abs(wl.normal(25, "S0", (2, cfg.H, F, cfg.dv))))
    z0 = wl.round_f32(np.abs(wl.normal(25, "z0", (2, cfg.H, F))))
    _, S, z = run_scan(hm, inp, "bf16", S0=S0, z0=z0, want_state=True)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_array_equal(z, z0)


def test_shapes_without_a_tensor_core_kernel(hm):
    # F = 128, dv = 64: served by the CUDA-core path; still within tolerance
    cfg = wl.ScanConfig("odd", 2, 300, 3, 64, 64, 64, "bf16", True, 31, 1 / 8)
    inp = wl.scan_inputs(cfg)
    o, S, z = run_scan(hm, inp, "bf16", want_state=True)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16


def test_precomputed_features_path(hm):
    # W_q = NULL: q and k are feature vectors already (F = d)
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=260, seed=26)
    phq = wl.round_bf16(oracle.featmap(inp["q"], inp["W_q"]))
    phk = wl.round_bf16(oracle.featmap(inp["k"], inp["W_k"]))
    feat = dict(inp, q=phq, k=phk)
    o, _, _ = run_scan(hm, feat, "bf16", with_W=False)
    o_ref = oracle.scan_recurrent(phq, phk, inp["v"], oracle.log_decay(inp["dt"], inp["A_log"]))
    assert rel_err(o, o_ref) <= TOL_BF16


@pytest.mark.parametrize("want_state", [False, True])
def test_more_heads_than_sms(hm, want_state):
    # 80 heads x 2 value halves = 160 CTAs per segment: one segment, and the
    # output (and state) grids take a second wave
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=10, L=300, seed=29)
    o, S, z = run_scan(hm, inp, "bf16", want_state=want_state)
    o_ref, S_ref, z_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    if want_state:
        assert rel_err(S, S_ref) <= TOL_BF16
        assert rel_err(z, z_ref) <= TOL_BF16


def test_precomputed_features_with_returned_state(hm):
    # W_q = NULL and S_out requested: the state phase covers every part with
    # the hi / lo split of w (.) v and no phik remainder plane (three stages)
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=700, seed=28)
    phq = wl.round_bf16(oracle.featmap(inp["q"], inp["W_q"]))
    phk = wl.round_bf16(oracle.featmap(inp["k"], inp["W_k"]))
    feat = dict(inp, q=phq, k=phk)
    o, S, z = run_scan(hm, feat, "bf16", with_W=False, want_state=True)
    o_ref, S_ref, z_ref = oracle.scan_recurrent(phq, phk, inp["v"], oracle.log_decay(inp["dt"], inp["A_log"]),
                                                return_state=True)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16
    assert rel_err(z, z_ref) <= TOL_BF16


def test_per_head_weights_and_biases(hm):
    # one Hedgehog projection (and bias) per head: the q and k maps run in one
    # launch with one CTA column per head
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=2, L=200, seed=27)
    H, p, d = cfg.H, cfg.p, cfg.d
    Wq = wl.round_bf16(wl.normal(27, "Wq_heads", (H, p, d), 1 / d))
    Wk = wl.round_bf16(wl.normal(27, "Wk_heads", (H, p, d), 1 / d))
    bq = wl.round_f32(wl.normal(27, "bq_heads", (H, p), 0.25))
    bk = wl.round_f32(wl.normal(27, "bk_heads", (H, p), 0.25))
    heads = dict(inp, W_q=Wq, W_k=Wk)
    o, S, z = run_scan(hm, heads, "bf16", want_state=True, w_head_stride=p * d, b_q=bq, b_k=bk)
    o_ref, S_ref, z_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], Wq, Wk, dt=inp["dt"], A_log=inp["A_log"],
                                          b_q=bq, b_k=bk, w_head_stride=p * d, return_state=True)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(S, S_ref) <= TOL_BF16
    assert rel_err(z, z_ref) <= TOL_BF16


def test_shared_weights_with_biases(hm):
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=333, seed=28)
    bq = wl.round_f32(wl.normal(28, "bq", (cfg.p,), 0.25))
    bk = wl.round_f32(wl.normal(28, "bk", (cfg.p,), 0.25))
    o, _, _ = run_scan(hm, inp, "bf16", b_q=bq, b_k=bk)
    o_ref = oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                            A_log=inp["A_log"], b_q=bq, b_k=bk)
    assert rel_err(o, o_ref) <= TOL_BF16
