"""Pins for the oracle's block around the mixer (no GPU): layer norm, GELU,
the MLP and the parallel GPT-NeoX block (HedgeMamba explainer sec. 5.1).

Each test checks the oracle against something other than its own formula: a
closed form, an invariant, an independent evaluation (the normal CDF by
numerical quadrature of the density instead of erf; the MLP by scalar loops),
or a special case of the block that reduces to one branch.
"""
import math

import numpy as np
import pytest

rng = np.random.default_rng(777)


# ---------------------------------------------------------------- layer norm

def test_layer_norm_rows_have_zero_mean_and_unit_scaled_variance(oracle_mod):
    x = rng.normal(size=(5, 3, 37)) * 3.0 + 1.5
    eps = 1e-5
    y = oracle_mod.layer_norm(x, eps=eps)
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-13)
    var = x.var(-1)
    # population variance of the output: var / (var + eps)
    np.testing.assert_allclose(y.var(-1), var / (var + eps), rtol=1e-12)


def test_layer_norm_two_valued_row_closed_form(oracle_mod):
    a, eps = 0.3, 1e-5
    x = np.array([[a, -a, a, -a]])
    y = oracle_mod.layer_norm(x, eps=eps)
    r = a / math.sqrt(a * a + eps)
    np.testing.assert_allclose(y, [[r, -r, r, -r]], rtol=1e-14)


def test_layer_norm_affine_and_shift_scale_invariance(oracle_mod):
    x = rng.normal(size=(4, 16))
    w = rng.normal(size=16)
    b = rng.normal(size=16)
    base = oracle_mod.layer_norm(x, eps=0.0)
    np.testing.assert_allclose(oracle_mod.layer_norm(x, w, b, eps=0.0), base * w + b, rtol=1e-13, atol=1e-14)
    # with eps = 0 the map forgets a positive scale and a shift of each row
    np.testing.assert_allclose(oracle_mod.layer_norm(2.5 * x + 7.0, eps=0.0), base, rtol=1e-11, atol=1e-12)
    # and a negative scale flips the sign
    np.testing.assert_allclose(oracle_mod.layer_norm(-x, eps=0.0), -base, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- GELU

def _phi_by_quadrature(x, n=20000):
    """Standard normal CDF as the integral of the density from -12 to x
    (composite Simpson rule), independent of erf."""
    lo = -12.0
    if x <= lo:
        return 0.0
    t = np.linspace(lo, x, 2 * n + 1)
    f = np.exp(-0.5 * t * t) / math.sqrt(2 * math.pi)
    h = (x - lo) / (2 * n)
    return h / 3 * (f[0] + f[-1] + 4 * f[1:-1:2].sum() + 2 * f[2:-1:2].sum())


def test_gelu_is_x_times_normal_cdf(oracle_mod):
    xs = np.array([-4.0, -1.7, -0.3, 0.2, 1.0, 2.9, 5.5])
    got = oracle_mod.gelu(xs)
    ref = np.array([x * _phi_by_quadrature(x) for x in xs])
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-14)


def test_gelu_special_values_and_reflection(oracle_mod):
    assert oracle_mod.gelu(np.array([0.0]))[0] == 0.0
    x = rng.normal(size=50) * 3
    # Phi(-x) = 1 - Phi(x)  =>  gelu(x) - gelu(-x) = x
    np.testing.assert_allclose(oracle_mod.gelu(x) - oracle_mod.gelu(-x), x, rtol=1e-13, atol=1e-14)
    # tails: gelu(x) -> x for large x, -> 0 for large negative x
    assert oracle_mod.gelu(np.array([30.0]))[0] == 30.0
    assert abs(oracle_mod.gelu(np.array([-30.0]))[0]) < 1e-190


# ---------------------------------------------------------------- MLP

def test_mlp_matches_scalar_loops(oracle_mod):
    D, Fm = 3, 5
    h = rng.normal(size=(2, D))
    W1, b1 = rng.normal(size=(Fm, D)), rng.normal(size=Fm)
    W2, b2 = rng.normal(size=(D, Fm)), rng.normal(size=D)
    got = oracle_mod.mlp(h, W1, b1, W2, b2)
    ref = np.zeros((2, D))
    for r in range(2):
        u = [sum(W1[f, i] * h[r, i] for i in range(D)) + b1[f] for f in range(Fm)]
        gu = [ui * _phi_by_quadrature(ui) for ui in u]
        for j in range(D):
            ref[r, j] = sum(W2[j, f] * gu[f] for f in range(Fm)) + b2[j]
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- parallel block

def _block_params(D, H, dh, p, K, Fm):
    E = H * dh
    mixer = dict(
        W_q=rng.normal(size=(E, D)) / math.sqrt(D), W_k=rng.normal(size=(E, D)) / math.sqrt(D),
        W_v=rng.normal(size=(E, D)) / math.sqrt(D), W_g=rng.normal(size=(E, D)) / math.sqrt(D),
        W_dt=rng.normal(size=(H, D)) / math.sqrt(D), conv_w=rng.normal(size=(3, E, K)) / 2,
        W_hq=rng.normal(size=(p, dh)) / math.sqrt(dh), W_hk=rng.normal(size=(p, dh)) / math.sqrt(dh),
        A_log=rng.uniform(0, math.log(16), size=H), W_o=rng.normal(size=(D, E)) / math.sqrt(E))
    return dict(ln1_w=1 + 0.1 * rng.normal(size=D), ln1_b=0.1 * rng.normal(size=D),
                ln2_w=1 + 0.1 * rng.normal(size=D), ln2_b=0.1 * rng.normal(size=D),
                W_fc1=rng.normal(size=(Fm, D)) / math.sqrt(D), b_fc1=0.1 * rng.normal(size=Fm),
                W_fc2=rng.normal(size=(D, Fm)) / math.sqrt(Fm), b_fc2=0.1 * rng.normal(size=D),
                mixer=mixer)


def test_block_with_both_branches_zeroed_is_the_identity(oracle_mod):
    B, L, D, H, dh, p, K, Fm = 2, 7, 16, 2, 8, 4, 4, 64
    prm = _block_params(D, H, dh, p, K, Fm)
    prm["mixer"]["W_o"] = np.zeros_like(prm["mixer"]["W_o"])
    prm["W_fc2"] = np.zeros_like(prm["W_fc2"])
    prm["b_fc2"] = np.zeros(D)
    x = rng.normal(size=(B, L, D))
    np.testing.assert_array_equal(oracle_mod.block_fwd(x, n_heads=H, **prm), x)


def test_block_without_mixer_is_a_per_token_mlp_on_the_second_norm(oracle_mod):
    # W_o = 0 silences the mixer; each token then goes through LN2 and the MLP
    # alone, which a per-token scalar loop evaluates independently
    B, L, D, H, dh, p, K, Fm = 1, 3, 16, 2, 8, 4, 4, 8
    prm = _block_params(D, H, dh, p, K, Fm)
    prm["mixer"]["W_o"] = np.zeros_like(prm["mixer"]["W_o"])
    x = rng.normal(size=(B, L, D))
    got = oracle_mod.block_fwd(x, n_heads=H, **prm)
    for t in range(L):
        row = x[0, t]
        mu = sum(row) / D
        var = sum((v - mu) ** 2 for v in row) / D
        h = [(row[i] - mu) / math.sqrt(var + 1e-5) * prm["ln2_w"][i] + prm["ln2_b"][i] for i in range(D)]
        u = [sum(prm["W_fc1"][f, i] * h[i] for i in range(D)) + prm["b_fc1"][f] for f in range(Fm)]
        gu = [ui * _phi_by_quadrature(ui) for ui in u]
        for j in range(D):
            ref = row[j] + sum(prm["W_fc2"][j, f] * gu[f] for f in range(Fm)) + prm["b_fc2"][j]
            assert got[0, t, j] == pytest.approx(ref, rel=1e-9, abs=1e-11)


def test_block_mixer_branch_reads_the_first_norm(oracle_mod):
    # with the MLP silenced the block adds the mixer of LN1(x), not of x or LN2(x):
    # changing ln2 leaves the output unchanged, changing ln1 does not
    B, L, D, H, dh, p, K, Fm = 2, 6, 16, 2, 8, 4, 4, 16
    prm = _block_params(D, H, dh, p, K, Fm)
    prm["W_fc2"] = np.zeros_like(prm["W_fc2"])
    prm["b_fc2"] = np.zeros(D)
    x = rng.normal(size=(B, L, D))
    out = oracle_mod.block_fwd(x, n_heads=H, **prm)
    prm2 = dict(prm, ln2_w=prm["ln2_w"] * 3, ln2_b=prm["ln2_b"] - 1)
    np.testing.assert_array_equal(oracle_mod.block_fwd(x, n_heads=H, **prm2), out)
    prm3 = dict(prm, ln1_b=prm["ln1_b"] + 0.5)
    assert np.abs(oracle_mod.block_fwd(x, n_heads=H, **prm3) - out).max() > 1e-3
    # a row scale of x is forgotten by LN1 up to eps, so the mixer branch is unchanged
    # (eps = 0 makes it exact)
    o1 = oracle_mod.block_fwd(x, n_heads=H, eps=0.0, **prm) - x
    o2 = oracle_mod.block_fwd(4.0 * x, n_heads=H, eps=0.0, **prm) - 4.0 * x
    np.testing.assert_allclose(o1, o2, rtol=1e-9, atol=1e-11)
