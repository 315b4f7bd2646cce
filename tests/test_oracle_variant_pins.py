"""CPU pins of the oracle's variant recurrences (no GPU):

* the step-scaled input of Mamba's discretisation (HedgeMamba explainer sec.
  5.2 calls Mamba's selective scan, whose input term is B-bar = Delta B; SSM
  article sec. 3.2: Delta = softplus(dt)):
      S_t = a_t S_{t-1} + Delta_t phik_t v_t^T,   z_t = a_t z_{t-1} + Delta_t phik_t
* a decay per feature (linear-attention tutorial sec. 4.4, gated linear
  attention S_i = diag(alpha_i) S_{i-1} + k_i v_i^T):
      S_t[f, :] = a_{t,f} S_{t-1}[f, :] + phik_t[f] v_t^T

* the rotary embedding on phi(Q), phi(K) (HedgeMamba explainer sec. 5.2),
  "rotate half" pairing (i, i + F/2), angle pos * base^(-2i/F).

Each recurrence variant is checked against an independent O(L^2) masked
form, closed forms on one and two tokens, and exact invariances that tie it
back to the pinned plain recurrence; the rotation against plane-rotation
closed forms, composition, relative-position invariance, and a split of the
sequence with carried state and a position offset."""
import math

import numpy as np
import pytest

rng = np.random.default_rng(20261203)


def _phi(shape):
    x = rng.random(shape) + 0.05
    return x / x.sum(-1, keepdims=True)


def _case(B=2, L=11, H=2, F=5, dv=3):
    return _phi((B, L, H, F)), _phi((B, L, H, F)), rng.normal(size=(B, L, H, dv))


def test_step_size_is_softplus(oracle_mod):
    d = oracle_mod.step_size(np.array([0.0, 3.0, -3.0, 40.0, -40.0]))
    assert d[0] == pytest.approx(math.log(2.0), rel=1e-15)
    assert d[1] - d[2] == pytest.approx(3.0, rel=1e-14)        # softplus(x) - softplus(-x) = x
    assert d[3] == pytest.approx(40.0, rel=1e-15)
    assert d[4] == pytest.approx(math.exp(-40.0), rel=1e-12)


def test_per_feature_log_decay_with_equal_rates_is_the_scalar_decay(oracle_mod):
    dt = rng.normal(size=(2, 7, 3))
    A = rng.uniform(0, math.log(16), size=3)
    laf = oracle_mod.log_decay_per_feature(dt, np.repeat(A[:, None], 4, axis=1))
    la = oracle_mod.log_decay(dt, A)
    np.testing.assert_array_equal(laf, np.repeat(la[..., None], 4, axis=-1))
    # and the rate of one feature scales its log decay alone
    A2 = np.repeat(A[:, None], 4, axis=1)
    A2[:, 2] += math.log(3.0)
    laf2 = oracle_mod.log_decay_per_feature(dt, A2)
    np.testing.assert_allclose(laf2[..., 2], 3.0 * la, rtol=1e-13)


def test_variants_off_equal_the_plain_recurrence(oracle_mod):
    phq, phk, v = _case()
    la = -rng.exponential(0.5, size=v.shape[:3])
    o1, S1, z1 = oracle_mod.scan_recurrent(phq, phk, v, la, return_state=True)
    o2, S2, z2 = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a=la, return_state=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


@pytest.mark.parametrize("scaled,per_feature,scalar", [(True, False, False), (True, False, True),
                                                        (False, True, False), (True, True, False)])
def test_variant_recurrence_equals_its_quadratic_form(oracle_mod, scaled, per_feature, scalar):
    phq, phk, v = _case()
    B, L, H, F = phq.shape
    la = -rng.exponential(0.5, size=(B, L, H)) if scalar else None
    laf = -rng.exponential(0.5, size=(B, L, H, F)) if per_feature else None
    sc = rng.uniform(0.1, 3.0, size=(B, L, H)) if scaled else None
    o_r = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a=la, log_a_f=laf, in_scale=sc)
    o_q = oracle_mod.scan_quadratic_ext(phq, phk, v, log_a=la, log_a_f=laf, in_scale=sc)
    np.testing.assert_allclose(o_r, o_q, rtol=1e-12, atol=1e-12)


def test_constant_step_size_scales_the_state_and_leaves_the_output(oracle_mod):
    phq, phk, v = _case()
    la = -rng.exponential(0.5, size=v.shape[:3])
    o0, S0, z0 = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a=la, return_state=True)
    o1, S1, z1 = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a=la, in_scale=np.full(v.shape[:3], 2.5),
                                               return_state=True)
    np.testing.assert_allclose(o1, o0, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S1, 2.5 * S0, rtol=1e-13)
    np.testing.assert_allclose(z1, 2.5 * z0, rtol=1e-13)


def test_step_scaled_input_on_one_and_two_tokens(oracle_mod):
    # one token: o_1 = v_1 whatever Delta_1 is; two tokens, a = 1:
    # o_2 = (D1 p1 v1 + D2 p2 v2) / (D1 p1 + D2 p2), p_j = phiq_2 . phik_j
    phq, phk, v = _case(B=1, L=2, H=1, F=4, dv=3)
    sc = np.array([[[0.3], [1.7]]])
    o = oracle_mod.scan_recurrent_ext(phq, phk, v, in_scale=sc)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], rtol=1e-14)
    p1 = phq[0, 1, 0] @ phk[0, 0, 0]
    p2 = phq[0, 1, 0] @ phk[0, 1, 0]
    ref = (0.3 * p1 * v[0, 0, 0] + 1.7 * p2 * v[0, 1, 0]) / (0.3 * p1 + 1.7 * p2)
    np.testing.assert_allclose(o[0, 1, 0], ref, rtol=1e-14)


def test_per_feature_decay_on_two_tokens(oracle_mod):
    # S_2 = diag(a_2) phik_1 v_1^T + phik_2 v_2^T, z_2 = a_2 (.) phik_1 + phik_2
    phq, phk, v = _case(B=1, L=2, H=1, F=4, dv=3)
    laf = np.zeros((1, 2, 1, 4))
    laf[0, 1, 0] = [-0.1, -1.0, -3.0, 0.0]
    o, S, z = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a_f=laf, return_state=True)
    a2 = np.exp(laf[0, 1, 0])
    S_ref = np.outer(a2 * phk[0, 0, 0], v[0, 0, 0]) + np.outer(phk[0, 1, 0], v[0, 1, 0])
    z_ref = a2 * phk[0, 0, 0] + phk[0, 1, 0]
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=1e-14)
    np.testing.assert_allclose(z[0, 0], z_ref, rtol=1e-14)
    np.testing.assert_allclose(o[0, 1, 0], phq[0, 1, 0] @ S_ref / (phq[0, 1, 0] @ z_ref), rtol=1e-14)


def test_per_feature_decay_with_equal_features_is_the_scalar_recurrence(oracle_mod):
    phq, phk, v = _case()
    la = -rng.exponential(0.5, size=v.shape[:3])
    F = phq.shape[-1]
    o1 = oracle_mod.scan_recurrent(phq, phk, v, la)
    o2 = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a_f=np.repeat(la[..., None], F, axis=-1))
    np.testing.assert_allclose(o2, o1, rtol=1e-13, atol=1e-14)


def test_full_reset_returns_the_value_in_both_variants(oracle_mod):
    # a = 0 on every feature at token t: o_t = v_t, with or without the step scale
    phq, phk, v = _case(L=9)
    laf = -rng.exponential(0.5, size=phq.shape)
    laf[:, 5] = -np.inf
    sc = rng.uniform(0.2, 2.0, size=v.shape[:3])
    o = oracle_mod.scan_recurrent_ext(phq, phk, v, log_a_f=laf, in_scale=sc)
    np.testing.assert_allclose(o[:, 5], v[:, 5], rtol=1e-13, atol=1e-14)


def test_scan_fwd_routes_the_variants(oracle_mod):
    B, L, H, d, p, dv = 1, 6, 2, 8, 4, 3
    q, k = rng.normal(size=(B, L, H, d)), rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, dv))
    Wq, Wk = rng.normal(size=(p, d)) / 3, rng.normal(size=(p, d)) / 3
    dt = rng.normal(size=(B, L, H))
    A = rng.uniform(0, 1, size=(H, 2 * p))
    o = oracle_mod.scan_fwd(q, k, v, Wq, Wk, dt=dt, A_log=A, dt_scaled_input=True)
    ref = oracle_mod.scan_recurrent_ext(oracle_mod.featmap(q, Wq), oracle_mod.featmap(k, Wk), v,
                                        log_a_f=oracle_mod.log_decay_per_feature(dt, A),
                                        in_scale=oracle_mod.step_size(dt))
    np.testing.assert_array_equal(o, ref)


# ---------------------------------------------------------------- rotary embedding on the features

def test_rope_position_zero_is_identity_and_pairs_keep_their_norm(oracle_mod):
    x = rng.normal(size=(5, 12))
    np.testing.assert_array_equal(oracle_mod.rope(x, 0.0), x)
    y = oracle_mod.rope(x, rng.uniform(0, 500, size=5))
    np.testing.assert_allclose(x[:, :6] ** 2 + x[:, 6:] ** 2, y[:, :6] ** 2 + y[:, 6:] ** 2, rtol=1e-12)


def test_rope_closed_forms(oracle_mod):
    # F = 2: a plane rotation by the position itself (theta_0 = base^0 = 1)
    x = np.array([[0.3, -1.2]])
    for t in (0.5, 3.0, 17.0):
        c, s = math.cos(t), math.sin(t)
        np.testing.assert_allclose(oracle_mod.rope(x, t), [[0.3 * c + 1.2 * s, 0.3 * s - 1.2 * c]], rtol=1e-14)
    # F = 4, base 100: pair (0, 2) at angle t, pair (1, 3) at angle t * 100^(-1/2) = t / 10
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    t = 2.0
    y = oracle_mod.rope(x, t, base=100.0)
    a0, a1 = t, t / 10
    ref = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
           1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    np.testing.assert_allclose(y[0], ref, rtol=1e-14)


def test_rope_composes_and_depends_on_relative_position(oracle_mod):
    x, y = rng.normal(size=(4, 16)), rng.normal(size=(4, 16))
    t, s, d = 7.0, 3.0, 41.0
    np.testing.assert_allclose(oracle_mod.rope(oracle_mod.rope(x, t), s), oracle_mod.rope(x, t + s),
                               rtol=1e-11, atol=1e-12)
    dot1 = np.sum(oracle_mod.rope(x, t) * oracle_mod.rope(y, s), axis=-1)
    dot2 = np.sum(oracle_mod.rope(x, t + d) * oracle_mod.rope(y, s + d), axis=-1)
    np.testing.assert_allclose(dot1, dot2, rtol=1e-11, atol=1e-12)


def test_rope_scan_split_with_carried_state_and_position_offset(oracle_mod):
    # running [0, L1) then [L1, L) from the carried state at positions L1.. equals one pass
    B, L, H, d, p, dv, L1 = 2, 40, 2, 8, 4, 3, 17
    q, k = rng.normal(size=(B, L, H, d)), rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, dv))
    Wq, Wk = rng.normal(size=(p, d)) / 4, rng.normal(size=(p, d)) / 4
    dt = rng.normal(size=(B, L, H)) + 2.0       # strong decay keeps the denominators positive
    A = np.array([0.5, 1.0])
    kw = dict(W_q=Wq, W_k=Wk, A_log=A, rope_base=10000.0)
    o = oracle_mod.scan_fwd(q, k, v, dt=dt, **kw)
    o1, S1, z1 = oracle_mod.scan_fwd(q[:, :L1], k[:, :L1], v[:, :L1], dt=dt[:, :L1], return_state=True, **kw)
    o2 = oracle_mod.scan_fwd(q[:, L1:], k[:, L1:], v[:, L1:], dt=dt[:, L1:], S0=S1, z0=z1, pos0=L1, **kw)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-11, atol=1e-12)
    # and the rotation is really applied: without it the outputs differ
    assert not np.allclose(oracle_mod.scan_fwd(q, k, v, dt=dt, W_q=Wq, W_k=Wk, A_log=A), o)
