"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a closed
form, an invariant the pages' definitions imply, a special case that reduces
to a textbook formula or a library routine, or an independent formulation of
the same quantity.  Together they are chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one in the decay) fails at least one of them.

Pages: HedgeMamba explainer (gsyq.cn 1418924) sec. 2.1, 2.3, 3.1, 5.2, 5.3;
linear-attention tutorial (cnblogs 22790249) sec. 2, 3, 4.3; SSM article
(quant67 56-ssm) sec. 3.2, 4.2.
"""
import math

import numpy as np
import pytest

rng = np.random.default_rng(12345)


def _phi_random(shape):
    """Strictly positive feature vectors (what the Hedgehog map produces)."""
    x = rng.random(shape) + 0.05
    return x / x.sum(-1, keepdims=True)


# ---------------------------------------------------------------- softplus / decay

def test_softplus_closed_forms(oracle_mod):
    sp = oracle_mod.softplus
    assert sp(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    for x in (-30.0, -3.0, -0.5, 0.25, 2.0, 40.0, 700.0):
        # softplus(x) - softplus(-x) = x
        assert sp(x) - sp(-x) == pytest.approx(x, rel=1e-13, abs=1e-13)
        # exp(-softplus(x)) = sigmoid(-x) = 1 / (1 + e^x)
        if x < 700:
            assert math.exp(-sp(x)) == pytest.approx(1.0 / (1.0 + math.exp(x)), rel=1e-12)
    assert sp(-800.0) == 0.0 or sp(-800.0) < 1e-300
    assert sp(1e300) == 1e300


def test_log_decay_closed_form(oracle_mod):
    # a = exp(-softplus(dt) e^{A_log}) = (1 + e^{dt})^(-e^{A_log})
    dt = rng.normal(size=(3, 5, 4))
    A_log = rng.uniform(0, math.log(16), size=4)
    la = oracle_mod.log_decay(dt, A_log)
    a = np.exp(la)
    ref = (1.0 + np.exp(dt)) ** (-np.exp(A_log))
    np.testing.assert_allclose(a, ref, rtol=1e-12)
    assert (a > 0).all() and (a < 1).all()
    # stage-1 identity init (exp(A_log) = 0) gives a = 1 exactly
    la0 = oracle_mod.log_decay(dt, np.full(4, -np.inf))
    assert (la0 == 0).all()
    # dt -> +inf gives a = 0 exactly
    la_inf = oracle_mod.log_decay(np.full((1, 1, 4), 1e300), A_log)
    assert (np.exp(la_inf) == 0).all()


# ---------------------------------------------------------------- Hedgehog map

def test_featmap_is_a_distribution_and_pairs_multiply_to_a_constant(oracle_mod):
    x = rng.normal(size=(7, 3, 16))
    W = rng.normal(size=(8, 16)) / 4
    phi = oracle_mod.featmap(x, W, H=3)
    assert phi.shape == (7, 3, 16)
    assert (phi > 0).all()
    np.testing.assert_allclose(phi.sum(-1), 1.0, rtol=1e-14)
    prod = phi[..., :8] * phi[..., 8:]
    np.testing.assert_allclose(prod, prod[..., :1].repeat(8, -1), rtol=1e-12)


def test_featmap_log_ratio_is_twice_the_projection(oracle_mod):
    # phi_f / phi_{f+p} = exp(2 u_f) with u = W x + b: pins orientation of W,
    # the sign of each half and the bias, against a library matmul
    x = rng.normal(size=(11, 24))
    W = rng.normal(size=(6, 24)) / 5
    b = rng.normal(size=6)
    phi = oracle_mod.featmap(x, W, bias=b)
    u = x @ W.T + b
    np.testing.assert_allclose(np.log(phi[:, :6] / phi[:, 6:]), 2 * u, rtol=1e-12, atol=1e-12)


def test_featmap_one_dim_is_a_logistic(oracle_mod):
    # d = p = 1: phi = [sigmoid(2u), sigmoid(-2u)], u = w x + b
    for w, b, x in ((0.7, 0.0, 1.3), (-2.0, 0.5, 0.25), (3.0, -1.0, -4.0)):
        phi = oracle_mod.featmap(np.array([[x]]), np.array([[w]]), bias=np.array([b]))
        u = w * x + b
        assert phi[0, 0] == pytest.approx(1 / (1 + math.exp(-2 * u)), rel=1e-14)
        assert phi[0, 1] == pytest.approx(1 / (1 + math.exp(2 * u)), rel=1e-14)


def test_featmap_zero_weight_is_uniform_and_negation_swaps_halves(oracle_mod):
    x = rng.normal(size=(5, 12))
    phi0 = oracle_mod.featmap(x, np.zeros((4, 12)))
    np.testing.assert_allclose(phi0, 1.0 / 8, rtol=1e-15)
    W = rng.normal(size=(4, 12))
    a = oracle_mod.featmap(x, W)
    b = oracle_mod.featmap(-x, W)
    np.testing.assert_allclose(b, np.concatenate([a[:, 4:], a[:, :4]], -1), rtol=1e-13)


def test_featmap_per_head_weights(oracle_mod):
    H, d, p = 3, 8, 4
    x = rng.normal(size=(2, 5, H, d))
    W = rng.normal(size=(H, p, d))
    phi = oracle_mod.featmap(x, W, H=H, w_head_stride=p * d)
    for h in range(H):
        ref = oracle_mod.featmap(x[:, :, h], W[h])
        np.testing.assert_allclose(phi[:, :, h], ref, rtol=1e-14)


def test_featmap_per_head_bias_log_ratio(oracle_mod):
    # per-head weights and biases (a bias has the per-head layout of its
    # weights: one [p] row per head): for each head h,
    # log(phi_f / phi_{f+p}) = 2 (W_h x + b_h)_f, against a library matmul
    H, d, p = 3, 10, 4
    x = rng.normal(size=(2, 7, H, d))
    W = rng.normal(size=(H, p, d)) / 3
    b = rng.normal(size=(H, p))
    phi = oracle_mod.featmap(x, W, bias=b, H=H, w_head_stride=p * d, b_head_stride=p)
    for h in range(H):
        u = x[:, :, h] @ W[h].T + b[h]
        np.testing.assert_allclose(np.log(phi[:, :, h, :p] / phi[:, :, h, p:]), 2 * u,
                                   rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- the scan

def _tiny_case(B=2, L=13, H=2, F=6, dv=3, decay=True, zero_at=None):
    phq = _phi_random((B, L, H, F))
    phk = _phi_random((B, L, H, F))
    v = rng.normal(size=(B, L, H, dv))
    la = -rng.exponential(0.7, size=(B, L, H)) if decay else None
    if zero_at is not None:
        la[:, zero_at, :] = -np.inf
    return phq, phk, v, la


@pytest.mark.parametrize("decay", [False, True])
def test_recurrence_equals_quadratic_masked_form(oracle_mod, decay):
    phq, phk, v, la = _tiny_case(decay=decay)
    o_rec = oracle_mod.scan_recurrent(phq, phk, v, la)
    o_quad = oracle_mod.scan_quadratic(phq, phk, v, la)
    np.testing.assert_allclose(o_rec, o_quad, rtol=1e-11, atol=1e-12)


def test_recurrence_with_a_zero_decay_resets(oracle_mod):
    phq, phk, v, la = _tiny_case(L=16, zero_at=9)
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    np.testing.assert_allclose(o, oracle_mod.scan_quadratic(phq, phk, v, la), rtol=1e-11, atol=1e-12)
    # with a_9 = 0 the output at t = 9 is exactly v_9
    np.testing.assert_allclose(o[:, 9], v[:, 9], rtol=1e-13, atol=1e-14)
    # and tokens before 9 no longer influence outputs from 9 on
    phq2, phk2, v2 = phq.copy(), phk.copy(), v.copy()
    phk2[:, :9] = _phi_random(phk2[:, :9].shape)
    v2[:, :9] = rng.normal(size=v2[:, :9].shape)
    o2 = oracle_mod.scan_recurrent(phq2, phk2, v2, la)
    np.testing.assert_allclose(o2[:, 9:], o[:, 9:], rtol=1e-12, atol=1e-13)


def test_all_zero_decay_returns_v(oracle_mod):
    phq, phk, v, _ = _tiny_case(decay=False)
    la = np.full(v.shape[:3], -np.inf)
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    np.testing.assert_allclose(o, v, rtol=1e-13, atol=1e-14)


def test_associativity_identity_without_decay(oracle_mod):
    # a = 1: o = phiQ cumsum_t(phiK^T V) / phiQ cumsum_t(phiK)   (matrix form)
    phq, phk, v, _ = _tiny_case(decay=False, L=21)
    o = oracle_mod.scan_recurrent(phq, phk, v, None)
    KV = np.cumsum(np.einsum("blhf,blhc->blhfc", phk, v), axis=1)
    Kc = np.cumsum(phk, axis=1)
    num = np.einsum("blhf,blhfc->blhc", phq, KV)
    den = np.einsum("blhf,blhf->blh", phq, Kc)
    np.testing.assert_allclose(o, num / den[..., None], rtol=1e-12)


def test_constant_decay_matches_retnet_matrix_form(oracle_mod):
    # a_t = gamma: weights gamma^(i-j) (phiq_i . phik_j) on j <= i
    B, L, H, F, dv = 1, 17, 3, 5, 4
    phq, phk = _phi_random((B, L, H, F)), _phi_random((B, L, H, F))
    v = rng.normal(size=(B, L, H, dv))
    gamma = 0.83
    la = np.full((B, L, H), math.log(gamma))
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    i = np.arange(L)
    D = np.where(i[:, None] >= i[None, :], gamma ** (i[:, None] - i[None, :]).clip(0), 0.0)
    for h in range(H):
        Wt = (phq[0, :, h] @ phk[0, :, h].T) * D
        ref = (Wt @ v[0, :, h]) / Wt.sum(1, keepdims=True)
        np.testing.assert_allclose(o[0, :, h], ref, rtol=1e-12)


def test_two_token_closed_form(oracle_mod):
    # F = 1: o_1 = v_1, o_2 = (a k1 v1 + k2 v2) / (a k1 + k2)
    k1, k2, q1, q2, v1, v2, a2 = 0.3, 0.9, 0.4, 0.7, 2.0, -1.0, 0.25
    phq = np.array([q1, q2]).reshape(1, 2, 1, 1)
    phk = np.array([k1, k2]).reshape(1, 2, 1, 1)
    v = np.array([v1, v2]).reshape(1, 2, 1, 1)
    la = np.log(np.array([0.5, a2])).reshape(1, 2, 1)
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    assert o[0, 0, 0, 0] == pytest.approx(v1, rel=1e-15)
    assert o[0, 1, 0, 0] == pytest.approx((a2 * k1 * v1 + k2 * v2) / (a2 * k1 + k2), rel=1e-14)


def test_outputs_are_convex_combinations_and_constant_v_is_returned(oracle_mod):
    phq, phk, v, la = _tiny_case(L=30)
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    run_min = np.minimum.accumulate(v, axis=1)
    run_max = np.maximum.accumulate(v, axis=1)
    assert (o >= run_min - 1e-12).all() and (o <= run_max + 1e-12).all()
    c = np.broadcast_to(rng.normal(size=(1, 1, 2, 3)), v.shape).copy()
    oc = oracle_mod.scan_recurrent(phq, phk, c, la)
    np.testing.assert_allclose(oc, c, rtol=1e-13, atol=1e-14)


def test_uniform_features_give_prefix_mean(oracle_mod):
    # W = 0 -> phi uniform -> with a = 1, o_t = mean(v_1..v_t)
    B, L, H, d, dv = 1, 19, 2, 8, 3
    q = rng.normal(size=(B, L, H, d))
    k = rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, dv))
    o = oracle_mod.scan_fwd(q, k, v, W_q=np.zeros((4, d)), W_k=np.zeros((4, d)))
    ref = np.cumsum(v, axis=1) / np.arange(1, L + 1)[None, :, None, None]
    np.testing.assert_allclose(o, ref, rtol=1e-13)


def test_query_scale_invariance(oracle_mod):
    phq, phk, v, la = _tiny_case()
    o = oracle_mod.scan_recurrent(phq, phk, v, la)
    scale = rng.uniform(0.1, 10, size=phq.shape[:3] + (1,))
    o2 = oracle_mod.scan_recurrent(phq * scale, phk, v, la)
    np.testing.assert_allclose(o2, o, rtol=1e-12)


@pytest.mark.parametrize("split", [1, 5, 12])
def test_split_with_carried_state_equals_one_pass(oracle_mod, split):
    # affine-map composition is associative: running [0, s) then [s, L) from
    # the carried (S, z) equals one pass over [0, L)
    phq, phk, v, la = _tiny_case(L=13)
    o, S, z = oracle_mod.scan_recurrent(phq, phk, v, la, return_state=True)
    o1, S1, z1 = oracle_mod.scan_recurrent(phq[:, :split], phk[:, :split], v[:, :split],
                                           la[:, :split], return_state=True)
    o2, S2, z2 = oracle_mod.scan_recurrent(phq[:, split:], phk[:, split:], v[:, split:],
                                           la[:, split:], S0=S1, z0=z1, return_state=True)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, rtol=1e-12)
    np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(z2, z, rtol=1e-12)


def test_end_state_closed_form(oracle_mod):
    # S_L = sum_j exp(sum_{j<t<=L} l_t) phik_j v_j^T, z_L likewise
    phq, phk, v, la = _tiny_case(L=9)
    _, S, z = oracle_mod.scan_recurrent(phq, phk, v, la, return_state=True)
    B, L, H, F = phk.shape
    for b in range(B):
        for h in range(H):
            w = np.array([math.exp(la[b, j + 1:, h].sum()) for j in range(L)])
            np.testing.assert_allclose(S[b, h], np.einsum("j,jf,jc->fc", w, phk[b, :, h], v[b, :, h]),
                                       rtol=1e-12)
            np.testing.assert_allclose(z[b, h], w @ phk[b, :, h], rtol=1e-12)


def test_decode_steps_continue_the_prefill(oracle_mod):
    phq, phk, v, la = _tiny_case(L=15)
    o_full = oracle_mod.scan_recurrent(phq, phk, v, la)
    _, S, z = oracle_mod.scan_recurrent(phq[:, :10], phk[:, :10], v[:, :10], la[:, :10],
                                        return_state=True)
    for t in range(10, 15):
        o_t, S, z = oracle_mod.decode_step(phq[:, t], phk[:, t], v[:, t], S, z, la[:, t])
        np.testing.assert_allclose(o_t, o_full[:, t], rtol=1e-12)


# ---------------------------------------------------------------- conv, gate, mixer

def test_causal_conv_matches_library_convolution(oracle_mod):
    B, L, C, K = 2, 11, 3, 4
    x = rng.normal(size=(B, L, C))
    w = rng.normal(size=(C, K))
    bias = rng.normal(size=C)
    y = oracle_mod.causal_conv(x, w, bias)
    for b in range(B):
        for c in range(C):
            # y_t = sum_j w[j] x_{t-(K-1)+j}: a full convolution with the
            # reversed kernel, first L outputs
            ref = np.convolve(x[b, :, c], w[c, ::-1])[:L] + bias[c]
            np.testing.assert_allclose(y[b, :, c], ref, rtol=1e-13, atol=1e-13)
    ident = np.zeros((C, K))
    ident[:, -1] = 1.0
    np.testing.assert_array_equal(oracle_mod.causal_conv(x, ident), x)
    shift = np.zeros((C, K))
    shift[:, 0] = 1.0
    ys = oracle_mod.causal_conv(x, shift)
    np.testing.assert_array_equal(ys[:, 3:], x[:, :-3])
    assert (ys[:, :3] == 0).all()


def _silu_inverse_of_one():
    # solve x * sigmoid(x) = 1 by bisection
    lo, hi = 0.0, 3.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mid / (1 + math.exp(-mid)) < 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_silu_and_its_inverse_at_one(oracle_mod):
    x0 = _silu_inverse_of_one()
    assert x0 == pytest.approx(1.2784645427610738, rel=1e-12)
    assert oracle_mod.silu(np.array([x0]))[0] == pytest.approx(1.0, rel=1e-14)
    assert oracle_mod.silu(np.array([0.0]))[0] == 0.0


def _mixer_weights(D, H, dh, p, K):
    E = H * dh
    return dict(
        W_q=rng.normal(size=(E, D)) / math.sqrt(D), W_k=rng.normal(size=(E, D)) / math.sqrt(D),
        W_v=rng.normal(size=(E, D)) / math.sqrt(D), W_g=rng.normal(size=(E, D)) / math.sqrt(D),
        W_dt=rng.normal(size=(H, D)) / math.sqrt(D), conv_w=rng.normal(size=(3, E, K)) / 2,
        W_hq=rng.normal(size=(p, dh)) / math.sqrt(dh), W_hk=rng.normal(size=(p, dh)) / math.sqrt(dh),
        A_log=rng.uniform(0, math.log(16), size=H), W_o=rng.normal(size=(D, E)) / math.sqrt(E))


def test_mixer_stage1_identity_reduces_to_linear_attention(oracle_mod):
    # HedgeMamba sec. 3.1: a = 1 (exp(A_log) = 0), conv kernel [0,..,0,1],
    # gate weights 0 with bias SiLU^-1(1) -> mixer = out_proj(LA(q, k, v))
    B, L, D, H, dh, p, K = 2, 9, 16, 2, 8, 4, 4
    w = _mixer_weights(D, H, dh, p, K)
    E = H * dh
    x = rng.normal(size=(B, L, D))
    w["A_log"] = np.full(H, -np.inf)
    w["conv_w"] = np.zeros((3, E, K))
    w["conv_w"][:, :, -1] = 1.0
    w["W_g"] = np.zeros((E, D))
    out = oracle_mod.mixer_fwd(x, n_heads=H, b_g=np.full(E, _silu_inverse_of_one()), **w)
    q = (x @ w["W_q"].T).reshape(B, L, H, dh)
    k = (x @ w["W_k"].T).reshape(B, L, H, dh)
    v = (x @ w["W_v"].T).reshape(B, L, H, dh)
    o = oracle_mod.scan_fwd(q, k, v, W_q=w["W_hq"], W_k=w["W_hk"])
    ref = o.reshape(B, L, E) @ w["W_o"].T
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_mixer_general_composition(oracle_mod):
    # the same wiring with every component active, built from the pinned steps
    B, L, D, H, dh, p, K = 2, 10, 16, 2, 8, 4, 4
    w = _mixer_weights(D, H, dh, p, K)
    E = H * dh
    x = rng.normal(size=(B, L, D))
    out = oracle_mod.mixer_fwd(x, n_heads=H, **w)
    xf = x.reshape(B * L, D)
    qkv = [oracle_mod.causal_conv((xf @ w[n].T).reshape(B, L, E), w["conv_w"][i])
           for i, n in enumerate(("W_q", "W_k", "W_v"))]
    g = xf @ w["W_g"].T
    dt = (xf @ w["W_dt"].T).reshape(B, L, H)
    a = (1.0 + np.exp(dt)) ** (-np.exp(w["A_log"]))   # closed form of the decay
    o = oracle_mod.scan_fwd(*[t.reshape(B, L, H, dh) for t in qkv], W_q=w["W_hq"], W_k=w["W_hk"],
                            dt=dt, A_log=w["A_log"])
    o2 = oracle_mod.scan_recurrent(oracle_mod.featmap(qkv[0].reshape(B, L, H, dh), w["W_hq"]),
                                   oracle_mod.featmap(qkv[1].reshape(B, L, H, dh), w["W_hk"]),
                                   qkv[2].reshape(B, L, H, dh), np.log(a))
    np.testing.assert_allclose(o, o2, rtol=1e-11)
    y = o.reshape(B * L, E) * (g / (1 + np.exp(-g)))
    np.testing.assert_allclose(out.reshape(B * L, D), y @ w["W_o"].T, rtol=1e-11, atol=1e-12)
    # batches are independent: evaluating a subset gives the same rows
    np.testing.assert_allclose(oracle_mod.mixer_fwd(x, n_heads=H, batches=[1], **w)[0], out[1],
                               rtol=1e-12)
