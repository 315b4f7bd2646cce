"""Pins of the oracle's backward pass (CPU, fp64): every gradient against
central finite differences of the forward oracle, the scan's gradients
against autograd of the independent O(L^2) masked form, and exact
invariants of the definition (outputs that do not depend on an input give a
zero gradient; degree-0 homogeneity gives Euler identities)."""
import numpy as np
import pytest
import torch

import workloads as wl


def _rand(seed, name, shape, std=1.0):
    return wl.normal(seed, name, shape, std=std)


def _tiny(seed=0, B=1, L=6, H=2, d=4, p=3, dv=3):
    return dict(q=_rand(seed, "q", (B, L, H, d)), k=_rand(seed, "k", (B, L, H, d)),
                v=_rand(seed, "v", (B, L, H, dv)), W_q=_rand(seed, "Wq", (p, d), 0.5),
                W_k=_rand(seed, "Wk", (p, d), 0.5), dt=_rand(seed, "dt", (B, L, H)),
                A_log=wl.uniform(seed, "A", (H,), 0.0, 1.0), do=_rand(seed, "do", (B, L, H, dv)))


def _loss(oracle_mod, x):
    o = oracle_mod.scan_fwd(x["q"], x["k"], x["v"], x["W_q"], x["W_k"], dt=x["dt"], A_log=x["A_log"])
    return float(np.sum(x["do"] * o))


@pytest.mark.parametrize("name,key", [("q", "dq"), ("k", "dk"), ("v", "dv"), ("W_q", "dW_q"),
                                      ("W_k", "dW_k"), ("dt", "ddt"), ("A_log", "dA_log")])
def test_scan_gradients_match_finite_differences(oracle_mod, name, key):
    x = _tiny()
    g = oracle_mod.scan_bwd(x["q"], x["k"], x["v"], x["W_q"], x["W_k"], x["do"], dt=x["dt"], A_log=x["A_log"])[key]
    h = 1e-6
    num = np.zeros_like(x[name])
    flat = x[name].reshape(-1)
    for i in range(flat.size):
        keep = flat[i]
        flat[i] = keep + h
        lp = _loss(oracle_mod, x)
        flat[i] = keep - h
        lm = _loss(oracle_mod, x)
        flat[i] = keep
        num.reshape(-1)[i] = (lp - lm) / (2 * h)
    np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


def test_state_gradients_match_finite_differences(oracle_mod):
    x = _tiny(seed=1)
    phq, phk = oracle_mod.featmap(x["q"], x["W_q"]), oracle_mod.featmap(x["k"], x["W_k"])
    la = oracle_mod.log_decay(x["dt"], x["A_log"])
    F, dv = phq.shape[-1], x["v"].shape[-1]
    S0 = np.abs(_rand(1, "S0", (1, 2, F, dv), 0.3))
    z0 = np.abs(_rand(1, "z0", (1, 2, F))) + 0.2
    _, _, _, _, dS0, dz0 = oracle_mod.scan_recurrent_bwd(phq, phk, x["v"], x["do"], la, S0, z0)
    h = 1e-6
    for arr, grad in ((S0, dS0), (z0, dz0)):
        num = np.zeros_like(arr)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = np.sum(x["do"] * oracle_mod.scan_recurrent(phq, phk, x["v"], la, S0, z0))
            flat[i] = keep - h
            lm = np.sum(x["do"] * oracle_mod.scan_recurrent(phq, phk, x["v"], la, S0, z0))
            flat[i] = keep
            num.reshape(-1)[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def _quadratic_torch(phq, phk, v, la):
    # o_i = sum_{j<=i} w_ij v_j / sum_{j<=i} w_ij,  w_ij = exp(sum_{j<t<=i} l_t) phq_i . phk_j
    c = torch.cumsum(la, dim=1)                                   # [B, L, H]
    dec = c[:, :, None, :] - c[:, None, :, :]                     # [B, i, j, H]
    L = phq.shape[1]
    mask = torch.tril(torch.ones(L, L, dtype=torch.bool))[None, :, :, None]
    e = torch.where(mask, torch.exp(torch.where(mask, dec, torch.zeros_like(dec))), torch.zeros_like(dec))
    s = torch.einsum("bihf,bjhf->bijh", phq, phk) * e
    return torch.einsum("bijh,bjhv->bihv", s, v) / s.sum(dim=2)[..., None]


def test_scan_gradients_match_autograd_of_the_quadratic_form(oracle_mod):
    B, L, H, F, dv = 2, 9, 3, 5, 4
    phq = np.exp(_rand(2, "pq", (B, L, H, F), 0.5))
    phk = np.exp(_rand(2, "pk", (B, L, H, F), 0.5))
    v = _rand(2, "v", (B, L, H, dv))
    la = -np.abs(_rand(2, "la", (B, L, H), 0.7))
    do = _rand(2, "do", (B, L, H, dv))
    g = oracle_mod.scan_recurrent_bwd(phq, phk, v, do, la)
    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (phq, phk, v, la)]
    o = _quadratic_torch(*t)
    (o * torch.tensor(do)).sum().backward()
    for ours, ref in zip(g[:4], t):
        np.testing.assert_allclose(ours, ref.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_constant_values_give_zero_weight_gradients(oracle_mod):
    # o_t = c whatever the weights when every v_t = c (convex combination)
    B, L, H, F, dv = 1, 8, 2, 6, 3
    phq = np.exp(_rand(3, "pq", (B, L, H, F)))
    phk = np.exp(_rand(3, "pk", (B, L, H, F)))
    c = _rand(3, "c", (1, 1, H, dv))
    v = np.broadcast_to(c, (B, L, H, dv)).copy()
    la = -np.abs(_rand(3, "la", (B, L, H)))
    do = _rand(3, "do", (B, L, H, dv))
    dphq, dphk, dv_, dla, _, _ = oracle_mod.scan_recurrent_bwd(phq, phk, v, do, la)
    np.testing.assert_allclose(dphq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dphk, 0.0, atol=1e-12)
    np.testing.assert_allclose(dla, 0.0, atol=1e-12)
    # the value gradients still carry do: sum over t of dv_t = sum over t of do_t
    np.testing.assert_allclose(dv_.sum(axis=1), do.sum(axis=1), rtol=1e-10)


def test_homogeneity_gives_euler_identities(oracle_mod):
    # o_t is unchanged by phq_t -> c phq_t, and (zero initial state) by scaling every phk
    B, L, H, F, dv = 2, 7, 2, 5, 3
    phq = np.exp(_rand(4, "pq", (B, L, H, F)))
    phk = np.exp(_rand(4, "pk", (B, L, H, F)))
    v = _rand(4, "v", (B, L, H, dv))
    la = -np.abs(_rand(4, "la", (B, L, H)))
    do = _rand(4, "do", (B, L, H, dv))
    dphq, dphk, _, _, _, _ = oracle_mod.scan_recurrent_bwd(phq, phk, v, do, la)
    np.testing.assert_allclose(np.sum(dphq * phq, axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(np.sum(dphk * phk, axis=(1, 3)), 0.0, atol=1e-11)


def test_featmap_gradient(oracle_mod):
    x = _rand(5, "x", (7, 4))
    W = _rand(5, "W", (3, 4), 0.6)
    dphi = _rand(5, "dphi", (7, 6))
    dx, dW, db = oracle_mod.featmap_bwd(x, W, dphi)
    h = 1e-6
    for arr, grad in ((x, dx), (W, dW)):
        num = np.zeros_like(arr)
        flat = arr.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = np.sum(dphi * oracle_mod.featmap(x, W))
            flat[i] = keep - h
            lm = np.sum(dphi * oracle_mod.featmap(x, W))
            flat[i] = keep
            num.reshape(-1)[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)
    # a constant upstream gradient meets a distribution: nothing flows back
    dx0, dW0, db0 = oracle_mod.featmap_bwd(x, W, np.full((7, 6), 0.37))
    np.testing.assert_allclose(dx0, 0.0, atol=1e-14)
    np.testing.assert_allclose(db0, 0.0, atol=1e-14)


def test_log_decay_gradient(oracle_mod):
    dt = _rand(6, "dt", (3, 5, 4), 2.0)
    A_log = wl.uniform(6, "A", (4,), -1.0, 2.0)
    g = _rand(6, "g", (3, 5, 4))
    ddt, dA = oracle_mod.log_decay_bwd(dt, A_log, g)
    h = 1e-6
    f = lambda a, b: np.sum(g * oracle_mod.log_decay(a, b))
    num = np.array([(f(dt, A_log + h * e) - f(dt, A_log - h * e)) / (2 * h) for e in np.eye(4)])
    np.testing.assert_allclose(dA, num, rtol=1e-7)
    i = (1, 2, 3)
    e = np.zeros_like(dt)
    e[i] = h
    np.testing.assert_allclose(ddt[i], (f(dt + e, A_log) - f(dt - e, A_log)) / (2 * h), rtol=1e-6)
