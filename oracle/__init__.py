"""fp64 CPU oracle for the HedgeMamba mixer scan.

TEST INFRASTRUCTURE ONLY.  The product (the CUDA library under
``selective_ssm_sequence_b200`` and its binding) never imports, loads or calls
anything in this package, and this package never imports the product.  The
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg are
the only callers.

The loops live in ``hm_oracle.c`` (plain C, double precision).  This module
builds it with gcc, wraps it with ctypes and composes the mixer from those
steps plus numpy matmuls (a library matmul is a single step of the mixer's
definition; nothing is blocked or fused).

Page citations (see ``hm_oracle.c`` for the full list):
  [HM]  HedgeMamba explainer (gsyq.cn 1418924): sec. 2.1 Hedgehog map,
        sec. 2.3 / 5.2 mixer, sec. 3.1 stage-1 identity init, sec. 5.3 map listing.
  [LA]  Linear-attention tutorial (cnblogs 22790249): sec. 2 kernel form and
        associativity, sec. 3 recurrent form, sec. 4.3 RetNet decay.
  [SSM] SSM article (quant67 56-ssm): sec. 3.2 softplus dt, sec. 4.2 affine
        composition, sec. 4.3 states recomputed in the backward pass.
  [HM] sec. 5.1 also gives the block around the mixer: GPT-NeoX's parallel
        residual block, x + mixer(norm1 x) + mlp(norm2 x) (``block_fwd``).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(forward) and ``tests/test_oracle_backward_pins.py`` (backward) against closed
forms, invariants, finite differences, a brute-force rational-arithmetic
evaluation or an independent formulation.  End-to-end numeric values are not printed on
the pages (no worked example), so absolute values rest on those pins.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hm_oracle.c")
_LIB = os.path.join(_HERE, "_hm_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile hm_oracle.c into a shared object next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.hmo_softplus.restype = ctypes.c_double
        lib.hmo_softplus.argtypes = [ctypes.c_double]
        lib.hmo_log_decay.restype = None
        lib.hmo_log_decay.argtypes = [P, I64, I, P, P]
        lib.hmo_featmap.restype = None
        lib.hmo_featmap.argtypes = [P, I64, I, I, I, P, I64, P, I64, P]
        lib.hmo_scan_recurrent.restype = I64
        lib.hmo_scan_recurrent.argtypes = [I64, I64, I, I, I, P, P, P, P, P, P, P, P, P]
        lib.hmo_scan_quadratic.restype = None
        lib.hmo_scan_quadratic.argtypes = [I64, I64, I, I, I, P, P, P, P, P]
        lib.hmo_decode_step.restype = I64
        lib.hmo_decode_step.argtypes = [I64, I, I, I, P, P, P, P, P, P, P]
        lib.hmo_scan_recurrent_ext.restype = I64
        lib.hmo_scan_recurrent_ext.argtypes = [I64, I64, I, I, I, P, P, P, P, P, P, P, P, P, P, P]
        lib.hmo_scan_quadratic_ext.restype = None
        lib.hmo_scan_quadratic_ext.argtypes = [I64, I64, I, I, I, P, P, P, P, P, P, P]
        lib.hmo_log_decay_f.restype = None
        lib.hmo_log_decay_f.argtypes = [P, I64, I, I, P, P]
        lib.hmo_step_size.restype = None
        lib.hmo_step_size.argtypes = [P, I64, P]
        lib.hmo_rope.restype = None
        lib.hmo_rope.argtypes = [P, I64, I, P, ctypes.c_double, P]
        lib.hmo_causal_conv.restype = None
        lib.hmo_causal_conv.argtypes = [I64, I64, I, I, P, P, P, P]
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    """Bound the OpenMP team used by the oracle loops (call before first use)."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))


# --------------------------------------------------------------------------
# single steps
# --------------------------------------------------------------------------

def softplus(x: float) -> float:
    """log(1 + e^x) ([SSM] sec. 3.2: dt goes through softplus)."""
    return _load().hmo_softplus(float(x))


def log_decay(dt, A_log):
    """l[b,t,h] = -softplus(dt[b,t,h]) * exp(A_log[h]); a = exp(l).

    dt: [..., H]; A_log: [H].  Returns an array shaped like dt."""
    dt = _f64(dt)
    A_log = _f64(A_log)
    H = A_log.shape[0]
    assert dt.shape[-1] == H
    out = np.empty_like(dt)
    _load().hmo_log_decay(_ptr(dt), dt.size // H, H, _ptr(A_log), _ptr(out))
    return out


def featmap(x, W, bias=None, H=1, w_head_stride=0, b_head_stride=0):
    """Hedgehog map phi = softmax([W x + b, -(W x + b)]) over 2p features
    ([HM] sec. 2.1, 5.3).  x: [..., d] (row r is head r mod H); W: [p, d]
    (or [H, p, d] with w_head_stride = p*d).  Returns [..., 2p]."""
    x = _f64(x)
    W = _f64(W)
    d = x.shape[-1]
    p = W.shape[-2]
    assert W.shape[-1] == d
    rows = x.size // d
    b = None if bias is None else _f64(bias)
    out = np.empty(x.shape[:-1] + (2 * p,), dtype=np.float64)
    _load().hmo_featmap(_ptr(x), rows, int(H), d, p, _ptr(W), int(w_head_stride),
                        _ptr(b), int(b_head_stride), _ptr(out))
    return out


def scan_recurrent(phq, phk, v, log_a=None, S0=None, z0=None, return_state=False):
    """Decayed normalised recurrence (spec definition):
    S_t = a_t S_{t-1} + phik_t v_t^T, z_t = a_t z_{t-1} + phik_t,
    o_t = phiq_t^T S_t / phiq_t^T z_t.  phq, phk: [B, L, H, F]; v: [B, L, H, dv];
    log_a: [B, L, H] or None (a = 1).  Raises if any denominator is <= 0."""
    phq, phk, v = _f64(phq), _f64(phk), _f64(v)
    B, L, H, F = phq.shape
    dv = v.shape[-1]
    assert phk.shape == phq.shape and v.shape[:3] == (B, L, H)
    la = None if log_a is None else _f64(log_a)
    if la is not None:
        assert la.shape == (B, L, H)
    S0a = None if S0 is None else _f64(S0)
    z0a = None if z0 is None else _f64(z0)
    o = np.empty((B, L, H, dv), dtype=np.float64)
    S_out = np.empty((B, H, F, dv), dtype=np.float64)
    z_out = np.empty((B, H, F), dtype=np.float64)
    bad = _load().hmo_scan_recurrent(B, L, H, F, dv, _ptr(phq), _ptr(phk), _ptr(v),
                                     _ptr(la), _ptr(S0a), _ptr(z0a), _ptr(o),
                                     _ptr(S_out), _ptr(z_out))
    if bad:
        raise FloatingPointError("oracle: %d denominators were not > 0" % bad)
    if return_state:
        return o, S_out, z_out
    return o


def rope(x, pos, base=10000.0):
    """Rotary embedding of feature vectors ([HM] sec. 5.2, RoPE on phi(Q),
    phi(K)); "rotate half" pairing (i, i + F/2), angle pos * base^(-2i/F).
    x: [..., F]; pos: broadcastable to x.shape[:-1] (absolute positions)."""
    x = _f64(x)
    F = x.shape[-1]
    assert F % 2 == 0
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), x.shape[:-1]))
    out = np.empty_like(x)
    _load().hmo_rope(_ptr(x), x.size // F, F, _ptr(p), float(base), _ptr(out))
    return out


def token_positions(B, L, H, pos0=0):
    """Absolute position of every (b, t, h) row of a [B, L, H, *] tensor: pos0 + t."""
    t = np.arange(L, dtype=np.float64) + float(pos0)
    return np.broadcast_to(t[None, :, None], (B, L, H))


def log_decay_per_feature(dt, A_log_f):
    """l[b,t,h,f] = -softplus(dt[b,t,h]) * exp(A_log_f[h,f]) (the per-feature
    decay variant; [LA] sec. 4.4).  dt: [..., H]; A_log_f: [H, F]."""
    dt = _f64(dt)
    A = _f64(A_log_f)
    H, F = A.shape
    assert dt.shape[-1] == H
    out = np.empty(dt.shape + (F,), dtype=np.float64)
    _load().hmo_log_decay_f(_ptr(dt), dt.size // H, H, F, _ptr(A), _ptr(out))
    return out


def step_size(dt):
    """Delta = softplus(dt) ([SSM] sec. 3.2), elementwise."""
    dt = _f64(dt)
    out = np.empty_like(dt)
    _load().hmo_step_size(_ptr(dt), dt.size, _ptr(out))
    return out


def scan_recurrent_ext(phq, phk, v, log_a=None, log_a_f=None, in_scale=None, S0=None, z0=None,
                       return_state=False):
    """The recurrence with the step-scaled input (in_scale = Delta, [HM]
    sec. 5.2 / [SSM] sec. 3.2) and/or a per-feature decay (log_a_f
    [B, L, H, F], [LA] sec. 4.4); see hmo_scan_recurrent_ext."""
    phq, phk, v = _f64(phq), _f64(phk), _f64(v)
    B, L, H, F = phq.shape
    dv = v.shape[-1]
    la = None if log_a is None else _f64(log_a)
    laf = None if log_a_f is None else _f64(log_a_f)
    sc = None if in_scale is None else _f64(in_scale)
    S0 = None if S0 is None else _f64(S0)
    z0 = None if z0 is None else _f64(z0)
    o = np.empty((B, L, H, dv), dtype=np.float64)
    S = np.empty((B, H, F, dv), dtype=np.float64) if return_state else None
    z = np.empty((B, H, F), dtype=np.float64) if return_state else None
    bad = _load().hmo_scan_recurrent_ext(B, L, H, F, dv, _ptr(phq), _ptr(phk), _ptr(v), _ptr(la),
                                         _ptr(laf), _ptr(sc), _ptr(S0), _ptr(z0), _ptr(o), _ptr(S),
                                         _ptr(z))
    if bad:
        raise FloatingPointError("oracle: %d denominators were not > 0" % bad)
    return (o, S, z) if return_state else o


def scan_quadratic_ext(phq, phk, v, log_a=None, log_a_f=None, in_scale=None):
    """O(L^2) masked form of scan_recurrent_ext (zero initial state)."""
    phq, phk, v = _f64(phq), _f64(phk), _f64(v)
    B, L, H, F = phq.shape
    dv = v.shape[-1]
    la = None if log_a is None else _f64(log_a)
    laf = None if log_a_f is None else _f64(log_a_f)
    sc = None if in_scale is None else _f64(in_scale)
    o = np.empty((B, L, H, dv), dtype=np.float64)
    _load().hmo_scan_quadratic_ext(B, L, H, F, dv, _ptr(phq), _ptr(phk), _ptr(v), _ptr(la), _ptr(laf),
                                   _ptr(sc), _ptr(o))
    return o


def scan_quadratic(phq, phk, v, log_a=None):
    """O(L^2) masked form ([LA] sec. 2): o_i = sum_{j<=i} w_ij v_j / sum_j w_ij,
    w_ij = exp(sum_{j<t<=i} l_t) phiq_i . phik_j.  Zero initial state."""
    phq, phk, v = _f64(phq), _f64(phk), _f64(v)
    B, L, H, F = phq.shape
    dv = v.shape[-1]
    la = None if log_a is None else _f64(log_a)
    o = np.empty((B, L, H, dv), dtype=np.float64)
    _load().hmo_scan_quadratic(B, L, H, F, dv, _ptr(phq), _ptr(phk), _ptr(v), _ptr(la), _ptr(o))
    return o


def decode_step(phq, phk, v, S, z, log_a=None):
    """One recurrent step per (batch, head); returns (o, S_new, z_new).
    phq, phk: [B, H, F]; v: [B, H, dv]; S: [B, H, F, dv]; z: [B, H, F];
    log_a: [B, H] or None."""
    phq, phk, v = _f64(phq), _f64(phk), _f64(v)
    B, H, F = phq.shape
    dv = v.shape[-1]
    S = _f64(S).copy()
    z = _f64(z).copy()
    la = None if log_a is None else _f64(log_a)
    o = np.empty((B, H, dv), dtype=np.float64)
    bad = _load().hmo_decode_step(B, H, F, dv, _ptr(phq), _ptr(phk), _ptr(v), _ptr(la),
                                  _ptr(S), _ptr(z), _ptr(o))
    if bad:
        raise FloatingPointError("oracle: %d denominators were not > 0" % bad)
    return o, S, z


def causal_conv(x, w, bias=None):
    """Depthwise causal conv along the sequence, zero left padding, no
    activation ([HM] sec. 2.3: short conv kept).  x: [B, L, C]; w: [C, K];
    bias: [C] or None."""
    x = _f64(x)
    w = _f64(w)
    B, L, C = x.shape
    K = w.shape[1]
    b = None if bias is None else _f64(bias)
    y = np.empty_like(x)
    _load().hmo_causal_conv(B, L, C, K, _ptr(x), _ptr(w), _ptr(b), _ptr(y))
    return y


def silu(x):
    """SiLU(x) = x * sigmoid(x) (the gate nonlinearity, [HM] sec. 3.1)."""
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


# --------------------------------------------------------------------------
# compositions
# --------------------------------------------------------------------------

def scan_fwd(q, k, v, W_q=None, W_k=None, dt=None, A_log=None, b_q=None, b_k=None,
             S0=None, z0=None, w_head_stride=0, return_state=False, dt_scaled_input=False,
             rope_base=None, pos0=0):
    """Feature map on q and k, then the decayed normalised recurrence.

    q, k: [B, L, H, d]; v: [B, L, H, dv]; W_q, W_k: [p, d] (or per-head); if
    W_q is None, q and k are taken as feature vectors already (F = d).
    dt: [B, L, H] or None (a = 1); A_log: [H], or [H, F] for a decay per
    feature.  dt_scaled_input: the input term is multiplied by Delta =
    softplus(dt) (Mamba's discretised input).  rope_base: rotary embedding of
    phi(q) and phi(k) (rope) at positions pos0 + t; None = off."""
    q, k = _f64(q), _f64(k)
    B, L, H, d = q.shape
    if W_q is None:
        phq, phk = q, k
    else:
        # biases are per head exactly when the weights are (one [p] row per head)
        bstride = W_q.shape[-2] if w_head_stride else 0
        phq = featmap(q, W_q, b_q, H=H, w_head_stride=w_head_stride, b_head_stride=bstride)
        phk = featmap(k, W_k, b_k, H=H, w_head_stride=w_head_stride, b_head_stride=bstride)
    if rope_base is not None:
        pos = token_positions(B, L, H, pos0)
        phq, phk = rope(phq, pos, rope_base), rope(phk, pos, rope_base)
    per_feature = A_log is not None and np.ndim(A_log) == 2
    if not per_feature and not dt_scaled_input:
        la = None if dt is None else log_decay(dt, A_log)
        return scan_recurrent(phq, phk, v, la, S0, z0, return_state=return_state)
    assert dt is not None, "the variants are functions of dt"
    la = None if per_feature else log_decay(dt, A_log)
    laf = log_decay_per_feature(dt, A_log) if per_feature else None
    sc = step_size(dt) if dt_scaled_input else None
    return scan_recurrent_ext(phq, phk, v, log_a=la, log_a_f=laf, in_scale=sc, S0=S0, z0=z0,
                              return_state=return_state)


# --------------------------------------------------------------------------
# backward (the derivative of the forward definition above, by the chain rule;
# the pages train the mixer by distillation, [HM] sec. 3, and Mamba's kernels
# recompute the states in the backward pass, [SSM] sec. 4.3)
# --------------------------------------------------------------------------

def scan_recurrent_bwd(phq, phk, v, do, log_a=None, S0=None, z0=None):
    """Gradients of sum(do * o) for o = scan_recurrent(phq, phk, v, log_a, S0, z0).

    Reverse-mode form of the recurrence, with n_t = S_t^T phq_t, d_t = phq_t . z_t,
    o_t = n_t / d_t and G_t, g_t the total gradients of S_t, z_t:
      dn_t = do_t / d_t,  dd_t = -(do_t . o_t) / d_t
      G_t = phq_t dn_t^T + a_{t+1} G_{t+1},   g_t = phq_t dd_t + a_{t+1} g_{t+1}
      dphq_t = S_t dn_t + z_t dd_t
      dphk_t = G_t v_t + g_t,   dv_t = G_t^T phk_t
      dlog_a_t = a_t (<G_t, S_{t-1}> + g_t . z_{t-1})
      dS0 = a_1 G_1,  dz0 = a_1 g_1
    The forward states are kept for the whole sequence (small cases only).
    Returns (dphq, dphk, dv, dlog_a, dS0, dz0); dlog_a is None without log_a."""
    phq, phk, v, do = _f64(phq), _f64(phk), _f64(v), _f64(do)
    B, L, H, F = phq.shape
    dv_ = v.shape[-1]
    la = None if log_a is None else _f64(log_a)
    a = np.ones((B, L, H)) if la is None else np.exp(la)
    S = np.zeros((B, H, F, dv_)) if S0 is None else _f64(S0).copy()
    z = np.zeros((B, H, F)) if z0 is None else _f64(z0).copy()
    Ss = np.empty((L + 1, B, H, F, dv_))
    zs = np.empty((L + 1, B, H, F))
    Ss[0], zs[0] = S, z
    for t in range(L):
        S = a[:, t, :, None, None] * S + phk[:, t, :, :, None] * v[:, t, :, None, :]
        z = a[:, t, :, None] * z + phk[:, t]
        Ss[t + 1], zs[t + 1] = S, z
    dphq = np.empty_like(phq)
    dphk = np.empty_like(phk)
    dv = np.empty_like(v)
    dla = np.empty((B, L, H))
    G = np.zeros((B, H, F, dv_))
    g = np.zeros((B, H, F))
    for t in range(L - 1, -1, -1):
        St, zt = Ss[t + 1], zs[t + 1]
        num = np.einsum("bhfv,bhf->bhv", St, phq[:, t])
        den = np.einsum("bhf,bhf->bh", zt, phq[:, t])
        if np.any(den <= 0):
            raise FloatingPointError("oracle: a denominator was not > 0")
        o = num / den[..., None]
        dn = do[:, t] / den[..., None]
        dd = -np.einsum("bhv,bhv->bh", do[:, t], o) / den
        if t + 1 < L:
            G = a[:, t + 1, :, None, None] * G
            g = a[:, t + 1, :, None] * g
        G = G + phq[:, t, :, :, None] * dn[:, :, None, :]
        g = g + phq[:, t] * dd[..., None]
        dphq[:, t] = np.einsum("bhfv,bhv->bhf", St, dn) + zt * dd[..., None]
        dphk[:, t] = np.einsum("bhfv,bhv->bhf", G, v[:, t]) + g
        dv[:, t] = np.einsum("bhfv,bhf->bhv", G, phk[:, t])
        dla[:, t] = a[:, t] * (np.einsum("bhfv,bhfv->bh", G, Ss[t]) + np.einsum("bhf,bhf->bh", g, zs[t]))
    dS0 = a[:, 0, :, None, None] * G
    dz0 = a[:, 0, :, None] * g
    return dphq, dphk, dv, (None if la is None else dla), dS0, dz0


def log_decay_bwd(dt, A_log, dlog_a):
    """Gradients of sum(dlog_a * l) for l = log_decay(dt, A_log):
    dl/ddt = -sigmoid(dt) exp(A_log) and dl/dA_log = l.  Returns (ddt, dA_log)."""
    dt, A_log, g = _f64(dt), _f64(A_log), _f64(dlog_a)
    sig = 1.0 / (1.0 + np.exp(-dt))
    ddt = -g * sig * np.exp(A_log)
    dA = np.sum(g * log_decay(dt, A_log), axis=tuple(range(g.ndim - 1)))
    return ddt, dA


def featmap_bwd(x, W, dphi, bias=None):
    """Gradients of sum(dphi * phi) for phi = featmap(x, W, bias) with one W
    shared by every row: with e = [u, -u], u = W x + b and phi = softmax(e),
      de = phi * (dphi - sum(dphi * phi)),  du = de[:p] - de[p:]
      dx = W^T du,  dW = sum over rows du x^T,  db = sum over rows du.
    Returns (dx, dW, db)."""
    x, W, dphi = _f64(x), _f64(W), _f64(dphi)
    p = W.shape[0]
    phi = featmap(x, W, bias)
    de = phi * (dphi - np.sum(dphi * phi, axis=-1, keepdims=True))
    du = de[..., :p] - de[..., p:]
    dx = du @ W
    du2 = du.reshape(-1, p)
    dW = du2.T @ x.reshape(-1, x.shape[-1])
    db = du2.sum(axis=0)
    return dx, dW, db


def scan_bwd(q, k, v, W_q, W_k, do, dt=None, A_log=None):
    """Gradients of sum(do * o) for o = scan_fwd(q, k, v, W_q, W_k, dt, A_log)
    (shared Hedgehog weights, no bias, zero initial state).
    Returns dict with dq, dk, dv, dW_q, dW_k and, with decay, ddt and dA_log."""
    phq = featmap(q, W_q)
    phk = featmap(k, W_k)
    la = None if dt is None else log_decay(dt, A_log)
    dphq, dphk, dv, dla, _, _ = scan_recurrent_bwd(phq, phk, v, do, la)
    dq, dWq, _ = featmap_bwd(q, W_q, dphq)
    dk, dWk, _ = featmap_bwd(k, W_k, dphk)
    out = {"dq": dq, "dk": dk, "dv": dv, "dW_q": dWq, "dW_k": dWk}
    if dt is not None:
        out["ddt"], out["dA_log"] = log_decay_bwd(dt, A_log, dla)
    return out


def mixer_fwd(x, W_q, W_k, W_v, W_g, W_dt, conv_w, W_hq, W_hk, A_log, W_o,
              conv_b=None, b_g=None, b_dt=None, n_heads=8, batches=None):
    """HedgeMamba mixer forward ([HM] sec. 2.3 and 5.2), plain composition:

      q, k, v, g = x W_{q,k,v,g}^T ;  dt = x W_dt^T (+ b_dt)
      q, k, v    = causal depthwise conv (width K) of each, + conv bias
      per head h (d_head = width / H): phi_q = hedgehog(q_h), phi_k = hedgehog(k_h)
      o          = decayed normalised recurrence(phi_q, phi_k, v, a(dt, A_log))
      y          = o * SiLU(g (+ b_g))
      out        = y W_o^T

    x: [B, L, D]; W_q..W_g: [E, D] (E = H * d_head); W_dt: [H, D];
    conv_w: [3, E, K] (q, k, v); conv_b: [3, E] or None; W_hq, W_hk: [p, d_head];
    A_log: [H]; W_o: [D, E].  ``batches`` restricts the evaluation to a subset
    of the batch (each batch row is independent)."""
    x = _f64(x)
    if batches is not None:
        x = x[list(batches)]
    B, L, D = x.shape
    H = int(n_heads)
    E = W_q.shape[0]
    dh = E // H
    xf = x.reshape(B * L, D)
    q = xf @ _f64(W_q).T
    k = xf @ _f64(W_k).T
    v = xf @ _f64(W_v).T
    g = xf @ _f64(W_g).T
    dt = xf @ _f64(W_dt).T
    if b_dt is not None:
        dt = dt + _f64(b_dt)
    if b_g is not None:
        g = g + _f64(b_g)
    cw = _f64(conv_w)
    cb = [None, None, None] if conv_b is None else [_f64(conv_b)[i] for i in range(3)]
    q = causal_conv(q.reshape(B, L, E), cw[0], cb[0])
    k = causal_conv(k.reshape(B, L, E), cw[1], cb[1])
    v = causal_conv(v.reshape(B, L, E), cw[2], cb[2])
    o = scan_fwd(q.reshape(B, L, H, dh), k.reshape(B, L, H, dh), v.reshape(B, L, H, dh),
                 W_q=W_hq, W_k=W_hk, dt=dt.reshape(B, L, H), A_log=A_log)
    y = o.reshape(B * L, E) * silu(g)
    out = y @ _f64(W_o).T
    return out.reshape(B, L, D)


# --------------------------------------------------------------------------
# the block around the mixer ([HM] sec. 5.1)
# --------------------------------------------------------------------------

def layer_norm(x, w=None, b=None, eps=1e-5):
    """Layer normalisation over the last axis, as the GPT-NeoX / Pythia block
    applies it to its input before the mixer and before the MLP ([HM] sec. 5.1):
    (x - mean) / sqrt(var + eps) * w + b, with var the population variance
    (mean of squared deviations).  w, b: [D] or None (1 and 0)."""
    x = _f64(x)
    mean = x.mean(axis=-1, keepdims=True)
    dev = x - mean
    var = (dev * dev).mean(axis=-1, keepdims=True)
    y = dev / np.sqrt(var + eps)
    if w is not None:
        y = y * _f64(w)
    if b is not None:
        y = y + _f64(b)
    return y


def _erf(x):
    from scipy.special import erf
    return erf(x)


def gelu(x):
    """GELU in its exact form, x * Phi(x) with Phi the standard normal CDF
    written through erf: 0.5 x (1 + erf(x / sqrt 2)) (the activation of the
    GPT-NeoX / Pythia MLP)."""
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / np.sqrt(2.0)))


def mlp(h, W_fc1, b_fc1, W_fc2, b_fc2):
    """The block's MLP: GELU(h W1^T + b1) W2^T + b2.  h: [..., D];
    W_fc1: [F, D]; b_fc1: [F] or None; W_fc2: [D, F]; b_fc2: [D] or None."""
    h = _f64(h)
    u = h @ _f64(W_fc1).T
    if b_fc1 is not None:
        u = u + _f64(b_fc1)
    y = gelu(u) @ _f64(W_fc2).T
    if b_fc2 is not None:
        y = y + _f64(b_fc2)
    return y


def block_fwd(x, ln1_w, ln1_b, ln2_w, ln2_b, W_fc1, b_fc1, W_fc2, b_fc2, mixer, eps=1e-5,
              n_heads=8, batches=None):
    """Parallel (GPT-NeoX / Pythia) block with the attention replaced by the
    HedgeMamba mixer ([HM] sec. 5.1, Lst. 1): both branches read the same
    input through their own normalisation and add into the residual,

      out = x + mixer(LN1(x)) + MLP(LN2(x)).

    x: [B, L, D]; ln*_w, ln*_b: [D]; MLP weights as in ``mlp``; ``mixer``: the
    keyword arguments of ``mixer_fwd`` other than x, n_heads and batches."""
    x = _f64(x)
    if batches is not None:
        x = x[list(batches)]
    h1 = layer_norm(x, ln1_w, ln1_b, eps)
    h2 = layer_norm(x, ln2_w, ln2_b, eps)
    return x + mixer_fwd(h1, n_heads=n_heads, **mixer) + mlp(h2, W_fc1, b_fc1, W_fc2, b_fc2)


def omp_threads_in_use() -> int:
    """Threads the OpenMP loops will use (OMP_NUM_THREADS or all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        try:
            return max(1, int(env))
        except ValueError:
            pass
    return os.cpu_count() or 1


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
