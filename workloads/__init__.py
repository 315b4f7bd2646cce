"""Seeded synthetic inputs for the HedgeMamba mixer-scan workloads.

This module is shared by the CUDA-path tests/benchmark and by the oracle
runs, and it holds none of the method's arithmetic: only random numbers,
shapes and the rounding of generated values to the storage dtype.

Generator (stated so that anyone can regenerate the same bytes):
  * every tensor has its own 64-bit stream key = FNV-1a-64(name) XOR
    (seed * 0x9E3779B97F4A7C15 mod 2^64);
  * splitmix64 over the counter 1, 2, 3, ... under that key gives uint64s;
  * a uniform in (0, 1) is ((x >> 11) + 0.5) * 2^-53;
  * normals come from Box-Muller on consecutive uniform pairs (u1, u2):
    sqrt(-2 ln u1) cos(2 pi u2) and sqrt(-2 ln u1) sin(2 pi u2), in fp64;
  * values meant for bf16 storage are rounded fp64 -> fp32 (round to nearest
    even) -> bf16 (round to nearest even), once, here.  Both the GPU run and
    the oracle consume the rounded values.

The five workloads follow the headline benchmark's configuration list; the
shapes, dtypes and value distributions are listed in ``CONFIGS``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

_GOLD = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for ch in name.encode():
        h ^= ch
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _key(seed: int, name: str) -> np.uint64:
    return np.uint64(_fnv1a64(name) ^ ((int(seed) * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF))


def splitmix64_at(key: np.uint64, ctr: np.ndarray) -> np.ndarray:
    """splitmix64 outputs for the given counters (uint64 array) under ``key``
    (computed in place: one output array, one temporary)."""
    with np.errstate(over="ignore"):
        z = np.multiply(ctr, _GOLD, dtype=np.uint64)
        z += key
        t = np.right_shift(z, np.uint64(30))
        z ^= t
        z *= _M1
        np.right_shift(z, np.uint64(27), out=t)
        z ^= t
        z *= _M2
        np.right_shift(z, np.uint64(31), out=t)
        z ^= t
    return z


def splitmix64(key: np.uint64, n: int) -> np.ndarray:
    """n consecutive splitmix64 outputs for counter 1..n under ``key``."""
    return splitmix64_at(key, np.arange(1, n + 1, dtype=np.uint64))


def _u01(bits: np.ndarray) -> np.ndarray:
    u = np.right_shift(bits, np.uint64(11)).astype(np.float64)
    u += 0.5
    u *= 2.0 ** -53
    return u


def _flat_index(shape, index):
    """Flat (C-order) indices of the sub-block ``index`` (a tuple of slices or
    ints for the leading dimensions) of an array of ``shape``, built from
    per-dimension index vectors (the full range is never materialised)."""
    shape = tuple(int(x) for x in shape)
    if index is None:
        return np.arange(int(np.prod(shape)), dtype=np.int64).reshape(shape)
    index = tuple(index) + (slice(None),) * (len(shape) - len(index))
    strides = [int(np.prod(shape[i + 1:])) for i in range(len(shape))]
    out = np.zeros((), dtype=np.int64)
    for n, ix, st in zip(shape, index, strides):
        if isinstance(ix, slice):
            r = np.arange(n, dtype=np.int64)[ix]
            out = out[..., None] + r * st
        else:
            j = int(ix)
            out = out + (j + n if j < 0 else j) * st
    return out


def uniform(seed: int, name: str, shape, lo: float = 0.0, hi: float = 1.0, index=None) -> np.ndarray:
    """Uniform(lo, hi) array of ``shape`` (or its sub-block ``index``): element n
    uses counter n + 1."""
    idx = _flat_index(shape, index)
    u = _u01(splitmix64_at(_key(seed, name), (idx + 1).astype(np.uint64)))
    return lo + (hi - lo) * u


def _contiguous_block(shape, index):
    """(start, count, block shape) when the sub-block ``index`` (leading ints,
    then at most one unit-step slice as its last entry) is one contiguous run
    of the flat C-order array; None otherwise."""
    shape = tuple(int(x) for x in shape)
    if index is None:
        return 0, int(np.prod(shape)), shape
    index = tuple(index)
    start = 0
    for i, ix in enumerate(index):
        st = int(np.prod(shape[i + 1:]))
        if isinstance(ix, slice):
            a, b, step = ix.indices(shape[i])
            if step != 1 or i != len(index) - 1:
                return None
            n = max(0, b - a)
            return start + a * st, n * st, (n,) + shape[i + 1:]
        j = int(ix)
        if j < 0:
            j += shape[i]
        start += j * st
    return start, int(np.prod(shape[len(index):])), shape[len(index):]


def normal(seed: int, name: str, shape, std: float = 1.0, index=None) -> np.ndarray:
    """N(0, std^2) array of ``shape`` (or its sub-block ``index``).  Element n
    is the cosine (n even) or sine (n odd) branch of Box-Muller on the uniform
    pair with counters 2*(n//2) + 1 and 2*(n//2) + 2."""
    blk = _contiguous_block(shape, index)
    if blk is not None and blk[1] > (1 << 16):
        start, count, bshape = blk
        return _normal_range(seed, name, start, count, std).reshape(bshape)
    idx = _flat_index(shape, index)
    m = (idx // 2).astype(np.uint64)
    key = _key(seed, name)
    u1 = _u01(splitmix64_at(key, 2 * m + np.uint64(1)))
    u2 = _u01(splitmix64_at(key, 2 * m + np.uint64(2)))
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    return std * np.where((idx & 1) == 0, r * np.cos(ang), r * np.sin(ang))


def _normal_range(seed, name, start, count, std):
    """Elements start .. start + count - 1 of the flat normal stream, in chunks,
    each Box-Muller pair computed once."""
    out = np.empty(count, dtype=np.float64)
    key = _key(seed, name)
    step = 1 << 22
    for s0 in range(start, start + count, step):
        s1 = min(start + count, s0 + step)
        m0, m1 = s0 // 2, (s1 + 1) // 2
        mm = np.arange(m0, m1, dtype=np.uint64)
        u1 = _u01(splitmix64_at(key, 2 * mm + np.uint64(1)))
        u2 = _u01(splitmix64_at(key, 2 * mm + np.uint64(2)))
        r = np.sqrt(-2.0 * np.log(u1))
        ang = 2.0 * math.pi * u2
        z = np.empty(2 * (m1 - m0), dtype=np.float64)
        z[0::2] = r * np.cos(ang)
        z[1::2] = r * np.sin(ang)
        out[s0 - start:s1 - start] = z[s0 - 2 * m0:s1 - 2 * m0]
    return std * out


# --------------------------------------------------------------------------
# storage rounding (fp64 -> fp32 -> bf16, both round-to-nearest-even)
# --------------------------------------------------------------------------

def to_bf16_bits(a) -> np.ndarray:
    """uint16 bf16 bit patterns of ``a`` (fp64 -> fp32 RNE -> bf16 RNE)."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    r = ((u + rounding) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(a) -> np.ndarray:
    """Values of ``a`` after rounding to bf16, returned as float64."""
    return bf16_bits_to_f32(to_bf16_bits(a)).astype(np.float64)


def round_f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def store(a, dtype: str) -> np.ndarray:
    """Round generated fp64 values to the storage dtype ('bf16' or 'f32');
    returns float64 holding exactly the stored values."""
    if dtype == "bf16":
        return round_bf16(a)
    if dtype == "f32":
        return round_f32(a)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class ScanConfig:
    name: str
    B: int
    L: int
    H: int
    d: int
    p: int
    dv: int
    io: str            # 'f32' or 'bf16' storage of q, k, v, W, o
    decay: bool        # dt/A_log present (False: a_t = 1)
    seed: int
    w_std: float       # std of the Hedgehog projection entries

    @property
    def F(self) -> int:
        return 2 * self.p

    @property
    def tokens(self) -> int:
        return self.B * self.L

    @property
    def token_heads(self) -> int:
        return self.B * self.L * self.H


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    d: int
    p: int
    dv: int
    prefill: int
    steps: int
    seed: int
    w_std: float

    @property
    def F(self) -> int:
        return 2 * self.p


@dataclasses.dataclass(frozen=True)
class MixerConfig:
    name: str
    B: int
    L: int
    d_model: int
    H: int
    p: int
    conv: int
    seed: int

    @property
    def d_head(self) -> int:
        return self.d_model // self.H


# "N(0, s)" in the configuration list is read as variance s.
TINY_F32 = ScanConfig("tiny_f32_B1_H2_L256_d32_F64", 1, 256, 2, 32, 32, 32, "f32", False, 0,
                      math.sqrt(1.0 / 32))
PREFILL_PYTHIA = ScanConfig("prefill_B4_H8_L2048_d256_F256_bf16", 4, 2048, 8, 256, 128, 256,
                            "bf16", True, 1, math.sqrt(1.0 / 256))
PREFILL_LONG = ScanConfig("prefill_B1_H8_L32768_d256_F256_bf16", 1, 32768, 8, 256, 128, 256,
                          "bf16", True, 2, math.sqrt(1.0 / 256))
DECODE = DecodeConfig("decode_256x8_F256_dv256_prefill1024_steps512", 256, 8, 256, 128, 256,
                      1024, 512, 3, math.sqrt(1.0 / 256))
MIXER = MixerConfig("mixer_B8_L4096_D2048_H8_p128", 8, 4096, 2048, 8, 128, 4, 4)

CONFIGS = {c.name: c for c in (TINY_F32, PREFILL_PYTHIA, PREFILL_LONG, DECODE, MIXER)}


def scan_inputs(cfg: ScanConfig, B: Optional[int] = None, L: Optional[int] = None,
                seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs of a prefill workload as float64 arrays holding the stored values.

    q, k ~ N(0,1) [B,L,H,d]; v ~ N(0,1) [B,L,H,dv]; W_q, W_k ~ N(0, w_std^2)
    [p, d] (independent); with decay: dt ~ N(0,1) [B,L,H] (fp32) and
    A_log ~ U(log 1, log 16) [H] (fp32).  B, L or seed may be overridden to
    make smaller cases of the same distribution."""
    B = cfg.B if B is None else B
    L = cfg.L if L is None else L
    s = cfg.seed if seed is None else seed
    io = cfg.io
    out = {
        "W_q": store(normal(s, "W_q", (cfg.p, cfg.d), cfg.w_std), io),
        "W_k": store(normal(s, "W_k", (cfg.p, cfg.d), cfg.w_std), io),
        "q": store(normal(s, "q", (B, L, cfg.H, cfg.d)), io),
        "k": store(normal(s, "k", (B, L, cfg.H, cfg.d)), io),
        "v": store(normal(s, "v", (B, L, cfg.H, cfg.dv)), io),
    }
    if cfg.decay:
        out["dt"] = store(normal(s, "dt", (B, L, cfg.H)), "f32")
        out["A_log"] = store(uniform(s, "A_log", (cfg.H,), 0.0, math.log(16.0)), "f32")
    return out


def decode_weights(cfg: DecodeConfig) -> Dict[str, np.ndarray]:
    """Hedgehog W_q, W_k (bf16, N(0, w_std^2)) and A_log ~ U(log 1, log 16)."""
    s = cfg.seed
    return {
        "W_q": store(normal(s, "W_q", (cfg.p, cfg.d), cfg.w_std), "bf16"),
        "W_k": store(normal(s, "W_k", (cfg.p, cfg.d), cfg.w_std), "bf16"),
        "A_log": store(uniform(s, "A_log", (cfg.H,), 0.0, math.log(16.0)), "f32"),
    }


def decode_prefill(cfg: DecodeConfig, index=None) -> Dict[str, np.ndarray]:
    """The seeded prefill tokens [B, prefill, H, *] (bf16 q/k/v ~ N(0,1), fp32
    dt ~ N(0,1)), or their sub-block ``index`` = (batch slice, token slice,
    head slice)."""
    s = cfg.seed
    B, P, H = cfg.B, cfg.prefill, cfg.H
    return {
        "q": store(normal(s, "pre_q", (B, P, H, cfg.d), index=index), "bf16"),
        "k": store(normal(s, "pre_k", (B, P, H, cfg.d), index=index), "bf16"),
        "v": store(normal(s, "pre_v", (B, P, H, cfg.dv), index=index), "bf16"),
        "dt": store(normal(s, "pre_dt", (B, P, H), index=index), "f32"),
    }


def decode_step_tokens(cfg: DecodeConfig, step: int) -> Dict[str, np.ndarray]:
    """Token of decode step ``step`` for every (batch, head): q, k [B, H, d],
    v [B, H, dv] (bf16, N(0,1)) and dt [B, H] (fp32, N(0,1))."""
    s = cfg.seed
    B, H = cfg.B, cfg.H
    tag = "step%d_" % step
    return {
        "q": store(normal(s, tag + "q", (B, H, cfg.d)), "bf16"),
        "k": store(normal(s, tag + "k", (B, H, cfg.d)), "bf16"),
        "v": store(normal(s, tag + "v", (B, H, cfg.dv)), "bf16"),
        "dt": store(normal(s, tag + "dt", (B, H)), "f32"),
    }


def mixer_weights(cfg: MixerConfig) -> Dict[str, np.ndarray]:
    """Mixer weights: projections N(0, 1/d_model) bf16 ([E, D], [H, D], [D, E]);
    conv w N(0, 1/K) fp32 [3, E, K]; Hedgehog W N(0, 1/d_head) bf16 [p, d_head];
    A_log ~ U(log 1, log 16) fp32 [H]."""
    s = cfg.seed
    D = cfg.d_model
    E = cfg.H * cfg.d_head
    wstd = math.sqrt(1.0 / D)
    return {
        "W_q": store(normal(s, "W_q", (E, D), wstd), "bf16"),
        "W_k": store(normal(s, "W_k", (E, D), wstd), "bf16"),
        "W_v": store(normal(s, "W_v", (E, D), wstd), "bf16"),
        "W_g": store(normal(s, "W_g", (E, D), wstd), "bf16"),
        "W_dt": store(normal(s, "W_dt", (cfg.H, D), wstd), "bf16"),
        "W_o": store(normal(s, "W_o", (D, E), math.sqrt(1.0 / E)), "bf16"),
        "conv_w": store(normal(s, "conv_w", (3, E, cfg.conv), math.sqrt(1.0 / cfg.conv)), "f32"),
        "W_hq": store(normal(s, "W_hq", (cfg.p, cfg.d_head), math.sqrt(1.0 / cfg.d_head)), "bf16"),
        "W_hk": store(normal(s, "W_hk", (cfg.p, cfg.d_head), math.sqrt(1.0 / cfg.d_head)), "bf16"),
        "A_log": store(uniform(s, "A_log", (cfg.H,), 0.0, math.log(16.0)), "f32"),
    }


def block_weights(cfg: MixerConfig, d_ff: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Weights of the parallel block around the mixer: layer-norm scales
    1 + N(0, 0.1^2) and shifts N(0, 0.1^2) (fp32 [D]); MLP d_model -> d_ff (4 d_model
    by default) -> d_model with weights N(0, 1/fan_in) bf16 and biases
    N(0, 0.1^2) fp32."""
    s = cfg.seed
    D = cfg.d_model
    F = 4 * D if d_ff is None else d_ff
    return {
        "ln1_w": store(1.0 + normal(s, "ln1_w", (D,), 0.1), "f32"),
        "ln1_b": store(normal(s, "ln1_b", (D,), 0.1), "f32"),
        "ln2_w": store(1.0 + normal(s, "ln2_w", (D,), 0.1), "f32"),
        "ln2_b": store(normal(s, "ln2_b", (D,), 0.1), "f32"),
        "W_fc1": store(normal(s, "W_fc1", (F, D), math.sqrt(1.0 / D)), "bf16"),
        "b_fc1": store(normal(s, "b_fc1", (F,), 0.1), "f32"),
        "W_fc2": store(normal(s, "W_fc2", (D, F), math.sqrt(1.0 / F)), "bf16"),
        "b_fc2": store(normal(s, "b_fc2", (D,), 0.1), "f32"),
    }


def mixer_x(cfg: MixerConfig, B: Optional[int] = None, L: Optional[int] = None) -> np.ndarray:
    B = cfg.B if B is None else B
    L = cfg.L if L is None else L
    return store(normal(cfg.seed, "x", (B, L, cfg.d_model)), "bf16")
