"""Thin Python binding of libhm.so, the HedgeMamba mixer-scan library for B200.

Argument marshalling only: every function here fills the C structs declared
in ``include/hm.h`` from torch tensors (device memory and streams come from
PyTorch) and calls the C entry point of the same name.  All arithmetic runs
in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
importing this package fails loudly if the built library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhm.so")

HM_OK, HM_ERR_INVALID_ARG, HM_ERR_UNSUPPORTED, HM_ERR_CUDA, HM_ERR_TIMEOUT, HM_ERR_DEVICE = range(6)
HM_F32, HM_BF16 = 0, 1
HM_FLAG_DT_SCALED_INPUT, HM_FLAG_PER_FEATURE_DECAY, HM_FLAG_ROPE = 1, 2, 4

if not os.path.exists(LIB_PATH):
    raise ImportError("libhm.so is not built (%s); run __graft_entry__.build() or "
                      "python selective_ssm_sequence_b200/_build.py" % LIB_PATH)

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class ScanArgs(ctypes.Structure):
    """Mirror of hm_scan_args."""
    _fields_ = [("B", _I64), ("L", _I64), ("H", _I), ("d", _I), ("p", _I), ("dv", _I),
                ("io_dtype", _I), ("q", _P), ("k", _P), ("v", _P), ("W_q", _P), ("W_k", _P),
                ("w_head_stride", _I64), ("b_q", _P), ("b_k", _P), ("dt", _P), ("A_log", _P),
                ("S0", _P), ("z0", _P), ("o", _P), ("S_out", _P), ("z_out", _P),
                ("workspace", _P), ("workspace_bytes", _SZ), ("flags", ctypes.c_uint),
                ("log_decay_out", _P), ("rope_base", ctypes.c_double), ("pos0", _I64)]


class ScanBwdArgs(ctypes.Structure):
    """Mirror of hm_scan_bwd_args."""
    _fields_ = [("B", _I64), ("L", _I64), ("H", _I), ("d", _I), ("p", _I), ("dv", _I), ("io_dtype", _I),
                ("q", _P), ("k", _P), ("v", _P), ("W_q", _P), ("W_k", _P), ("dt", _P), ("A_log", _P),
                ("S0", _P), ("z0", _P), ("dout", _P), ("grad_q", _P), ("grad_k", _P), ("grad_v", _P),
                ("grad_W_q", _P), ("grad_W_k", _P), ("grad_dt", _P), ("grad_A_log", _P), ("grad_S0", _P),
                ("grad_z0", _P), ("workspace", _P), ("workspace_bytes", _SZ)]


class CombineArgs(ctypes.Structure):
    """Mirror of hm_combine_args."""
    _fields_ = [("n_parts", _I64), ("BH", _I64), ("F", _I), ("dv", _I), ("per_feature", _I),
                ("parts", _P), ("part_len", _I64), ("S0", _P), ("z0", _P), ("only_part", _I64),
                ("S_start", _P), ("z_start", _P), ("S_end", _P), ("z_end", _P)]


class DecodeArgs(ctypes.Structure):
    """Mirror of hm_decode_args."""
    _fields_ = [("B", _I64), ("H", _I), ("d", _I), ("p", _I), ("dv", _I), ("io_dtype", _I),
                ("q", _P), ("k", _P), ("v", _P), ("W_q", _P), ("W_k", _P),
                ("w_head_stride", _I64), ("b_q", _P), ("b_k", _P), ("dt", _P), ("A_log", _P),
                ("S", _P), ("z", _P), ("o", _P), ("workspace", _P), ("workspace_bytes", _SZ),
                ("flags", ctypes.c_uint), ("rope_base", ctypes.c_double), ("positions", _P)]


class MixerArgs(ctypes.Structure):
    """Mirror of hm_mixer_args."""
    _fields_ = [("B", _I64), ("L", _I64), ("d_model", _I), ("H", _I), ("E", _I), ("p", _I),
                ("conv_k", _I), ("x", _P), ("W_q", _P), ("W_k", _P), ("W_v", _P), ("W_g", _P),
                ("W_dt", _P), ("b_dt", _P), ("b_g", _P), ("conv_w", _P), ("conv_b", _P),
                ("W_hq", _P), ("W_hk", _P), ("A_log", _P), ("W_o", _P), ("out", _P)]


class BlockArgs(ctypes.Structure):
    """Mirror of hm_block_args."""
    _fields_ = [("mixer", MixerArgs), ("ln1_w", _P), ("ln1_b", _P), ("ln2_w", _P), ("ln2_b", _P),
                ("eps", ctypes.c_float), ("d_ff", _I), ("W_fc1", _P), ("b_fc1", _P), ("W_fc2", _P),
                ("b_fc2", _P)]


lib.hm_status_string.restype = ctypes.c_char_p
lib.hm_status_string.argtypes = [_I]
lib.hm_last_error_detail.restype = ctypes.c_char_p
lib.hm_last_error_detail.argtypes = []
lib.hm_version.restype = ctypes.c_char_p
lib.hm_featmap.restype = _I
lib.hm_featmap.argtypes = [_P, _I, _I64, _I, _I, _I, _P, _I64, _P, _P, _I, _P]
lib.hm_scan_workspace_size.restype = _SZ
lib.hm_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
lib.hm_scan_chunked_fwd.restype = _I
lib.hm_scan_chunked_fwd.argtypes = [ctypes.POINTER(ScanArgs), _P]
lib.hm_decode_workspace_size.restype = _SZ
lib.hm_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
lib.hm_step_decode.restype = _I
lib.hm_step_decode.argtypes = [ctypes.POINTER(DecodeArgs), _P]
lib.hm_step_decode_noalloc.restype = _I
lib.hm_step_decode_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), _P]
lib.hm_mixer_workspace_size.restype = _SZ
lib.hm_mixer_workspace_size.argtypes = [ctypes.POINTER(MixerArgs)]
lib.hm_mixer_fwd.restype = _I
lib.hm_mixer_fwd.argtypes = [ctypes.POINTER(MixerArgs), _P, _SZ, _P]
lib.hm_block_workspace_size.restype = _SZ
lib.hm_block_workspace_size.argtypes = [ctypes.POINTER(BlockArgs)]
lib.hm_block_fwd.restype = _I
lib.hm_block_fwd.argtypes = [ctypes.POINTER(BlockArgs), _P, _SZ, _P]
lib.hm_scan_bwd_workspace_size.restype = _SZ
lib.hm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanBwdArgs)]
lib.hm_scan_bwd.restype = _I
lib.hm_scan_bwd.argtypes = [ctypes.POINTER(ScanBwdArgs), _P]
lib.hm_scan_combine.restype = _I
lib.hm_scan_combine.argtypes = [ctypes.POINTER(CombineArgs), _P]
lib.hm_launch_count.restype = ctypes.c_uint64
lib.hm_launch_count.argtypes = []
lib.hm_get_device_error.restype = _I
lib.hm_get_device_error.argtypes = [_P]
lib.hm_selftest_wait_timeout.restype = _I
lib.hm_selftest_wait_timeout.argtypes = [ctypes.c_uint32, _P]

EXPORTED = ("hm_status_string", "hm_last_error_detail", "hm_version", "hm_featmap",
            "hm_scan_workspace_size", "hm_scan_chunked_fwd", "hm_decode_workspace_size",
            "hm_step_decode", "hm_mixer_workspace_size", "hm_mixer_fwd", "hm_get_device_error",
            "hm_launch_count", "hm_step_decode_noalloc", "hm_selftest_wait_timeout", "hm_scan_combine",
            "hm_scan_bwd_workspace_size", "hm_scan_bwd", "hm_block_workspace_size", "hm_block_fwd")


class HMError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = lib.hm_last_error_detail().decode()
        msg = "%s: %s" % (where, lib.hm_status_string(status).decode())
        if detail:
            msg += " (%s)" % detail
        super().__init__(msg)


def _check(status: int, where: str) -> None:
    if status != HM_OK:
        raise HMError(status, where)


# ---------------------------------------------------------------- marshalling helpers

def _ptr(t) -> Optional[int]:
    """Device address of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return HM_F32
    if t.dtype == torch.bfloat16:
        return HM_BF16
    raise TypeError("unsupported dtype %s (float32 or bfloat16)" % t.dtype)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _require_cuda(*ts) -> None:
    for t in ts:
        if t is not None and not isinstance(t, int) and not t.is_cuda:
            raise ValueError("libhm works on device memory; got a CPU tensor")


# ---------------------------------------------------------------- entry points

def hm_version() -> str:
    return lib.hm_version().decode()


def hm_featmap(x, W, phi, H: int = 1, bias=None, w_head_stride: int = 0, stream=None) -> None:
    """phi = softmax([W x + b, -(W x + b)]) row-wise.  x: [..., d] (row r is
    head r mod H); W: [p, d] (or per-head, with w_head_stride); phi: [..., 2p]."""
    _require_cuda(x, W, phi, bias)
    d = x.shape[-1]
    p = W.shape[-2]
    rows = x.numel() // d
    st = lib.hm_featmap(_ptr(x), _dtype_code(x), rows, int(H), d, p, _ptr(W), int(w_head_stride),
                        _ptr(bias), _ptr(phi), _dtype_code(phi), _stream(stream))
    _check(st, "hm_featmap")


def scan_args(q, k, v, o, W_q=None, W_k=None, dt=None, A_log=None, S0=None, z0=None,
              S_out=None, z_out=None, b_q=None, b_k=None, w_head_stride: int = 0,
              workspace=None, flags: int = 0, log_decay_out=None, rope_base: float = 0.0,
              pos0: int = 0) -> ScanArgs:
    """Fill an hm_scan_args from tensors (q, k: [B, L, H, d]; v, o: [B, L, H, dv]).
    o = None (with S_out) makes a state-only call; q may then be None too."""
    B, L, H, d = k.shape
    dv = v.shape[-1]
    a = ScanArgs()
    a.B, a.L, a.H, a.d, a.dv = B, L, H, d, dv
    a.p = W_q.shape[-2] if W_q is not None else 0
    a.io_dtype = _dtype_code(k)
    a.q, a.k, a.v, a.o = _ptr(q), _ptr(k), _ptr(v), _ptr(o)
    a.W_q, a.W_k, a.w_head_stride = _ptr(W_q), _ptr(W_k), int(w_head_stride)
    a.b_q, a.b_k = _ptr(b_q), _ptr(b_k)
    a.dt, a.A_log = _ptr(dt), _ptr(A_log)
    a.S0, a.z0, a.S_out, a.z_out = _ptr(S0), _ptr(z0), _ptr(S_out), _ptr(z_out)
    a.flags = int(flags)
    a.log_decay_out = _ptr(log_decay_out)
    a.rope_base, a.pos0 = float(rope_base), int(pos0)
    if workspace is not None:
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    # the struct holds raw addresses: keep the tensors alive as long as it lives
    a._refs = (q, k, v, o, W_q, W_k, dt, A_log, S0, z0, S_out, z_out, b_q, b_k, workspace, log_decay_out)
    return a


def hm_scan_workspace_size(args: ScanArgs) -> int:
    return int(lib.hm_scan_workspace_size(ctypes.byref(args)))


def hm_scan_chunked_fwd(args: ScanArgs, stream=None) -> None:
    _check(lib.hm_scan_chunked_fwd(ctypes.byref(args), _stream(stream)), "hm_scan_chunked_fwd")


def scan_bwd_args(q, k, v, dout, grad_q, grad_k, grad_v, W_q=None, W_k=None, grad_W_q=None,
                  grad_W_k=None, dt=None, A_log=None, grad_dt=None, grad_A_log=None, S0=None, z0=None,
                  grad_S0=None, grad_z0=None, workspace=None) -> ScanBwdArgs:
    """Fill an hm_scan_bwd_args (forward inputs, dout [B, L, H, dv] and the fp32
    gradient buffers)."""
    B, L, H, d = q.shape
    a = ScanBwdArgs()
    a.B, a.L, a.H, a.d, a.dv = B, L, H, d, v.shape[-1]
    a.p = W_q.shape[-2] if W_q is not None else 0
    a.io_dtype = _dtype_code(q)
    a.q, a.k, a.v, a.dout = _ptr(q), _ptr(k), _ptr(v), _ptr(dout)
    a.W_q, a.W_k, a.dt, a.A_log, a.S0, a.z0 = map(_ptr, (W_q, W_k, dt, A_log, S0, z0))
    a.grad_q, a.grad_k, a.grad_v = _ptr(grad_q), _ptr(grad_k), _ptr(grad_v)
    a.grad_W_q, a.grad_W_k, a.grad_dt, a.grad_A_log = map(_ptr, (grad_W_q, grad_W_k, grad_dt, grad_A_log))
    a.grad_S0, a.grad_z0 = _ptr(grad_S0), _ptr(grad_z0)
    if workspace is not None:
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a._refs = (q, k, v, dout, grad_q, grad_k, grad_v, W_q, W_k, grad_W_q, grad_W_k, dt, A_log, grad_dt,
               grad_A_log, S0, z0, grad_S0, grad_z0, workspace)
    return a


def hm_scan_bwd_workspace_size(args: ScanBwdArgs) -> int:
    return int(lib.hm_scan_bwd_workspace_size(ctypes.byref(args)))


def hm_scan_bwd(args: ScanBwdArgs, stream=None) -> None:
    _check(lib.hm_scan_bwd(ctypes.byref(args), _stream(stream)), "hm_scan_bwd")


def combine_args(parts, n_parts: int, BH: int, F: int, dv: int, part_len: int, S_start, z_start,
                 per_feature: bool = False, S0=None, z0=None, only_part: int = -1, S_end=None,
                 z_end=None) -> CombineArgs:
    """Fill an hm_combine_args: `parts` holds n_parts records of part_len fp32
    values, each [log_decay (padded to 4) | S | z] of one sequence segment."""
    a = CombineArgs()
    a.n_parts, a.BH, a.F, a.dv, a.per_feature = int(n_parts), int(BH), int(F), int(dv), int(per_feature)
    a.parts, a.part_len = _ptr(parts), int(part_len)
    a.S0, a.z0, a.only_part = _ptr(S0), _ptr(z0), int(only_part)
    a.S_start, a.z_start, a.S_end, a.z_end = _ptr(S_start), _ptr(z_start), _ptr(S_end), _ptr(z_end)
    a._refs = (parts, S0, z0, S_start, z_start, S_end, z_end)
    return a


def hm_scan_combine(args: CombineArgs, stream=None) -> None:
    _check(lib.hm_scan_combine(ctypes.byref(args), _stream(stream)), "hm_scan_combine")


def combine_record_len(BH: int, F: int, dv: int, per_feature: bool = False) -> int:
    """fp32 values of one [log_decay | S | z] record (the log-decay part padded to 4)."""
    nl = BH * F if per_feature else BH
    return (nl + 3) // 4 * 4 + BH * F * dv + BH * F


def decode_args(q, k, v, o, S, z, W_q=None, W_k=None, dt=None, A_log=None, b_q=None, b_k=None,
                w_head_stride: int = 0, workspace=None, flags: int = 0, rope_base: float = 0.0,
                positions=None) -> DecodeArgs:
    """Fill an hm_decode_args (q, k: [B, H, d]; v, o: [B, H, dv]; S: [B, H, F, dv])."""
    B, H, d = q.shape
    a = DecodeArgs()
    a.B, a.H, a.d, a.dv = B, H, d, v.shape[-1]
    a.p = W_q.shape[-2] if W_q is not None else 0
    a.io_dtype = _dtype_code(q)
    a.q, a.k, a.v, a.o = _ptr(q), _ptr(k), _ptr(v), _ptr(o)
    a.W_q, a.W_k, a.w_head_stride = _ptr(W_q), _ptr(W_k), int(w_head_stride)
    a.b_q, a.b_k = _ptr(b_q), _ptr(b_k)
    a.dt, a.A_log = _ptr(dt), _ptr(A_log)
    a.S, a.z = _ptr(S), _ptr(z)
    a.flags = int(flags)
    a.rope_base, a.positions = float(rope_base), _ptr(positions)
    if workspace is not None:
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a._refs = (q, k, v, o, S, z, W_q, W_k, dt, A_log, b_q, b_k, workspace, positions)
    return a


def hm_decode_workspace_size(args: DecodeArgs) -> int:
    return int(lib.hm_decode_workspace_size(ctypes.byref(args)))


def hm_step_decode(args: DecodeArgs, stream=None) -> None:
    _check(lib.hm_step_decode(ctypes.byref(args), _stream(stream)), "hm_step_decode")


def hm_step_decode_noalloc(args: DecodeArgs, stream=None) -> None:
    """hm_step_decode without a caller-provided workspace: for callers that
    cannot allocate device memory.  The feature vectors use a fixed 4 MiB
    device array inside the library (B * H * F <= 524288 when W_q is given);
    calls that overlap on the GPU share that array and must be serialised."""
    _check(lib.hm_step_decode_noalloc(ctypes.byref(args), _stream(stream)), "hm_step_decode_noalloc")


def mixer_args(x, out, W_q, W_k, W_v, W_g, W_dt, conv_w, W_hq, W_hk, A_log, W_o, n_heads: int,
               conv_b=None, b_g=None, b_dt=None) -> MixerArgs:
    """Fill an hm_mixer_args (x, out: [B, L, D]; W_*: [E, D]; conv_w: [3, E, K])."""
    B, L, D = x.shape
    a = MixerArgs()
    a.B, a.L, a.d_model, a.H, a.E = B, L, D, int(n_heads), W_q.shape[0]
    a.p = W_hq.shape[0]
    a.conv_k = conv_w.shape[-1]
    a.x, a.out = _ptr(x), _ptr(out)
    a.W_q, a.W_k, a.W_v, a.W_g, a.W_dt, a.W_o = map(_ptr, (W_q, W_k, W_v, W_g, W_dt, W_o))
    a.b_dt, a.b_g = _ptr(b_dt), _ptr(b_g)
    a.conv_w, a.conv_b = _ptr(conv_w), _ptr(conv_b)
    a.W_hq, a.W_hk, a.A_log = _ptr(W_hq), _ptr(W_hk), _ptr(A_log)
    a._refs = (x, out, W_q, W_k, W_v, W_g, W_dt, conv_w, W_hq, W_hk, A_log, W_o, conv_b, b_g, b_dt)
    return a


def hm_mixer_workspace_size(args: MixerArgs) -> int:
    return int(lib.hm_mixer_workspace_size(ctypes.byref(args)))


def hm_mixer_fwd(args: MixerArgs, workspace, stream=None) -> None:
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.hm_mixer_fwd(ctypes.byref(args), _ptr(workspace), nbytes, _stream(stream)),
           "hm_mixer_fwd")


def block_args(x, out, mixer: dict, ln1_w, ln1_b, ln2_w, ln2_b, W_fc1, b_fc1, W_fc2, b_fc2, n_heads: int,
               eps: float = 1e-5) -> BlockArgs:
    """Fill an hm_block_args: ``mixer`` holds the mixer_args keywords other
    than x, out and n_heads; x, out: [B, L, D]; W_fc1: [d_ff, D]; W_fc2: [D, d_ff]."""
    a = BlockArgs()
    m = mixer_args(x, out, n_heads=n_heads, **mixer)
    a.mixer = m
    a.ln1_w, a.ln1_b, a.ln2_w, a.ln2_b = map(_ptr, (ln1_w, ln1_b, ln2_w, ln2_b))
    a.eps = float(eps)
    a.d_ff = W_fc1.shape[0]
    a.W_fc1, a.b_fc1, a.W_fc2, a.b_fc2 = map(_ptr, (W_fc1, b_fc1, W_fc2, b_fc2))
    a._refs = (m._refs, ln1_w, ln1_b, ln2_w, ln2_b, W_fc1, b_fc1, W_fc2, b_fc2)
    return a


def hm_block_workspace_size(args: BlockArgs) -> int:
    return int(lib.hm_block_workspace_size(ctypes.byref(args)))


def hm_block_fwd(args: BlockArgs, workspace, stream=None) -> None:
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.hm_block_fwd(ctypes.byref(args), _ptr(workspace), nbytes, _stream(stream)), "hm_block_fwd")


def hm_launch_count() -> int:
    """Kernels enqueued by libhm.so in this process so far."""
    return int(lib.hm_launch_count())


def hm_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word status."""
    return int(lib.hm_get_device_error(_stream(stream)))


def hm_selftest_wait_timeout(polls: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test (records HM_ERR_TIMEOUT on the device)."""
    _check(lib.hm_selftest_wait_timeout(int(polls), _stream(stream)), "hm_selftest_wait_timeout")


def alloc_workspace(nbytes: int, device=None):
    """A 256-byte-aligned device byte buffer of at least nbytes (torch allocation)."""
    import torch
    n = max(int(nbytes), 1) + 256
    buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    off = (-buf.data_ptr()) % 256
    return buf[off:off + max(int(nbytes), 1)]
