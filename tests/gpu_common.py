"""Helpers shared by the GPU parity tests: device tensors from the seeded
generator, calls through the C ABI, and the error metric."""
import numpy as np

import workloads as wl

# Tolerances of the headline benchmark's parity bar: max relative error
# 1e-4 for the fp32 configuration, 2e-2 for bf16 inputs with fp32 accumulation.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_err(x, r):
    """max_i |x_i - r_i| / max(|r_i|, rms(r)).

    o is a convex combination of v, so entries near zero are common and a
    bare ratio would be ill-posed; the rms floor keeps the metric relative to
    the output's scale."""
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    scale = max(float(np.sqrt(np.mean(r * r))), 1e-30)
    return float(np.max(np.abs(x - r) / np.maximum(np.abs(r), scale)))


def rel_err_rows(x, r):
    """max_i |x_i - r_i| / max(|r_i|, rms of r's row) over rows of the last axis.

    For outputs whose scale varies by orders of magnitude from token to token
    (with a = 1 the mixer's output at token t is a t-token average, ~1/sqrt(t)
    of the first token's), the floor is the token's own output scale instead
    of the whole tensor's."""
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    scale = np.maximum(np.sqrt(np.mean(r * r, axis=-1, keepdims=True)), 1e-30)
    return float(np.max(np.abs(x - r) / np.maximum(np.abs(r), scale)))


def rel_err_norm(x, r):
    """Normwise relative error ||x - r||_2 / ||r||_2."""
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return float(np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-300))


def dev_tensor(a, dtype, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_scan(hm, inp, io, with_W=True, S0=None, z0=None, want_state=False, decay=True,
             w_head_stride=0, b_q=None, b_k=None):
    """Prefill through hm_scan_chunked_fwd; returns (o, S, z) as float64."""
    import torch
    q = dev_tensor(inp["q"], io)
    k = dev_tensor(inp["k"], io)
    v = dev_tensor(inp["v"], io)
    Wq = dev_tensor(inp["W_q"], io) if with_W else None
    Wk = dev_tensor(inp["W_k"], io) if with_W else None
    dt = dev_tensor(inp["dt"], "f32") if (decay and "dt" in inp) else None
    A_log = dev_tensor(inp["A_log"], "f32") if (decay and "A_log" in inp) else None
    o = torch.empty_like(v)
    B, L, H, d = inp["q"].shape
    F = 2 * inp["W_q"].shape[-2] if with_W else d
    dv = inp["v"].shape[-1]
    S = z = None
    if want_state:
        S = torch.full((B, H, F, dv), float("nan"), device="cuda")
        z = torch.full((B, H, F), float("nan"), device="cuda")
    tS0 = dev_tensor(S0, "f32") if S0 is not None else None
    tz0 = dev_tensor(z0, "f32") if z0 is not None else None
    tbq = dev_tensor(b_q, "f32") if b_q is not None else None
    tbk = dev_tensor(b_k, "f32") if b_k is not None else None
    args = hm.scan_args(q, k, v, o, W_q=Wq, W_k=Wk, dt=dt, A_log=A_log, S0=tS0, z0=tz0,
                        S_out=S, z_out=z, b_q=tbq, b_k=tbk, w_head_stride=w_head_stride)
    ws = hm.alloc_workspace(hm.hm_scan_workspace_size(args))
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    hm.hm_scan_chunked_fwd(args)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    return to_np(o), (to_np(S) if S is not None else None), (to_np(z) if z is not None else None)
