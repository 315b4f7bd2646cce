#!/usr/bin/env python
"""Benchmark of the HedgeMamba mixer scan on B200 (prints one JSON line).

Default workload: the long-context prefill (B=1, H=8, L=32768, d = dv = 256,
Hedgehog 256->128 so F = 256, bf16 q/k/v, fp32 state and accumulation,
dt ~ N(0,1), A_log ~ U(0, log 16)), the largest single-GPU scan workload;
`--workload prefill` runs the Pythia-1B-shaped B=4, L=2048 case.  One step is
one pass of the whole hot path over one batch: the Hedgehog map on q and on k,
then the decayed normalised chunked scan, through one C-ABI call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|prefill|decode|mixer] [--batch B]

Multi-GPU (N > 1, launched by torchrun): every rank runs its own batch (its
own seed); there is no data-path collective ("weak" scaling).  Times are
device times (CUDA events) and the reported time is the max over ranks.

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events
on the launching stream, with a 512 MiB buffer write between steps (outside
the events) so that no step finds its inputs in the 126 MB L2.

--impl reference times the fp64 CPU oracle (the reference for this method)
on bounded samples of the same workload on the host cores; rank 0 only.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

# ---------------------------------------------------------------- peaks

_FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the B200's spec sheet: HBM3e bandwidth and dense bf16 tensor throughput
_SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(_FALLBACK_PEAKS), "fallback"


# DRAM bytes per launch of the dominant call from an ncu capture of the
# current kernel versions (dram__bytes_read.sum + dram__bytes_write.sum,
# summed over the call's kernels; ncu runs each kernel with cold caches), or
# None when a kernel changed since the counters were taken
# (profiles/scan_call_traffic.md).  Prefill B4 H8 L2048: scan_state
# 33,733,888 + 35,072, scan_carry 16,852,992, scan_out 109,465,600 +
# 7,543,040.  Long context B1 H8 L32768: scan_state 240,059,648 + 3,171,584,
# scan_carry 16,860,672, scan_out 420,714,240 + 109,503,232.
NCU_TRAFFIC_BYTES = {
    ("scan_chunked (features precomputed)", "prefill_B4_H8_L2048_d256_F256_bf16"): 167572736,
    ("scan_chunked (features precomputed)", "prefill_B1_H8_L32768_d256_F256_bf16"): 790018304,
}

# ---------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU, read in the
    background while the timed region runs.

    Reads only: NVML queries every 5 ms (pynvml), else `nvidia-smi -lms 50`.
    summary() keeps the samples taken between mark_start() and mark_stop(),
    the host-side bounds of the timed region."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.samples = []        # (host time, sm MHz, max sm MHz, set of reason names)
        self.t0 = self.t1 = None
        self.source = None
        self._stop = threading.Event()
        self.thread = None
        self.proc = None
        self.nv = self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = self._nvml_handle(device)
        except Exception:
            self.nv = self.handle = None

    def _nvml_handle(self, device):
        nv = self.nv
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(device)

    def start(self):
        if self.handle is not None:
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
        else:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "--query-gpu=" + self.SMI_FIELDS, "--format=csv,noheader,nounits",
                     "-lms", "50", "-i", str(self.device)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                return
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self):
        nv, hd = self.nv, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        masks = [(n, getattr(nv, attr, 0)) for n, attr in self.REASONS]
        try:
            mx = float(nv.nvmlDeviceGetMaxClockInfo(hd, nv.NVML_CLOCK_SM))
        except Exception:
            mx = None
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                sm = float(nv.nvmlDeviceGetClockInfo(hd, nv.NVML_CLOCK_SM))
                bits = int(get_reasons(hd))
                self.samples.append((t, sm, mx, {n for n, m in masks if m and bits & m}))
            except Exception:
                pass
            time.sleep(0.005)

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            rs = {n for n, val in zip(names, parts[5:9]) if val.lower().startswith("active")}
            self.samples.append((time.perf_counter(), sm, mx, rs))

    def sample_now(self):
        """One synchronous read (NVML only), so that a timed region shorter
        than the polling period still has samples."""
        if self.handle is None:
            return
        nv, hd = self.nv, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        try:
            mx = float(nv.nvmlDeviceGetMaxClockInfo(hd, nv.NVML_CLOCK_SM))
        except Exception:
            mx = None
        try:
            t = time.perf_counter()
            sm = float(nv.nvmlDeviceGetClockInfo(hd, nv.NVML_CLOCK_SM))
            bits = int(get_reasons(hd))
            self.samples.append((t, sm, mx, {n for n, attr in self.REASONS
                                             if getattr(nv, attr, 0) and bits & getattr(nv, attr, 0)}))
        except Exception:
            pass

    def mark_start(self):
        self.t0 = time.perf_counter()
        self.sample_now()

    def in_flight(self):
        """Call once the timed work is enqueued and before waiting for it:
        one more synchronous sample while the GPU runs it."""
        self.sample_now()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        lo = self.t0 if self.t0 is not None else -float("inf")
        hi = self.t1 if self.t1 is not None else float("inf")
        inside = [x for x in self.samples if lo <= x[0] <= hi]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0,
                    "source": self.source}
        reasons = set()
        for x in inside:
            reasons |= x[3]
        mxs = [x[2] for x in inside if x[2] is not None]
        return {"sm_mhz": statistics.median(x[1] for x in inside),
                "sm_max_mhz": max(mxs) if mxs else None,
                "reasons": sorted(reasons), "samples": len(inside), "source": self.source}


# ---------------------------------------------------------------- helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def to_dev(a, dtype, torch):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def max_over_ranks(x: float, world: int, torch, device: str = "cuda") -> float:
    """The slowest rank's time (all ranks take part; NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank generates its own batch (weak scaling, no data exchange)."""
    return base_seed + 1000 * rank


def whole_job_rate(units_per_rank: int, world: int, ms_max: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU oracle baseline

def oracle_prefill_rate(cfg, budget_s: float = 12.0):
    """fp64 oracle (feature maps + recurrence) on all B*H heads of the
    workload for its first T tokens, T grown until ~budget_s of CPU work.
    Returns (tokens_per_s, threads, sample description, seconds)."""
    import oracle
    oracle.build()
    T = 16
    while True:
        inp = wl.scan_inputs(cfg, L=T)
        t0 = time.perf_counter()
        oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"],
                        dt=inp.get("dt"), A_log=inp.get("A_log"))
        dt = time.perf_counter() - t0
        if dt >= budget_s or T >= cfg.L:
            break
        grow = max(2, min(8, int(budget_s / max(dt, 1e-3))))
        T = min(cfg.L, T * grow)
    threads = min(oracle.omp_threads_in_use(), cfg.B * cfg.H)
    sample = ("fp64 oracle (Hedgehog maps + recurrence) on all %d (batch, head) pairs, first %d of "
              "%d tokens" % (cfg.B * cfg.H, T, cfg.L))
    return cfg.B * T / dt, threads, sample, dt


# ---------------------------------------------------------------- prefill workload

def algorithmic_per_token_head(F: int, d: int, p: int, dv: int):
    """Algorithmic FLOPs and HBM bytes per (batch, token, head) of the prefill.

    FLOPs: two Hedgehog projections 2*(2*d*p) + the normalised recurrence
    4*F*(dv + 1) (state update and readout of the numerator, F*dv each as
    multiply-add, plus the denominator).  Bytes (bf16 io): q, k, v read, o
    written (2 bytes each element) and dt (4 bytes)."""
    flops_featmap = 2 * (2 * d * p)
    flops_scan = 4 * F * (dv + 1)
    bytes_fused = 2 * (2 * d + dv + dv) + 4
    return flops_featmap, flops_scan, bytes_fused


def bench_prefill(cfg, args, rank, world, torch):
    import selective_ssm_sequence_b200 as hm

    peaks, peak_kind = load_peaks()
    seed = rank_seed(cfg.seed, rank)
    inp = wl.scan_inputs(cfg, seed=seed)
    B, L, H, d, p, dv = cfg.B, cfg.L, cfg.H, cfg.d, cfg.p, cfg.dv
    F = 2 * p
    q, k, v = (to_dev(inp[n], "bf16", torch) for n in ("q", "k", "v"))
    Wq, Wk = to_dev(inp["W_q"], "bf16", torch), to_dev(inp["W_k"], "bf16", torch)
    dtt, A_log = to_dev(inp["dt"], "f32", torch), to_dev(inp["A_log"], "f32", torch)
    o = torch.empty_like(v)
    # the step: one call, feature maps computed inside (both in one launch)
    full = hm.scan_args(q, k, v, o, W_q=Wq, W_k=Wk, dt=dtt, A_log=A_log)
    ws_full = hm.alloc_workspace(hm.hm_scan_workspace_size(full))
    full.workspace, full.workspace_bytes = ws_full.data_ptr(), ws_full.numel()
    # breakdown only: the scan call on precomputed features
    phq = torch.empty(B, L, H, F, device="cuda", dtype=torch.bfloat16)
    phk = torch.empty_like(phq)
    hm.hm_featmap(q, Wq, phq, H=H)
    hm.hm_featmap(k, Wk, phk, H=H)
    fargs = hm.scan_args(phq, phk, v, o, dt=dtt, A_log=A_log)
    ws = hm.alloc_workspace(hm.hm_scan_workspace_size(fargs))
    fargs.workspace, fargs.workspace_bytes = ws.data_ptr(), ws.numel()
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    calls = [lambda: hm.hm_scan_chunked_fwd(full), lambda: hm.hm_scan_chunked_fwd(fargs)]
    # Each C-ABI call is captured once into its own CUDA graph and replayed:
    # the timed region then holds device work only (no Python / ctypes / host
    # enqueue latency).
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for c in calls:
            c()
    torch.cuda.synchronize()
    graphs, launches_per_call = [], []
    for c in calls:
        n0 = hm.hm_launch_count()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            c()
        graphs.append(g)
        launches_per_call.append(hm.hm_launch_count() - n0)
    launches_per_step = launches_per_call[0]
    torch.cuda.synchronize()

    def timed(graph, evs):
        for e in evs:
            flush.zero_()
            e[0].record(stream)
            graph.replay()
            e[1].record(stream)

    K, W = args.steps, args.warmup
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    evs_scan = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    warm = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(W)]
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    timed(graphs[0], warm)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark_start()
    timed(graphs[0], evs)
    sampler.in_flight()
    torch.cuda.synchronize()
    sampler.mark_stop()
    launches = launches_per_step * K
    barrier(world)
    torch.cuda.synchronize()
    sampler.stop()
    assert hm.hm_get_device_error() == hm.HM_OK
    # breakdown (outside the timed step): the scan call alone
    timed(graphs[1], warm)
    timed(graphs[1], evs_scan)
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK

    t_step = [e[0].elapsed_time(e[1]) for e in evs]
    t_sc = [e[0].elapsed_time(e[1]) for e in evs_scan]
    ms_step = max_over_ranks(sum(t_step) / K, world, torch)
    ms_scan = max_over_ranks(sum(t_sc) / K, world, torch)
    ms_fmap = max(ms_step - ms_scan, 0.0) / 2   # per feature map (both run in one launch)

    th = B * L * H
    fl_fm, fl_sc, _ = algorithmic_per_token_head(F, d, p, dv)
    value = whole_job_rate(B * L, world, ms_step)

    # dominant call and its roofline
    bw = peaks["hbm_gbs"]
    tf = peaks["bf16_tflops"]
    fm_bytes = th * (2 * d + 2 * F)      # x read, phi written (bf16), per launch
    fm_flops = th * 2 * d * p
    sc_bytes = th * (2 * F + 2 * F + 2 * dv + 4 + 2 * dv)  # phiq, phik, v, dt read; o written
    sc_flops = th * fl_sc
    if ms_scan >= ms_fmap:
        name, nbytes, nflops, ms = "scan_chunked (features precomputed)", sc_bytes, sc_flops, ms_scan
    else:
        name, nbytes, nflops, ms = "hedgehog_featmap", fm_bytes, fm_flops, ms_fmap
    intensity = nflops / nbytes
    ridge = tf * 1e12 / (bw * 1e9)
    if intensity >= ridge:
        roof = {"bound": "tensor", "achieved": nflops / (ms * 1e-3) / 1e12, "peak": tf,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": bw, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_of_spec"] = roof["achieved"] / (_SPEC_PEAKS["hbm_gbs"] if roof["bound"] == "hbm"
                                               else _SPEC_PEAKS["bf16_tflops"])
    roof["traffic"] = NCU_TRAFFIC_BYTES.get((name, cfg.name))
    roof["kernel"] = name
    roof["peak_source"] = peak_kind
    roof["ms_per_launch"] = ms

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = bench_prefill_e2e(cfg, inp, Wq, Wk, A_log, args, world, torch, hm, flush)

    step_flops = th * (fl_fm + fl_sc)
    result = {
        "metric": "tokens/sec of HedgeMamba mixer scan fwd on 1 B200; % of tensor/HBM roofline",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 + Box-Muller, rounded to bf16)",
        "config": {"workload": cfg.name, "B": B, "L": L, "H": H, "d": d, "F": F, "dv": dv,
                   "tokens_per_gpu": B * L, "l2": "512 MiB buffer written between timed steps",
                   "step": "hm_scan_chunked_fwd(q, k, v, W_q, W_k, dt, A_log): both Hedgehog maps "
                           "(one launch) and the chunked scan",
                   "launch": "the call replayed from a CUDA graph captured once"},
        "roofline": roof,
        "step_roofline": {"bound": "tensor", "flops_per_token_head": fl_fm + fl_sc,
                          "achieved": step_flops / (ms_step * 1e-3) / 1e12, "peak": tf,
                          "unit": "TFLOP/s", "frac": step_flops / (ms_step * 1e-3) / 1e12 / tf,
                          "frac_of_spec": step_flops / (ms_step * 1e-3) / 1e12 / _SPEC_PEAKS["bf16_tflops"],
                          "peak_source": peak_kind},
        "breakdown_ms": {"featmap_q_and_k": 2 * ms_fmap, "scan": ms_scan,
                         "note": "scan = the call on precomputed features, timed separately; "
                                 "featmap = step - scan"},
        "gpu_launches": int(launches),
        "e2e": e2e,
        "clocks": sampler.summary(),
    }
    return result


def bench_prefill_e2e(cfg, inp, Wq, Wk, A_log, args, world, torch, hm, flush):
    """Same metric through the C ABI with the step's inputs copied from pinned
    host memory and the outputs copied back, all inside the timed region.

    The batch is cut into pieces (one sequence each; a single sequence is cut
    into 8 runs of tokens whose final state starts the next run), and the
    pieces are pipelined on three streams: the upload of piece i + 1 and the
    download of piece i - 1 overlap the scan of piece i (PCIe is full duplex).
    The timed region runs from an event before the first upload to an event
    after the last download, on the device timeline."""
    B, L, H, d, p, dv = cfg.B, cfg.L, cfg.H, cfg.d, cfg.p, cfg.dv
    F = 2 * p
    hq, hk, hv = (torch.from_numpy(inp[n].astype(np.float32)).to(torch.bfloat16).pin_memory()
                  for n in ("q", "k", "v"))
    hdt = torch.from_numpy(inp["dt"].astype(np.float32)).pin_memory()
    ho = torch.empty(B, L, H, dv, dtype=torch.bfloat16).pin_memory()
    q = torch.empty(hq.shape, dtype=torch.bfloat16, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty(hv.shape, dtype=torch.bfloat16, device="cuda")
    dtt = torch.empty(hdt.shape, dtype=torch.float32, device="cuda")
    o = torch.empty_like(v)
    if B > 1:
        pieces = [(b, b + 1, 0, L) for b in range(B)]
    else:
        n = 8 if L % (8 * 64) == 0 else 1
        pieces = [(0, 1, i * (L // n), (i + 1) * (L // n)) for i in range(n)]
    chained = B == 1 and len(pieces) > 1
    # state carried between the runs of one sequence (two buffers, alternating)
    Sbuf = [torch.empty(1, H, F, dv, device="cuda") for _ in range(2)] if chained else None
    zbuf = [torch.empty(1, H, F, device="cuda") for _ in range(2)] if chained else None
    args_list = []
    for i, (b0, b1, t0, t1) in enumerate(pieces):
        sl = (slice(b0, b1), slice(t0, t1))
        S0 = Sbuf[(i - 1) % 2] if chained and i > 0 else None
        z0 = zbuf[(i - 1) % 2] if chained and i > 0 else None
        So = Sbuf[i % 2] if chained and i + 1 < len(pieces) else None
        zo = zbuf[i % 2] if chained and i + 1 < len(pieces) else None
        a = hm.scan_args(q[sl], k[sl], v[sl], o[sl], W_q=Wq, W_k=Wk, dt=dtt[sl], A_log=A_log,
                         S0=S0, z0=z0, S_out=So, z_out=zo)
        args_list.append(a)
    ws = hm.alloc_workspace(max(hm.hm_scan_workspace_size(a) for a in args_list))
    for a in args_list:
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    main = torch.cuda.current_stream()
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdt))
    d2h = ho.numel() * ho.element_size()

    def step(e0, e1):
        e0.record(main)
        for st in (s_in, s_comp, s_out):
            st.wait_event(e0)
        done_in, done_comp = [], []
        for i, (b0, b1, t0, t1) in enumerate(pieces):
            sl = (slice(b0, b1), slice(t0, t1))
            with torch.cuda.stream(s_in):
                for dst, src in ((q, hq), (k, hk), (v, hv), (dtt, hdt)):
                    dst[sl].copy_(src[sl], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
                done_in.append(ev)
            s_comp.wait_event(done_in[i])
            hm.hm_scan_chunked_fwd(args_list[i], s_comp)
            ev = torch.cuda.Event()
            ev.record(s_comp)
            done_comp.append(ev)
            s_out.wait_event(ev)
            with torch.cuda.stream(s_out):
                ho[sl].copy_(o[sl], non_blocking=True)
        main.wait_stream(s_out)
        main.wait_stream(s_comp)
        e1.record(main)

    for _ in range(max(1, args.warmup)):
        flush.zero_()
        step(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    barrier(world)
    K = max(1, min(args.steps, 50))
    ts = []
    for _ in range(K):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step(e0, e1)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    assert hm.hm_get_device_error() == hm.HM_OK
    barrier(world)
    ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in ts) / K, world, torch)
    return {"value": B * L * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": K,
            "call": "hm_scan_chunked_fwd (feature maps + scan) per piece of %d, pinned-host copies "
                    "pipelined on three streams" % len(pieces)}


# ---------------------------------------------------------------- decode workload

def bench_decode(cfg, args, rank, world, torch):
    """512 consecutive hm_step_decode calls over 256 sequences x 8 heads with
    an fp32 state (256 x 256 per head); the state starts from the GPU's own
    1024-token prefill (hm_scan_chunked_fwd) of the seeded prompt.  The
    per-step tokens cycle through 16 seeded steps.  Each step is replayed from a
    CUDA graph (one featmap launch per q / k and one decode launch)."""
    import selective_ssm_sequence_b200 as hm
    peaks, peak_kind = load_peaks()
    if args.batch:
        cfg = dataclasses.replace(cfg, B=args.batch, name=cfg.name + "_batch%d" % args.batch)
    w = wl.decode_weights(cfg)
    B, H, F, dv = cfg.B, cfg.H, cfg.F, cfg.dv
    tWq, tWk = to_dev(w["W_q"], "bf16", torch), to_dev(w["W_k"], "bf16", torch)
    tA = to_dev(w["A_log"], "f32", torch)
    S = torch.empty(B, H, F, dv, device="cuda")
    z = torch.empty(B, H, F, device="cuda")
    # prefill in batch slices (keeps host-side generation small)
    for b0 in range(0, B, 32):
        pre = wl.decode_prefill(cfg, index=(slice(b0, b0 + 32),))
        q, k, v = (to_dev(pre[n], "bf16", torch) for n in ("q", "k", "v"))
        dtt = to_dev(pre["dt"], "f32", torch)
        o = torch.empty_like(v)
        a = hm.scan_args(q, k, v, o, W_q=tWq, W_k=tWk, dt=dtt, A_log=tA, S_out=S[b0:b0 + 32],
                         z_out=z[b0:b0 + 32])
        ws = hm.alloc_workspace(hm.hm_scan_workspace_size(a))
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
        hm.hm_scan_chunked_fwd(a)
    torch.cuda.synchronize()
    nstep_tokens = 16
    toks = [wl.decode_step_tokens(cfg, t) for t in range(nstep_tokens)]
    tq = [to_dev(t["q"], "bf16", torch) for t in toks]
    tk = [to_dev(t["k"], "bf16", torch) for t in toks]
    tv = [to_dev(t["v"], "bf16", torch) for t in toks]
    tdt = [to_dev(t["dt"], "f32", torch) for t in toks]
    o = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")
    dargs = [hm.decode_args(tq[i], tk[i], tv[i], o, S, z, W_q=tWq, W_k=tWk, dt=tdt[i], A_log=tA)
             for i in range(nstep_tokens)]
    ws = hm.alloc_workspace(hm.hm_decode_workspace_size(dargs[0]))
    for a in dargs:
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    graphs = []
    n0 = hm.hm_launch_count()
    for a in dargs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            hm.hm_step_decode(a)
        graphs.append(g)
    per_step = (hm.hm_launch_count() - n0) // nstep_tokens
    torch.cuda.synchronize()
    steps = args.steps if args.steps else cfg.steps
    for i in range(max(3, args.warmup)):
        graphs[i % nstep_tokens].replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    e0.record(stream)
    for i in range(steps):
        graphs[i % nstep_tokens].replay()
    e1.record(stream)
    sampler.in_flight()
    torch.cuda.synchronize()
    sampler.mark_stop()
    sampler.stop()
    assert hm.hm_get_device_error() == hm.HM_OK
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, torch)
    state_bytes = B * H * (2 * F * dv * 4 + 2 * F * 4)
    io_bytes = B * H * (2 * cfg.d * 2 + dv * 2 + 4 + dv * 2)
    gbs = (state_bytes + io_bytes) / (ms * 1e-3) / 1e9
    return {
        "metric": "decode tokens/sec (one token per sequence per step)",
        "value": B * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 io, fp32 state", "data": "synthetic",
        "config": {"workload": cfg.name, "B": B, "H": H, "F": F, "dv": dv,
                   "l2": "state 1.08 GB per step, larger than L2"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "frac_of_spec": gbs / _SPEC_PEAKS["hbm_gbs"],
                     "bytes_per_step": state_bytes + io_bytes, "peak_source": peak_kind,
                     "kernel": "whole step (the q and k feature maps in one launch + the decode launch)"},
        "gpu_launches": per_step * steps,
        "clocks": sampler.summary(),
    }


# ---------------------------------------------------------------- mixer workload

def bench_mixer(cfg, args, rank, world, torch, block=False):
    """Full mixer forward (B8 L4096 D2048 H8), one hm_mixer_fwd per step,
    replayed from a CUDA graph; with ``block`` the parallel GPT-NeoX block
    around it (layer norms, mixer, MLP d_model -> 4 d_model -> d_model,
    residual), one hm_block_fwd per step."""
    import selective_ssm_sequence_b200 as hm
    peaks, peak_kind = load_peaks()
    if args.batch:
        cfg = dataclasses.replace(cfg, B=args.batch, name=cfg.name + "_batch%d" % args.batch)
    w = wl.mixer_weights(cfg)
    t = {k: to_dev(v, "f32" if k in ("conv_w", "A_log") else "bf16", torch) for k, v in w.items()}
    x = to_dev(wl.mixer_x(cfg), "bf16", torch)
    out = torch.empty_like(x)
    d_ff = 4 * cfg.d_model
    if block:
        bw = {k: to_dev(v, "bf16" if k.startswith("W_") else "f32", torch)
              for k, v in wl.block_weights(cfg, d_ff).items()}
        a = hm.block_args(x, out, t, n_heads=cfg.H, **bw)
        ws = hm.alloc_workspace(hm.hm_block_workspace_size(a))
        call = lambda: hm.hm_block_fwd(a, ws)
    else:
        a = hm.mixer_args(x, out, t["W_q"], t["W_k"], t["W_v"], t["W_g"], t["W_dt"], t["conv_w"],
                          t["W_hq"], t["W_hk"], t["A_log"], t["W_o"], n_heads=cfg.H)
        ws = hm.alloc_workspace(hm.hm_mixer_workspace_size(a))
        call = lambda: hm.hm_mixer_fwd(a, ws)
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = hm.hm_launch_count()
    with torch.cuda.graph(g, stream=cap):
        call()
    per_step = hm.hm_launch_count() - n0
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    evs = []
    sampler.mark_start()
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        evs.append((e0, e1))
    sampler.in_flight()
    torch.cuda.synchronize()
    sampler.mark_stop()
    sampler.stop()
    assert hm.hm_get_device_error() == hm.HM_OK
    ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in evs) / args.steps, world, torch)
    D, E, L, B = cfg.d_model, cfg.d_model, cfg.L, cfg.B
    flops_tok = 2 * D * 4 * E + 2 * D * cfg.H + 2 * E * D + 2 * 2 * cfg.d_head * cfg.p * cfg.H \
        + 4 * 2 * cfg.p * (cfg.d_head + 1) * cfg.H + 3 * 2 * cfg.conv * E
    if block:
        flops_tok += 2 * 2 * D * d_ff   # the MLP's two GEMMs
    tf = flops_tok * B * L / (ms * 1e-3) / 1e12
    name = cfg.name.replace("mixer", "block") if block else cfg.name
    return {
        "metric": ("parallel block" if block else "mixer") + " forward tokens/sec",
        "value": B * L * world / (ms * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict({"workload": name, "B": B, "L": L, "d_model": D, "H": cfg.H},
                                            **({"d_ff": d_ff} if block else {})),
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16_tflops"], "frac_of_spec": tf / _SPEC_PEAKS["bf16_tflops"],
                     "flops_per_token": flops_tok, "peak_source": peak_kind,
                     "kernel": "whole block forward" if block else "whole mixer forward"},
        "gpu_launches": per_step * args.steps,
        "clocks": sampler.summary(),
    }


# ---------------------------------------------------------------- backward workload

def backward_flops_per_token_head(F: int, d: int, p: int, dv: int) -> int:
    """Algorithmic FLOPs of the scan's backward per (batch, token, head): the
    forward state recomputed (2 F dv), dphiq = S dn (2 F dv), the adjoint
    update (2 F dv), dphik = G v (2 F dv) and dv = G^T phik (2 F dv); the
    feature maps' dx = du W and dW += du x^T for q and k (4 x 2 p d)."""
    return 10 * F * dv + 8 * p * d


def bench_backward(cfg, args, rank, world, torch):
    """hm_scan_bwd on the Pythia-shaped prefill (B4 H8 L2048): gradients of
    sum(dout * o) for q, k, v, W_q, W_k, dt and A_log, one call per step,
    replayed from a CUDA graph."""
    import selective_ssm_sequence_b200 as hm
    peaks, peak_kind = load_peaks()
    inp = wl.scan_inputs(cfg, seed=rank_seed(cfg.seed, rank))
    B, L, H, d, p, dv = cfg.B, cfg.L, cfg.H, cfg.d, cfg.p, cfg.dv
    F = 2 * p
    q, k, v = (to_dev(inp[n], "bf16", torch) for n in ("q", "k", "v"))
    Wq, Wk = to_dev(inp["W_q"], "bf16", torch), to_dev(inp["W_k"], "bf16", torch)
    dtt, A_log = to_dev(inp["dt"], "f32", torch), to_dev(inp["A_log"], "f32", torch)
    dout = to_dev(wl.normal(cfg.seed, "dout", (B, L, H, dv)), "bf16", torch)
    f32 = lambda *shape: torch.empty(shape, device="cuda")
    a = hm.scan_bwd_args(q, k, v, dout, f32(B, L, H, d), f32(B, L, H, d), f32(B, L, H, dv), W_q=Wq, W_k=Wk,
                         grad_W_q=f32(p, d), grad_W_k=f32(p, d), dt=dtt, A_log=A_log, grad_dt=f32(B, L, H),
                         grad_A_log=f32(H))
    ws = hm.alloc_workspace(hm.hm_scan_bwd_workspace_size(a))
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        hm.hm_scan_bwd(a)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = hm.hm_launch_count()
    with torch.cuda.graph(g, stream=cap):
        hm.hm_scan_bwd(a)
    per_step = hm.hm_launch_count() - n0
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    evs = []
    sampler.mark_start()
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        evs.append((e0, e1))
    sampler.in_flight()
    torch.cuda.synchronize()
    sampler.mark_stop()
    sampler.stop()
    assert hm.hm_get_device_error() == hm.HM_OK
    ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in evs) / args.steps, world, torch)
    fl = backward_flops_per_token_head(F, d, p, dv) * B * L * H
    # CUDA-core fp32 peak from the unit counts: 148 SMs x 128 FMA lanes x 2 flops x the SM clock
    clk = sampler.summary().get("sm_max_mhz") or 1965.0
    alu_peak = 148 * 128 * 2 * clk * 1e6 / 1e12
    tfs = fl / (ms * 1e-3) / 1e12
    return {
        "metric": "backward tokens/sec (gradients of the prefill: q, k, v, W_q, W_k, dt, A_log)",
        "value": B * L * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp32 math", "data": "synthetic",
        "config": {"workload": "backward_" + cfg.name, "B": B, "L": L, "H": H, "F": F, "dv": dv,
                   "l2": "512 MiB buffer written between timed steps"},
        "roofline": {"bound": "alu", "achieved": tfs, "peak": alu_peak, "unit": "TFLOP/s", "frac": tfs / alu_peak,
                     "flops_per_token_head": backward_flops_per_token_head(F, d, p, dv),
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x max SM clock",
                     "kernel": "whole backward call"},
        "gpu_launches": per_step * args.steps,
        "clocks": sampler.summary(),
    }


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    cfg = {"prefill": wl.PREFILL_PYTHIA}.get(args.workload, wl.PREFILL_LONG)
    # each step: the oracle on every (batch, head) pair for a 64-token slice of
    # the sequence (a bounded sample of the workload)
    T = 64
    inp = wl.scan_inputs(cfg, L=T)
    for _ in range(args.warmup):
        oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                        A_log=inp["A_log"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.scan_fwd(inp["q"], inp["k"], inp["v"], inp["W_q"], inp["W_k"], dt=inp["dt"],
                        A_log=inp["A_log"])
    sec = (time.perf_counter() - t0) / max(1, args.steps)
    value = cfg.B * T / sec
    cores = min(oracle.omp_threads_in_use(), cfg.B * cfg.H)
    sample = ("fp64 CPU oracle, all %d (batch, head) pairs x %d tokens per step"
              % (cfg.B * cfg.H, T))
    return {
        "impl": "reference",
        "metric": "tokens/sec of HedgeMamba mixer scan fwd on 1 B200; % of tensor/HBM roofline",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.L, "H": cfg.H, "d": cfg.d,
                   "F": cfg.F, "dv": cfg.dv},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "long", "decode", "mixer", "block", "backward"],
                    default="long",
                    help="long: B1 H8 L32768 prefill (default, the largest single-GPU scan "
                         "workload); prefill: B4 H8 L2048; decode: 256 x 8 heads, 512 steps; "
                         "mixer: B8 L4096 D2048; block: the parallel block around that mixer "
                         "(MLP width 8192); backward: hm_scan_bwd on B4 H8 L2048")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (decode: sequences, mixer: B) for small "
                         "profiling captures; the reported config says so")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank, world, local = dist_env()

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.workload == "decode":
        res = bench_decode(wl.DECODE, args, rank, world, torch)
    elif args.workload in ("mixer", "block"):
        res = bench_mixer(wl.MIXER, args, rank, world, torch, block=args.workload == "block")
    elif args.workload == "backward":
        res = bench_backward(wl.PREFILL_PYTHIA, args, rank, world, torch)
    else:
        cfg = {"prefill": wl.PREFILL_PYTHIA, "long": wl.PREFILL_LONG}[args.workload]
        res = bench_prefill(cfg, args, rank, world, torch)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in ("prefill", "long"):
        rate, cores, sample, sec = oracle_prefill_rate(cfg)
        res["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": sample, "seconds": sec}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
