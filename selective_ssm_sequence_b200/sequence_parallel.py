"""Sequence-parallel prefill: one long sequence cut into consecutive segments,
one segment per rank (one process per GPU, torch.distributed over NCCL).

The recurrence S_t = a_t S_{t-1} + phi(k_t) v_t^T (and z likewise) makes each
segment an affine map of the state it starts from, S -> exp(lambda) S + S_seg,
where lambda is the segment's summed log decay and S_seg its end state from a
zero start.  These maps compose associatively (SSM article sec. 4.2), so:

  1. every rank runs a state-only scan of its own segment from a zero start
     (hm_scan_chunked_fwd with o = NULL, S_out, z_out, log_decay_out);
  2. one all-gather exchanges the [log_decay | S | z] records (per head:
     1 + F*dv + F fp32 values, about 263 KB for F = dv = 256);
  3. each rank composes the records of the ranks before it (hm_scan_combine
     with only_part = rank) into its segment's start state;
  4. each rank scans its segment from that start (hm_scan_chunked_fwd with S0)
     and writes its outputs; the last rank's S_out is the sequence's final state.

This module only orders the C-ABI calls and the collective; every arithmetic
step runs in libhm's kernels.  The compute steps are taken from an `ops`
object so that the ordering and the exchange can be exercised without a GPU;
the default is the library itself (`LibOps`).
"""
from __future__ import annotations


class LibOps:
    """The three compute steps, on CUDA tensors through libhm."""

    def __init__(self, hm=None):
        if hm is None:
            import selective_ssm_sequence_b200 as hm
        self.hm = hm

    def empty(self, n: int, like):
        import torch
        return torch.empty(n, dtype=torch.float32, device=like.device)

    def _ws(self, args):
        ws = self.hm.alloc_workspace(self.hm.hm_scan_workspace_size(args), args._refs[1].device)
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        return ws

    def segment_record(self, seg, record, BH, F, dv, flags):
        """State-only scan of the segment from a zero start into `record`
        ([log_decay (padded) | S | z], fp32)."""
        hm = self.hm
        nl = BH * F if flags & hm.HM_FLAG_PER_FEATURE_DECAY else BH
        off_S = (nl + 3) // 4 * 4
        off_z = off_S + BH * F * dv
        lam = record[:nl]
        S = record[off_S:off_z].view(-1)
        z = record[off_z:off_z + BH * F]
        B, L, H = seg["k"].shape[:3]
        a = hm.scan_args(None, seg["k"], seg["v"], None, W_q=seg.get("W_q"), W_k=seg.get("W_k"),
                         dt=seg.get("dt"), A_log=seg.get("A_log"), S_out=S, z_out=z, flags=flags,
                         b_q=seg.get("b_q"), b_k=seg.get("b_k"), w_head_stride=seg.get("w_head_stride", 0),
                         log_decay_out=lam, rope_base=seg.get("rope_base", 0.0), pos0=seg.get("pos0", 0))
        ws = self._ws(a)
        hm.hm_scan_chunked_fwd(a)
        del ws

    def start_state(self, gathered, n_parts, rank, BH, F, dv, flags, S0, z0, S_start, z_start):
        hm = self.hm
        a = hm.combine_args(gathered, n_parts, BH, F, dv, hm.combine_record_len(BH, F, dv, bool(
            flags & hm.HM_FLAG_PER_FEATURE_DECAY)), S_start, z_start,
            per_feature=bool(flags & hm.HM_FLAG_PER_FEATURE_DECAY), S0=S0, z0=z0, only_part=rank)
        hm.hm_scan_combine(a)

    def scan(self, seg, o, S0, z0, S_out, z_out, flags):
        hm = self.hm
        a = hm.scan_args(seg["q"], seg["k"], seg["v"], o, W_q=seg.get("W_q"), W_k=seg.get("W_k"),
                         dt=seg.get("dt"), A_log=seg.get("A_log"), S0=S0, z0=z0, S_out=S_out, z_out=z_out,
                         flags=flags, b_q=seg.get("b_q"), b_k=seg.get("b_k"),
                         w_head_stride=seg.get("w_head_stride", 0), rope_base=seg.get("rope_base", 0.0),
                         pos0=seg.get("pos0", 0))
        ws = self._ws(a)
        hm.hm_scan_chunked_fwd(a)
        del ws


def record_len(BH: int, F: int, dv: int, per_feature: bool) -> int:
    """fp32 values of one rank's [log_decay | S | z] record (log decay padded to 4)."""
    nl = BH * F if per_feature else BH
    return (nl + 3) // 4 * 4 + BH * F * dv + BH * F


def prefill_sequence_parallel(seg: dict, o, F: int, flags: int = 0, S0=None, z0=None, S_out=None,
                              z_out=None, group=None, ops=None) -> None:
    """Prefill of one sequence split over the ranks of `group`.

    seg: this rank's consecutive token range, as tensors q, k [B, Ls, H, d],
    v [B, Ls, H, dv] and optionally W_q, W_k, dt [B, Ls, H], A_log, biases;
    with HM_FLAG_ROPE also "rope_base" and "pos0" (the position of this rank's
    first token); rank r holds tokens after those of ranks 0..r-1.
    o [B, Ls, H, dv] gets this segment's outputs.  S0, z0: the state before rank 0's tokens (only
    rank 0's arguments are used; NULL = zero).  S_out, z_out: this rank's end
    state, i.e. on the last rank the state after the whole sequence.
    F is the feature dimension (2p with Hedgehog weights, else d)."""
    import torch
    import torch.distributed as dist
    ops = ops or LibOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    k = seg["k"]
    B, _, H = k.shape[:3]
    dv = seg["v"].shape[-1]
    BH = B * H
    per_feature = bool(flags & 2)
    n = record_len(BH, F, dv, per_feature)
    mine = ops.empty(n, k)
    mine.zero_()
    ops.segment_record(seg, mine, BH, F, dv, flags)
    # the exchange: every rank's record, in rank order (one collective)
    parts = [ops.empty(n, k) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    gathered = torch.cat(parts)
    # the initial state lives on rank 0; the others learn whether there is one,
    # and its value, through these broadcasts
    has0 = torch.tensor([1 if (rank == 0 and S0 is not None) else 0], dtype=torch.int32, device=k.device)
    dist.broadcast(has0, src=dist.get_global_rank(group, 0) if group is not None else 0, group=group)
    if int(has0.item()):
        init = ops.empty(BH * F * dv + BH * F, k)
        if rank == 0:
            init[:BH * F * dv].copy_(S0.reshape(-1))
            init[BH * F * dv:].copy_(z0.reshape(-1))
        dist.broadcast(init, src=dist.get_global_rank(group, 0) if group is not None else 0, group=group)
        S_init, z_init = init[:BH * F * dv], init[BH * F * dv:]
    else:
        S_init = z_init = None
    S_start = ops.empty(BH * F * dv, k)
    z_start = ops.empty(BH * F, k)
    ops.start_state(gathered, world, rank, BH, F, dv, flags, S_init, z_init, S_start, z_start)
    ops.scan(seg, o, S_start.view(B, H, F, dv), z_start.view(B, H, F), S_out, z_out, flags)
