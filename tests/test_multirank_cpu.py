"""The N > 1 benchmark path on CPU: two gloo ranks (127.0.0.1) each take
their own seeded batch (no data-path collective: the work shards by batch),
the per-rank times are reduced to the slowest, and the whole-job rate counts
every rank's units."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=8, seed=bench.rank_seed(cfg.seed, rank))
    # a stand-in per-rank time; the slowest must win
    my_ms = 1.0 + rank
    ms = bench.max_over_ranks(my_ms, world, torch, device="cpu")
    rate = bench.whole_job_rate(cfg.B * cfg.L, world, ms)
    out[rank] = (float(inp["q"][0, 0, 0, 0]), ms, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_batch_and_take_the_slowest_time():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    (q0, ms0, r0), (q1, ms1, r1) = out[0], out[1]
    assert q0 != q1                   # different seeded batches per rank
    assert ms0 == ms1 == 2.0          # max over ranks
    assert r0 == r1 == pytest.approx(4 * 2048 * 2 / 2e-3)
