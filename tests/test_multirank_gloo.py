"""The N > 1 path of bench.py on CPU: two gloo ranks (world size 2) run the
host logic that bench.py uses under torchrun -- per-rank seeded inputs of the
same shape, a barrier, the max of the ranks' times, and the whole-job
weak-scaling throughput -- without a GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench
    from quantized_attention_block_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        got_ws, got_rank, _ = bench._dist()
        w = W.small_variant(W.get("prefill"), N=256, B=1, Hq=2)
        q, k, v = W.make_qkv(w, seed=bench.rank_seed(w, got_rank))
        bench._barrier(got_ws)
        local_ms = 1.0 + got_rank  # rank 1 is the slow one
        ms_max = bench._max_over_ranks(local_ms, got_ws)
        value = bench.weak_scaling_tops(w.ops(), ms_max, got_ws)
        out[rank] = (got_ws, got_rank, tuple(q.shape), float(q.float().sum()), ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ws = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(ws, _free_port(), out), nprocs=ws, start_method="spawn", join=True)
    r0, r1 = out[0], out[1]
    assert (r0[0], r0[1]) == (2, 0) and (r1[0], r1[1]) == (2, 1)
    assert r0[2] == r1[2]                       # same per-rank workload shape (weak scaling)
    assert r0[3] != r1[3]                       # each rank draws its own inputs
    assert r0[4] == r1[4] == 2.0                # time of the slowest rank, seen by both
    from quantized_attention_block_b200 import workloads as W
    w = W.small_variant(W.get("prefill"), N=256, B=1, Hq=2)
    assert r0[5] == pytest.approx(2 * w.ops() / 2.0e-3 / 1e12)  # both ranks' ops / max time
