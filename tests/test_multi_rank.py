"""Multi-rank host logic of bench.py on CPU (gloo, world_size 2): each rank
draws an independent batch, timings combine as the max over ranks, and the
whole-job value counts every rank's tokens."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from chunk_wise_hierarchical_landmark_b200 import synth
    from chunk_wise_hierarchical_landmark_b200 import workloads as W
    w = W.PREFILL_128K.with_(Hq=2, Hkv=1, L=256)
    q, k, v, lmk = synth.make_inputs(w, "cpu", seed=w.seed + rank)  # per-rank seed offset
    gathered = [torch.empty_like(q) for _ in range(ws)]
    dist.all_gather(gathered, q)
    ms = 10.0 * (rank + 1)
    slowest = bench.max_over_ranks(ms, ws)
    value = bench.aggregate_value(w.B * w.L, ms, ws)
    assert bench.dist_env() == (ws, rank, rank)
    out[rank] = (slowest, value, bool(torch.equal(gathered[0], gathered[1])))
    bench.barrier(ws)
    dist.destroy_process_group()


def test_two_ranks_gloo():
    ws, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, join=True, start_method="spawn")
    for r in range(ws):
        slowest, value, same = out[r]
        assert slowest == 20.0                       # max over ranks
        assert value == pytest.approx(2 * 256 / 0.020)  # all ranks' tokens / slowest time
        assert not same                              # independent batches per rank
