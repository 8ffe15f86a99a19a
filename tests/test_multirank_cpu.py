"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The path shards into independent layers per rank with no data-path
collective; the only cross-rank steps are a barrier and the maximum of the
per-rank step time.  These run here with gloo ranks on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(synth.WORKLOADS["llama8b_decode"], rank)
        ms = 10.0 + 5.0 * rank                     # the slower rank sets the time
        ms_max = bench.max_over_ranks(dist, ms, torch.device("cpu"))
        dist.barrier()
        k = synth.kv_slab(w, "K", 0, 0, 0, 4)     # each rank's own data
        out[rank] = (w.data_seed, ms_max, bench.whole_job_value(w.n_keys, world, ms_max), k.float().sum().item())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_the_max_time():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][1] == res[1][1] == 15.0
    assert res[0][0] != res[1][0]                   # distinct data per rank
    assert res[0][3] != res[1][3]
    n = synth.WORKLOADS["llama8b_decode"].n_keys
    assert res[0][2] == pytest.approx(2 * n / 15e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(None, 3.5, None) == 3.5
    assert bench.whole_job_value(1000, 1, 2.0) == pytest.approx(5e5)
