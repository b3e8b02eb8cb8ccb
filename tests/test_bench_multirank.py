"""The benchmark's multi-GPU path is N independent replicas: every rank owns
its own requests and the only collective is the max of the step time.  This
runs that host-side logic as two gloo ranks on the CPU."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens, tables, nb = bench.replica_workload(rank)
        fake_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(fake_ms)
        value, tok = bench.job_throughput(bench.kv_bytes(lens) * bench.LAYERS, world, ms)
        out[rank] = (int(lens.sum()), int(nb), tables[0, :4].tolist(), ms, value, tok)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # replicas own different requests
    assert res[0][0] != res[1][0] or res[0][2] != res[1][2]
    # both ranks see the max over ranks
    assert res[0][3] == res[1][3] == 15.0
    # whole-job throughput counts every rank's work over the slowest rank's time
    lens0, _, _ = bench.replica_workload(0)
    want = bench.kv_bytes(lens0) * bench.LAYERS * world / 15e-3 / 1e9
    assert abs(res[0][4] - want) / want < 1e-12
    assert abs(res[0][5] - bench.S * world / 15e-3) < 1e-6


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
