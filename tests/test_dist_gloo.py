"""The multi-rank plumbing of the benchmark on CPU with the gloo backend,
world size 2: per-rank seeds give independent batches, device time is the
max over ranks, and the whole-job rate counts every rank's bytes."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from decode_attention_07_b200.configs import WORKLOADS
from decode_attention_07_b200.inputs import bf16_bits, make_inputs


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["ragged_64k"].with_(B=2, Hq=4, Hkv=2, Lmax=128)
        x = make_inputs(w, bench.rank_seed(7, rank), device="cpu")
        digest = torch.tensor([float(bf16_bits(x.k).astype(np.int64).sum() % 1000003)], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        local_ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(local_ms, "cpu")
        result[rank] = (ms_max, [g.item() for g in gathered], int(x.seqlens_host.sum()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = free_port()
    with mp.Manager() as m:
        result = m.dict()
        mp.spawn(worker, args=(world, port, result), nprocs=world, join=True)
        res = dict(result)
    assert res[0][0] == res[1][0] == 15.0                  # max over ranks, same on every rank
    assert res[0][1] == res[1][1] and res[0][1][0] != res[0][1][1]   # independent batches per rank
    assert bench.whole_job_gbs(2, 1e9, 10, 20.0) == 2 * 1e9 * 10 / 0.02 / 1e9
