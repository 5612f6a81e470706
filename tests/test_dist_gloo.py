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


# ----------------------------------------- context parallelism (sequence sharding) --

def cp_worker(rank, world, port, result):
    """One rank of a sequence-sharded decode: attention over its token range
    (oracle, CPU), all-gather of the partials through the product's
    gather_partials, then the log-sum-exp reduction (oracle combine)."""
    import oracle
    from decode_attention_07_b200 import context
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["ragged_64k"].with_(B=3, Hq=4, Hkv=2, Lmax=150)
        x = make_inputs(w, 5, device="cpu", seqlens=[150, 40, 0])   # the same cache on every rank
        lo, hi = context.token_range(w.Lmax, rank, world)
        lens = context.local_seqlens(x.seqlens, lo).clamp(0, hi - lo).numpy().astype(np.int32)
        o, l = oracle.attention(bf16_bits(x.q), bf16_bits(x.k[:, :, lo:hi]), bf16_bits(x.v[:, :, lo:hi]), lens,
                                x.scale)
        all_o, all_l = context.gather_partials(torch.from_numpy(o), torch.from_numpy(l))
        R = all_o.shape[0]
        po = all_o.permute(1, 2, 0, 3).reshape(-1, R, w.D).numpy()      # rows x parts x D
        pl = all_l.permute(1, 2, 0).reshape(-1, R).numpy()
        mo, ml = oracle.combine(po, pl)
        ref_o, ref_l = oracle.attention(bf16_bits(x.q), bf16_bits(x.k), bf16_bits(x.v), x.seqlens_host, x.scale)
        err_o = float(np.abs(mo - ref_o.reshape(-1, w.D)).max())
        same_inf = bool(np.array_equal(np.isneginf(ml), np.isneginf(ref_l.reshape(-1))))
        fin = ~np.isneginf(ml)
        err_l = float(np.abs(ml[fin] - ref_l.reshape(-1)[fin]).max())
        result[rank] = (lo, hi, err_o, err_l, same_inf, R)
    finally:
        dist.destroy_process_group()


def test_context_parallel_two_ranks_gloo():
    world = 2
    port = free_port()
    with mp.Manager() as m:
        result = m.dict()
        mp.spawn(cp_worker, args=(world, port, result), nprocs=world, join=True)
        res = dict(result)
    assert (res[0][0], res[0][1], res[1][0], res[1][1]) == (0, 75, 75, 150)   # the ranges tile [0, Lmax)
    for r in range(world):
        _, _, err_o, err_l, same_inf, R = res[r]
        assert R == world and same_inf and err_o < 1e-12 and err_l < 1e-12


def test_token_ranges_tile_the_cache():
    from decode_attention_07_b200 import context
    for Lmax in (0, 1, 7, 64, 1000, 16384):
        for world in (1, 2, 3, 8):
            rs = [context.token_range(Lmax, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == Lmax
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            assert max(h - l for l, h in rs) - min(h - l for l, h in rs) <= 1


# ------------------------------------------------ bench.py --gpus N launcher --

def _bench(args, env_extra, timeout=300):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", **env_extra)   # the CPU path: gloo
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        if k not in env_extra:
            env.pop(k, None)
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=root, env=env, capture_output=True, text=True,
                       timeout=timeout)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return r, [json.loads(ln) for ln in lines]


def test_bench_gpus_flag_starts_one_process_per_rank():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself; both
    join one process group and rank 0 alone prints the line."""
    r, lines = _bench(["--gpus", "2", "--check-launch"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    assert len(lines) == 1
    d = lines[0]
    assert d["n_gpus"] == 2 and d["ranks_joined"] == 2 and d["backend"] == "gloo"
    assert len(set(d["pids"])) == 2 and os.getpid() not in d["pids"]


def test_bench_rejects_a_world_size_that_differs_from_gpus():
    r, lines = _bench(["--gpus", "2", "--check-launch"], {"WORLD_SIZE": "3", "RANK": "0"})
    assert r.returncode != 0 and not lines
    assert "WORLD_SIZE=3 but --gpus 2" in r.stderr


def test_bench_single_rank_needs_no_process_group():
    r, lines = _bench(["--check-launch"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    assert lines == [{"check_launch": True, "n_gpus": 1, "ranks_joined": 1, "pids": lines[0]["pids"],
                      "backend": None}]
