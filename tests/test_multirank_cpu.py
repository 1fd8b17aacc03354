"""The multi-rank host logic of the benchmark on CPU: two gloo ranks, each with
its own shard of sequences, agree on the slowest rank's time and on the
whole-job throughput (weak scaling, no collective on the data path), and take
a collective branch together when only one of them qualifies."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    from mla_latent_kv_43_b200 import inputs as gen
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = gen.WORKLOADS["tiny_fp32"]
        shard = bench.shard_workload(w, rank)
        host = gen.generate(shard)
        my_ms = 1.0 + rank                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(my_ms, world, device="cpu")
        bench.barrier(world, device="cpu")
        value = bench.job_throughput(shard.batch * shard.n_q, world, slowest)
        # every rank sees the other's checksum of its inputs
        csum = torch.tensor([float(host["q_nope"].double().sum())])
        allc = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(allc, csum)
        # a branch every rank must take together: taken only when all ranks qualify
        mixed = bench.all_ranks(rank == 0, world, device="cpu")
        both = bench.all_ranks(True, world, device="cpu")
        out[rank] = (slowest, value, shard.seed, [float(c) for c in allc], mixed, both)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (s0, v0, seed0, c0, m0, b0), (s1, v1, seed1, c1, m1, b1) = out[0], out[1]
    assert s0 == s1 == 2.0                        # max over ranks
    assert v0 == v1 == 2 * 2 / 2e-3               # 2 query tokens per rank, 2 ranks, 2 ms
    assert seed0 != seed1                         # distinct shards
    assert c0 == c1 and c0[0] != c0[1]            # the shards' inputs differ
    assert (m0, m1, b0, b1) == (False, False, True, True)
