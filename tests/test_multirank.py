"""Multi-rank host logic of the data-parallel decode, on CPU with gloo (world size 2).

The decode step shards over sequences: each rank owns a disjoint batch and no
data crosses ranks; only the timing reduction (max over ranks) is collective.
These tests run that host path without a GPU: the reduction, the per-rank
workloads, and that per-rank oracle decodes of the shards, gathered, equal one
decode of the whole batch.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))


def _worker(rank: int, port: int, out_dir: str):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import bench
    from latent_kv_decode_b200 import workloads as wl
    from oracle import mla as omla

    _init(rank, port)
    try:
        res = {}
        # 1. max over ranks, as the bench reduces its step times
        res["max"] = bench.max_over_ranks([rank + 1.0, 10.0 - rank], dist)
        # 2. per-rank workloads: same shape, distinct data
        w = bench.make_workload("dsv3_b2_lk64", rank)
        shapes = [w.q_nope.shape, w.kv_cache.shape, w.wkv_b.shape]
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, (shapes, float(w.q_nope[0, 0, 0, 0])))
        res["shapes_equal"] = all(g[0] == shapes for g in gathered)
        res["data_distinct"] = len({g[1] for g in gathered}) == WORLD
        # 3. sharded decode: this rank's sequences of one job (shared weights)
        job = wl.make_mla(B=2 * WORLD, H=8, Q=2, Dn=64, Dr=32, Vd=64, Ckv=128, Lk=80,
                          dtype="f32", seed=7, lk_range=(1, 80), causal=True)
        sel = slice(2 * rank, 2 * rank + 2)
        out = omla.mla_decode_step(job.q_nope[sel], job.q_pe[sel], job.kv_cache[sel],
                                   job.pe_cache[sel], job.wkv_b, job.softmax_scale,
                                   seq_lens=job.seq_lens[sel], causal=True)
        parts = [None] * WORLD
        dist.all_gather_object(parts, np.asarray(out))
        if rank == 0:
            whole = omla.mla_decode_step(job.q_nope, job.q_pe, job.kv_cache, job.pe_cache,
                                         job.wkv_b, job.softmax_scale, seq_lens=job.seq_lens,
                                         causal=True)
            res["shard_err"] = float(np.max(np.abs(np.concatenate(parts, axis=0) - whole)))
            res["shard_scale"] = float(np.max(np.abs(whole)))
        res["tokens_per_s"] = bench.job_tokens_per_s(64, 1, WORLD, 2.0)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), res, allow_pickle=True)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("multirank")
    mp.start_processes(_worker, args=(_free_port(), str(out)), nprocs=WORLD, join=True,
                       start_method="spawn")
    return [np.load(out / f"rank{r}.npy", allow_pickle=True).item() for r in range(WORLD)]


def test_max_over_ranks_is_elementwise_max_on_every_rank(results):
    for r in results:
        assert r["max"] == [2.0, 10.0]


def test_ranks_get_same_shape_distinct_data(results):
    assert all(r["shapes_equal"] for r in results)
    assert all(r["data_distinct"] for r in results)


def test_sharded_oracle_decode_equals_whole_batch(results):
    r0 = results[0]
    assert r0["shard_err"] <= 1e-12 * max(1.0, r0["shard_scale"])


def test_job_throughput_counts_every_rank(results):
    # 64 rows per rank, 2 ranks, 2 ms per step -> 64000 rows/s
    assert all(abs(r["tokens_per_s"] - 64000.0) < 1e-6 for r in results)
