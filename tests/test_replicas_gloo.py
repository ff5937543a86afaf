"""Multi-process (world size 2, gloo, CPU) checks of the replica plumbing that
bench.py uses under torchrun: each rank owns independent work, results do not
depend on the number of ranks, and the timing is the max over ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        # independent matrices, sharded across ranks: each rank quantizes its own
        n_items = 5
        mine = {}
        for i in bench.shard(n_items, rank, world):
            W = synth.bits(synth.normal_bf16((64, 256), 0.02, seed=i, outlier_frac=0.01))
            mine[i] = oracle.quantize_pack(W)[0].sum(dtype=np.int64).item()
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        t = bench.max_over_ranks(float(rank + 1) * 0.5, world)
        out[rank] = (gathered, t)
    finally:
        dist.destroy_process_group()


def test_two_replicas_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    import oracle
    import synth
    want = {}
    for i in range(5):
        W = synth.bits(synth.normal_bf16((64, 256), 0.02, seed=i, outlier_frac=0.01))
        want[i] = oracle.quantize_pack(W)[0].sum(dtype=np.int64).item()
    for r in range(world):
        gathered, t = out[r]
        merged = {}
        for d in gathered:
            assert not (set(d) & set(merged)), "a work item ran on two ranks"
            merged.update(d)
        assert merged == want
        assert t == 1.0                       # max over ranks of 0.5, 1.0


def test_shard_partitions():
    for n in [0, 1, 5, 96]:
        for world in [1, 2, 3, 8]:
            parts = [list(bench.shard(n, r, world)) for r in range(world)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
