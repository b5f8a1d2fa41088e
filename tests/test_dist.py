"""The multi-process path on CPU: two gloo ranks. Timings are combined as the
max over ranks and throughput counts every rank's work; the head partition
covers every (batch, kv head) unit exactly once and reassembles the full
output."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from diffusion_transformer_attention_bidirectional_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        local_ms = [12.5, 20.0][rank]
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.job_throughput(1e12, world, ms)
        # each rank fills its share of a [B, L, Hq, d] output through the views
        B, L, Hq, Hkv, d = 2, 5, 12, 6, 4
        q = torch.zeros(B, L, Hq, d)
        k = torch.zeros(B, L, Hkv, d)
        out = torch.full((B, L, Hq, d), -1.0)
        _, _, _, _, o = shard.shard_views(q, k, k, None, out, rank, world)
        o.fill_(float(rank))
        mine = out.clone()
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        full = torch.full_like(out, -1.0)
        for r, t in enumerate(gathered):
            g0, g1 = shard.kv_head_range(Hkv, r, world)
            rep = Hq // Hkv
            full[:, :, g0 * rep:g1 * rep] = t[:, :, g0 * rep:g1 * rep]
        results[rank] = (ms, value, bool((full >= 0).all()), full[0, 0, :, 0].tolist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    for r in range(world):
        ms, value, covered, heads = results[r]
        assert ms == 20.0                     # the max over ranks
        assert abs(value - 2 * 1e12 / 20e-3 / 1e12) < 1e-9
        assert covered
        assert heads == [0.0] * 6 + [1.0] * 6  # rank 0: kv heads 0-2 -> q heads 0-5


def test_partition_covers_units_once():
    for Hkv in (1, 5, 12):
        for world in (1, 2, 3, 4, 8):
            parts = shard.partition(Hkv, world)
            covered = [g for a, b in parts for g in range(a, b)]
            assert covered == list(range(Hkv))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
