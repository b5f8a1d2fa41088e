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


def _sequence_parallel_worker(rank, world, port, results):
    """Rank `rank` of a block split by token: the QK prologue on its token shard,
    an all-to-all to the head split (token order of the shards, heads
    head_range(.., world, j) to rank j), the oracle core on its heads over the
    whole sequence, the inverse all-to-all, all in fp64."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import dataclasses

        import numpy as np

        from diffusion_transformer_attention_bidirectional_b200 import seqpar
        from oracle import krea_oracle as ko
        from synth import inputs as S

        case = S.Case("seqpar", 1, 4, 2, 64, 16, 8, 8, dtype="f16", mode="scanline", window=3, gate=True,
                      prologue=True, seed=7)
        L, Ls = case.seq_len, case.seq_len // world
        q, k, v, g = S.make_inputs(case)
        pos = ko.rope_positions(case.text_len, case.grid_h, case.grid_w)
        t0, t1 = seqpar.token_range(Ls, rank)
        mine = {"q": torch.from_numpy(ko.qk_prologue(q[:, t0:t1], pos[t0:t1])),
                "k": torch.from_numpy(ko.qk_prologue(k[:, t0:t1], pos[t0:t1])),
                "v": v[:, t0:t1].double(), "g": g[:, t0:t1].double()}

        def to_heads(x):  # [1, Ls, H, d] token shard -> [1, L, H / world, d] head shard
            H = x.shape[2]
            send = torch.stack([x[:, :, slice(*seqpar.head_range(H, world, j))] for j in range(world)]).contiguous()
            recv = torch.empty_like(send)
            dist.all_to_all_single(recv, send)
            return torch.cat(list(recv), dim=1)  # source ranks hold consecutive token ranges

        def to_seq(y):  # [1, L, Hr, d] head shard -> [1, Ls, world * Hr, d] token shard
            send = torch.stack([y[:, slice(*seqpar.token_range(Ls, j))] for j in range(world)]).contiguous()
            recv = torch.empty_like(send)
            dist.all_to_all_single(recv, send)
            return torch.cat(list(recv), dim=2)  # source rank j held heads head_range(.., j)

        h = {n: to_heads(x) for n, x in mine.items()}
        sub = dataclasses.replace(case, q_heads=case.q_heads // world, kv_heads=case.kv_heads // world)
        o_heads = torch.from_numpy(ko.attention(sub, h["q"], h["k"], h["v"], h["g"])["out"])
        o_mine = to_seq(o_heads).numpy()
        full = ko.attention(case, ko.qk_prologue(q, pos), ko.qk_prologue(k, pos), v, g)["out"]
        results[rank] = float(np.abs(o_mine - full[:, t0:t1]).max())
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_split_reassembles_the_core():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_sequence_parallel_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    for r in range(world):
        assert results[r] < 1e-12, results[r]


def test_sequence_parallel_ranges():
    from diffusion_transformer_attention_bidirectional_b200 import seqpar

    assert [seqpar.head_range(48, 4, j) for j in range(4)] == [(0, 12), (12, 24), (24, 36), (36, 48)]
    assert [seqpar.head_range(12, 4, j) for j in range(4)] == [(0, 3), (3, 6), (6, 9), (9, 12)]
    # query head h reads kv head h // 4, and both land on the same rank
    for W in (1, 2, 3, 4, 6, 12):
        for h in range(48):
            j = next(r for r in range(W) if seqpar.head_range(48, W, r)[0] <= h < seqpar.head_range(48, W, r)[1])
            a, b = seqpar.head_range(12, W, j)
            assert a <= h // 4 < b
    assert seqpar.token_range(1152, 3) == (3456, 4608)
    import pytest

    with pytest.raises(ValueError):
        seqpar.head_range(12, 5, 0)


def _sequence_parallel_class_worker(rank, world, port, shared_dir, results):
    """SequenceParallelAttention with world = 2 on gloo ranks. Its host logic runs
    unchanged: buffer allocation, the exchange of handles, the tables of
    destinations in rank order, the barriers. What runs on a GPU is replaced:
    buffers are file-backed shared arrays (the handle is the path), the pushes
    write into them by the layout rule of the C ABI, and the core and the
    prologue are the fp64 oracle."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import dataclasses
        import json
        import tempfile

        import numpy as np

        from diffusion_transformer_attention_bidirectional_b200 import seqpar
        from oracle import krea_oracle as ko
        from synth import inputs as S

        arrays = {}  # fake "device pointer" -> the shared array it addresses

        class FileBuffer:
            def __init__(self, shape, dtype):
                fd, self.path = tempfile.mkstemp(dir=shared_dir)
                os.close(fd)
                self.shape = tuple(shape)
                self.arr = np.memmap(self.path, dtype=np.float64, mode="w+", shape=self.shape)
                self.arr[...] = np.nan
                self.ptr = id(self.arr)
                arrays[self.ptr] = self.arr

            def handle_bytes(self):
                return json.dumps([self.path, self.shape]).encode()

            def tensor(self):
                return torch.from_numpy(self.arr)

        class FileMapping:
            def __init__(self, handle):
                path, shape = json.loads(handle.decode())
                self.arr = np.memmap(path, dtype=np.float64, mode="r+", shape=tuple(shape))
                self.ptr = id(self.arr)
                arrays[self.ptr] = self.arr

        case = S.Case("seqpar_cls", 1, 4, 2, 64, 16, 8, 8, dtype="f16", mode="scanline", window=3, gate=True,
                      prologue=True, seed=9)
        L, Ls = case.seq_len, case.seq_len // world
        pos = ko.rope_positions(case.text_len, case.grid_h, case.grid_w)

        def push_heads(y, dests, r):  # the rule of krea_attn_seq_to_heads
            H = y.shape[2]
            hpr = H // dests.world
            for h in range(H):
                arrays[dests.ptrs[h // hpr]][:, r * Ls:(r + 1) * Ls, h % hpr] = y[:, :, h]

        def fake_prologue(x, table, dests, r, gamma=None, rope=None):
            push_heads(ko.qk_prologue(x, table[r * Ls:(r + 1) * Ls]), dests, r)

        def fake_seq_to_heads(x, dests, r):
            push_heads(np.asarray(x, dtype=np.float64), dests, r)

        def fake_heads_to_seq(y, dests, r):  # the rule of krea_attn_heads_to_seq
            y = np.asarray(y)
            Hr = y.shape[2]
            for t in range(y.shape[1]):
                arrays[dests.ptrs[t // Ls]][:, t % Ls, r * Hr:(r + 1) * Hr] = y[:, t]

        def fake_core(q, k, v, gate, *, out, **kw):
            sub = dataclasses.replace(case, q_heads=q.shape[2], kv_heads=k.shape[2])
            out[...] = torch.from_numpy(ko.attention(sub, q, k, v, gate)["out"])

        seqpar.qk_prologue_to_heads = fake_prologue
        seqpar.seq_to_heads = fake_seq_to_heads
        seqpar.heads_to_seq = fake_heads_to_seq
        seqpar._core = fake_core
        seqpar.SequenceParallelAttention.buffer_cls = FileBuffer
        seqpar.SequenceParallelAttention.mapping_cls = FileMapping
        # a gloo group is refused on the real path (its all-reduce is not ordered
        # on a CUDA stream); here every buffer is host memory, so it orders them
        try:
            seqpar.SequenceParallelAttention(1, Ls, case.q_heads, case.kv_heads, case.head_dim,
                                             dtype=torch.float64, out_dtype=torch.float64, device="cpu")
            raise AssertionError("a gloo group was accepted")
        except RuntimeError as e:
            assert "ordered on the CUDA stream" in str(e)
        seqpar.SequenceParallelAttention.barrier_backends = ("gloo",)

        spa = seqpar.SequenceParallelAttention(1, Ls, case.q_heads, case.kv_heads, case.head_dim,
                                               dtype=torch.float64, out_dtype=torch.float64, device="cpu")
        assert spa.world == world and spa.rank == rank
        q, k, v, g = S.make_inputs(case)
        t0, t1 = seqpar.token_range(Ls, rank)
        out = spa(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1].double(), g[:, t0:t1].double(), pos,
                  text_len=case.text_len, grid_h=case.grid_h, grid_w=case.grid_w, mode="scanline", window=3)
        full = ko.attention(case, ko.qk_prologue(q, pos), ko.qk_prologue(k, pos), v, g)["out"]
        results[rank] = float(np.abs(out.numpy() - full[:, t0:t1]).max())
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_attention_two_ranks_host_logic(tmp_path):
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_sequence_parallel_class_worker, args=(world, _free_port(), str(tmp_path), results), nprocs=world,
             join=True)
    for r in range(world):
        assert results[r] < 1e-12, results[r]
