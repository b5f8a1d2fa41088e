"""Sequence-parallel callers: the joint [text, image] sequence moved between a
split by token and a split by head around the attention core.

A block that keeps its activations split by token across `world` ranks (rank r
holds tokens [r * Ls, (r + 1) * Ls)) hands the core, on rank j, the whole
sequence of a slice of the heads: query heads [j Hq / world, (j + 1) Hq / world)
and the kv heads they read, [j Hkv / world, (j + 1) Hkv / world) (query head h
reads kv head h // (Hq / Hkv), the repeat_interleave order of "Krea 2 TileMix
Attention (FP16/INT8 tiles)", section "What it actually patches"). Heads are
independent, so the core runs unchanged; the pages themselves describe no
multi-GPU split.

Every copy is a push by this library's kernels into the owner's buffer in its
final layout: peer memory (a CUDA IPC mapping over NVLink) for other ranks, this
GPU's memory for itself. `Destinations` is the table of those buffers as one
process addresses them. The caller orders the ranks (`SequenceParallelAttention`
does it with one-element all-reduces on the stream).
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import check, lib

_DT = {torch.float16: _lib.DTYPE["f16"], torch.bfloat16: _lib.DTYPE["bf16"], torch.float32: _lib.DTYPE["f32"]}


def token_range(tokens_per_rank: int, rank: int) -> Tuple[int, int]:
    """Tokens [start, stop) of the joint sequence held by `rank`."""
    return rank * tokens_per_rank, (rank + 1) * tokens_per_rank


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Heads [start, stop) that `rank` attends over (heads % world == 0)."""
    if heads % world:
        raise ValueError(f"{heads} heads do not split over {world} ranks")
    n = heads // world
    return rank * n, (rank + 1) * n


class Destinations:
    """dst[j] of every rank j as this process addresses it, with the (b, token,
    head) element strides that all of them share."""

    def __init__(self, ptrs: Sequence[int], strides: Sequence[int], dtype: torch.dtype):
        if not 1 <= len(ptrs) <= _lib.EXCHANGE_MAX_RANKS:
            raise ValueError("between 1 and 16 ranks")
        self.ptrs = [int(p) for p in ptrs]
        self.strides = tuple(int(s) for s in strides[:3])
        self.dtype = dtype

    @classmethod
    def of(cls, tensors: Sequence[torch.Tensor]) -> "Destinations":
        """From tensors of one shape, dtype and strides (this GPU's memory)."""
        t0 = tensors[0]
        for t in tensors:
            if not t.is_cuda:
                raise ValueError("destinations are CUDA tensors")
            if t.shape != t0.shape or t.stride() != t0.stride() or t.dtype != t0.dtype:
                raise ValueError("every destination has the same shape, strides and dtype")
            if t.stride(3) != 1:
                raise ValueError("head_dim must be contiguous")
        return cls([t.data_ptr() for t in tensors], t0.stride()[:3], t0.dtype)

    @property
    def world(self) -> int:
        return len(self.ptrs)

    def struct(self, rank: int, tokens_per_rank: int) -> _lib.Exchange:
        ex = _lib.Exchange()
        ex.world = self.world
        ex.rank = rank
        ex.tokens_per_rank = tokens_per_rank
        ex.reserved = 0
        for j, p in enumerate(self.ptrs):
            ex.dst[j] = p
        for i in range(3):
            ex.dst_stride[i] = self.strides[i]
        return ex


def _stream(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _check_src(x: torch.Tensor, dests: Destinations) -> None:
    if not x.is_cuda:
        raise ValueError("the source is a CUDA tensor")
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("the source is [B, tokens, heads, head_dim] with head_dim contiguous")
    if x.dtype != dests.dtype:
        raise ValueError("source and destinations have one dtype")


def seq_to_heads(x: torch.Tensor, dests: Destinations, rank: int, stream=None) -> None:
    """This rank's token shard x [B, Ls, H, d] into every rank's head shard:
    row (b, t, h) -> dests[h // (H / world)] at (b, rank * Ls + t, h % (H / world))."""
    _check_src(x, dests)
    B, Ls, H, d = x.shape
    ex = dests.struct(rank, Ls)
    xs = (ctypes.c_int64 * 3)(*x.stride()[:3])
    check(lib().krea_attn_seq_to_heads(x.data_ptr(), B, H, d, _DT[x.dtype], xs, ctypes.byref(ex),
                                       _stream(stream, x.device)), "seq_to_heads")


def heads_to_seq(y: torch.Tensor, dests: Destinations, rank: int, stream=None) -> None:
    """This rank's heads over the whole sequence, y [B, world * Ls, Hr, d], back to
    every rank's token shard: row (b, t, h) -> dests[t // Ls] at (b, t % Ls, rank * Hr + h)."""
    _check_src(y, dests)
    B, L, Hr, d = y.shape
    if L % dests.world:
        raise ValueError("the sequence does not split evenly over the ranks")
    ex = dests.struct(rank, L // dests.world)
    ys = (ctypes.c_int64 * 3)(*y.stride()[:3])
    check(lib().krea_attn_heads_to_seq(y.data_ptr(), B, Hr, d, _DT[y.dtype], ys, ctypes.byref(ex),
                                       _stream(stream, y.device)), "heads_to_seq")


def qk_prologue_to_heads(x: torch.Tensor, table: torch.Tensor, dests: Destinations, rank: int,
                         gamma: Optional[torch.Tensor] = None, rope: Optional[_lib.RopeParams] = None,
                         stream=None) -> None:
    """RMSNorm + 3-axis RoPE of this rank's token shard x [B, Ls, H, d], stored as
    seq_to_heads stores rows; `table` covers the whole sequence (row rank * Ls + t)."""
    from . import rope_params

    _check_src(x, dests)
    B, Ls, H, d = x.shape
    rope = rope if rope is not None else rope_params(d)
    g = gamma.to(torch.float32).contiguous() if gamma is not None else None
    ex = dests.struct(rank, Ls)
    xs = (ctypes.c_int64 * 3)(*x.stride()[:3])
    check(lib().krea_attn_qk_prologue_to_heads(x.data_ptr(), g.data_ptr() if g is not None else None,
                                               table.data_ptr(), B, H, d, _DT[x.dtype], xs, ctypes.byref(rope),
                                               ctypes.byref(ex), _stream(stream, x.device)),
          "qk_prologue_to_heads")


# ----------------------------------------------------------------------------- buffers other ranks map
_TYPESTR = {torch.float16: "<f2", torch.float32: "<f4", torch.bfloat16: "<i2"}  # bf16 travels as int16


class _DeviceArray:
    """A device buffer described by __cuda_array_interface__, for torch.as_tensor."""

    def __init__(self, ptr: int, shape, dtype: torch.dtype, owner):
        self._owner = owner  # keeps the allocation or mapping alive while a tensor views it
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": _TYPESTR[dtype],
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class PeerBuffer:
    """A contiguous [shape] buffer of this GPU that other processes can map."""

    def __init__(self, shape, dtype: torch.dtype):
        self.shape, self.dtype = tuple(shape), dtype
        n = 1
        for s in self.shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        ptr = ctypes.c_void_p()
        self.handle = (ctypes.c_ubyte * _lib.IPC_HANDLE_BYTES)()
        check(lib().krea_attn_ipc_alloc(nbytes, ctypes.byref(ptr), self.handle), "ipc_alloc")
        self.ptr = ptr.value

    def handle_bytes(self) -> bytes:
        return bytes(self.handle)

    def tensor(self) -> torch.Tensor:
        t = torch.as_tensor(_DeviceArray(self.ptr, self.shape, self.dtype, self), device="cuda")
        return t.view(torch.bfloat16) if self.dtype == torch.bfloat16 else t

    def __del__(self):
        if getattr(self, "ptr", None):
            lib().krea_attn_ipc_free(self.ptr)
            self.ptr = None


class PeerMapping:
    """Another process's PeerBuffer mapped into this one (its device pointer only)."""

    def __init__(self, handle: bytes):
        buf = (ctypes.c_ubyte * _lib.IPC_HANDLE_BYTES).from_buffer_copy(handle)
        ptr = ctypes.c_void_p()
        check(lib().krea_attn_ipc_open(buf, ctypes.byref(ptr)), "ipc_open")
        self.ptr = ptr.value

    def __del__(self):
        if getattr(self, "ptr", None):
            lib().krea_attn_ipc_close(self.ptr)
            self.ptr = None


# ----------------------------------------------------------------------------- one rank's end
def _core(q, k, v, gate, **kw):
    """The attention core on this rank's heads over the whole sequence."""
    from . import attention

    return attention(q, k, v, gate, **kw)


class SequenceParallelAttention:
    """The attention core for a block whose activations are split by token over
    the ranks of `group` (None: one rank). Per call: q and k through the QK
    prologue straight into the owners' head shards, v and gate copied the same
    way, the core on this rank's heads over the whole sequence, its output pushed
    back to the token shards. Buffers are allocated once; the handles of other
    ranks' buffers are exchanged with all_gather_object when world > 1, so each
    process sets its own device (torch.cuda.set_device) before building one, and
    all ranks build theirs together. Ranks of one node only (CUDA IPC)."""

    # how buffers other ranks map are made and opened (CUDA IPC)
    buffer_cls = PeerBuffer
    mapping_cls = PeerMapping
    # Process-group backends whose all-reduce orders the ranks' device work: NCCL
    # runs it on the current CUDA stream, so every rank's stores into peer buffers
    # issued before it have completed when work after it starts. Other backends
    # give no such ordering on the stream; world > 1 refuses them.
    barrier_backends = ("nccl",)

    def __init__(self, batch: int, tokens_per_rank: int, q_heads: int, kv_heads: int, head_dim: int,
                 dtype: torch.dtype = torch.bfloat16, out_dtype: torch.dtype = torch.float32, group=None,
                 with_gate: bool = True, device="cuda"):
        import torch.distributed as dist

        self.group = group
        if group is not None or (dist.is_available() and dist.is_initialized()):
            self.world, self.rank = dist.get_world_size(group), dist.get_rank(group)
        else:
            self.world, self.rank = 1, 0
        W = self.world
        head_range(q_heads, W, 0)
        head_range(kv_heads, W, 0)
        self.B, self.Ls, self.d = batch, tokens_per_rank, head_dim
        self.Hq, self.Hkv, self.dtype, self.out_dtype = q_heads, kv_heads, dtype, out_dtype
        L = W * tokens_per_rank
        shapes = {"q": ((batch, L, q_heads // W, head_dim), dtype), "k": ((batch, L, kv_heads // W, head_dim), dtype),
                  "v": ((batch, L, kv_heads // W, head_dim), dtype),
                  "out": ((batch, tokens_per_rank, q_heads, head_dim), out_dtype)}
        if with_gate:
            shapes["gate"] = ((batch, L, q_heads // W, head_dim), dtype)
        self.local, self.dests, self._keep = {}, {}, []
        if W == 1:
            for name, (shape, dt) in shapes.items():
                self.local[name] = torch.empty(shape, dtype=dt, device=device)
                self.dests[name] = Destinations.of([self.local[name]])
            self.o_heads = torch.empty((batch, L, q_heads, head_dim), dtype=out_dtype, device=device)
            return
        backend = dist.get_backend(group)
        if backend not in self.barrier_backends:
            raise RuntimeError(f"SequenceParallelAttention over {W} ranks needs a process group whose "
                               f"collectives are ordered on the CUDA stream ({', '.join(self.barrier_backends)}); "
                               f"got {backend}")
        own = {name: self.buffer_cls(shape, dt) for name, (shape, dt) in shapes.items()}
        self._keep.append(own)
        handles = {name: b.handle_bytes() for name, b in own.items()}
        gathered: List[dict] = [None] * W
        dist.all_gather_object(gathered, handles, group=group)
        for name, (shape, dt) in shapes.items():
            ptrs = []
            for j in range(W):
                if j == self.rank:
                    ptrs.append(own[name].ptr)
                else:
                    m = self.mapping_cls(gathered[j][name])
                    self._keep.append(m)
                    ptrs.append(m.ptr)
            self.local[name] = own[name].tensor()
            strides = torch.empty(shape, dtype=dt, device="meta").stride()
            self.dests[name] = Destinations(ptrs, strides, dt)
        self.o_heads = torch.empty((batch, L, q_heads // W, head_dim), dtype=out_dtype, device=device)
        self._flag = torch.zeros(1, dtype=torch.float32, device=device)

    def _barrier(self) -> None:
        """Stream-ordered: work after it on this stream starts once every rank's
        work before it has completed."""
        if self.world > 1:
            import torch.distributed as dist

            dist.all_reduce(self._flag, group=self.group)

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor],
                 table: torch.Tensor, *, text_len: int, grid_h: int, grid_w: int, mode: str = "dense",
                 gamma_q: Optional[torch.Tensor] = None, gamma_k: Optional[torch.Tensor] = None,
                 rope: Optional[_lib.RopeParams] = None, **opts) -> torch.Tensor:
        """q, k raw (before RMSNorm and RoPE), v, gate: this rank's token shards
        [B, Ls, H, d]. Returns this rank's token shard of the output [B, Ls, Hq, d]
        (a buffer reused by the next call)."""
        if (gate is None) != ("gate" not in self.local):
            raise ValueError("gate given to an instance built without one, or missing")
        r = self.rank
        self._barrier()  # every rank is done reading the buffers of the previous call
        qk_prologue_to_heads(q, table, self.dests["q"], r, gamma_q, rope)
        qk_prologue_to_heads(k, table, self.dests["k"], r, gamma_k, rope)
        seq_to_heads(v, self.dests["v"], r)
        if gate is not None:
            seq_to_heads(gate, self.dests["gate"], r)
        self._barrier()  # this rank's head shards are complete
        _core(self.local["q"], self.local["k"], self.local["v"], self.local.get("gate"), text_len=text_len,
              grid_h=grid_h, grid_w=grid_w, mode=mode, out=self.o_heads, **opts)
        heads_to_seq(self.o_heads, self.dests["out"], r)
        self._barrier()  # this rank's token shard of the output is complete
        return self.local["out"]
