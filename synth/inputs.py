"""Seeded synthetic inputs for the Krea 2 attention core.

This module only draws numbers: it holds none of the attention arithmetic (no
scores, no softmax, no maps, no quantisation), so that both the CUDA path and
the oracle can be fed the same tensors without sharing any of the method.

Shapes follow the Krea 2 renders the pages describe:

* 48 query heads sharing 12 KV heads of width 128 (hidden 6144 = 48 x 128), from
  "Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What it actually patches",
  and "LayerStream: Krea2 Chunking", section "Weights stream; activations don't".
* a 1024 x 1024 render becomes a 64 x 64 token grid ("Krea 2 Scanline Attention",
  section "What the mask actually is"); a 4 MP render a 128 x 128 grid (~16k tokens).
* text prefix padded to 512 in training (same page, same section).

Tensors are q, k and v in the layout [batch, tokens, heads, head_dim] (head_dim
contiguous), plus the optional sigmoid-gate logits [batch, tokens, q_heads,
head_dim]. A case with `prologue=True` describes raw q/k projections: the q and
k the attention sees are those after the QK prologue (RMSNorm + 3-axis RoPE),
which is part of the method and is applied by whoever consumes the draws (the
oracle in the tests, the library's prologue kernel on the GPU), never here.

Random numbers come from numpy's PCG64 generator, one independent stream per
(seed, tensor) pair, drawn in float32 and rounded once to the storage dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

# Stream ids: one independent generator per tensor of a case.
_STREAM = {"q": 1, "k": 2, "v": 3, "gate": 4, "koff": 5}

_TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@dataclasses.dataclass
class Case:
    """One attention workload. Sizes only; no arithmetic of the method."""

    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    text_len: int
    grid_h: int
    grid_w: int
    dtype: str = "bf16"            # input dtype: "f16" or "bf16"
    out_dtype: str = "f32"         # output dtype: "f32" or the input dtype
    mode: str = "dense"            # "dense" | "tilemix" | "scanline"
    seed: int = 0
    gate: bool = False
    qk_dist: str = "normal"        # "normal" | "normal_koffset"
    prologue: bool = False         # q/k are raw projections: the QK prologue comes first
    softmax_scale: float = 0.0     # 0 -> 1/sqrt(head_dim)
    # TileMix
    pattern: str = "band"          # "zero" | "band" | "one"
    percentage: float = 0.5
    band_blocks: int = 2
    smooth_k: bool = True
    qk_fp32_accumulate: bool = False
    # scanline
    window: int = 11
    tile_aligned: bool = True
    text_pad: int = 0              # 0 -> max(512, ceil128(text_len))
    # query slicing
    q_len: int = 0                 # 0 -> one slice over all tokens

    @property
    def seq_len(self) -> int:
        return self.text_len + self.grid_h * self.grid_w


def _normal(seed: int, stream: str, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng([seed, _STREAM[stream]])
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def make_inputs(case: Case, with_gate: Optional[bool] = None):
    """Return CPU torch tensors (q, k, v, gate-or-None) in the case's dtype."""
    B, L, Hq, Hkv, d = case.batch, case.seq_len, case.q_heads, case.kv_heads, case.head_dim
    q = _normal(case.seed, "q", (B, L, Hq, d))
    k = _normal(case.seed, "k", (B, L, Hkv, d))
    v = _normal(case.seed, "v", (B, L, Hkv, d))
    if case.qk_dist == "normal_koffset":
        # a shared per-(kv head, channel) offset ~ N(0.5, 0.1) on every key
        off = _normal(case.seed, "koff", (1, 1, Hkv, d), mean=0.5, std=0.1)
        k = k + off
    use_gate = case.gate if with_gate is None else with_gate
    gate = _normal(case.seed, "gate", (B, L, Hq, d)) if use_gate else None
    td = _TORCH_DTYPE[case.dtype]

    def cast(a):
        return None if a is None else torch.from_numpy(a).to(td)

    return cast(q), cast(k), cast(v), cast(gate)


def constant_fill(shape, value: float, dtype: str) -> torch.Tensor:
    return torch.full(shape, value, dtype=_TORCH_DTYPE[dtype])


# --- the five workloads -------------------------------------------------------

def tiny_dense() -> Case:
    """B=1, 4 q heads / 1 KV head, d=64, 16 text + 8x8 image tokens, fp16, scale 1/8."""
    return Case("tiny_dense", 1, 4, 1, 64, 16, 8, 8, dtype="f16", mode="dense", seed=1,
                softmax_scale=1.0 / math.sqrt(64))


def dense_1mp() -> Case:
    """Krea 2 1 MP: 48/12 heads, d=128, 512 text + 64x64 grid, bf16, gate; q/k are raw
    projections that go through the QK prologue (RMSNorm + 3-axis RoPE) first."""
    return Case("dense_1mp", 1, 48, 12, 128, 512, 64, 64, dtype="bf16", mode="dense", seed=2,
                gate=True, prologue=True)


def scanline_1mp() -> Case:
    """Scanline 1 MP: window 11, tile_aligned, text padded to 512, bf16 N(0,1)."""
    return Case("scanline_1mp", 1, 48, 12, 128, 512, 64, 64, dtype="bf16", mode="scanline",
                seed=3, window=11, tile_aligned=True, text_pad=512)


def tilemix_band_4mp() -> Case:
    """TileMix band 4 MP: fp16, K with a shared channel offset, smooth_k, band +-2, p=0.5."""
    return Case("tilemix_band_4mp", 1, 48, 12, 128, 512, 128, 128, dtype="f16", mode="tilemix",
                seed=4, qk_dist="normal_koffset", pattern="band", percentage=0.5,
                band_blocks=2, smooth_k=True)


def cfg_pair_4mp_sliced() -> Case:
    """CFG pair at 4 MP: B=2, bf16, gate, queries in 4096-token slices."""
    return Case("cfg_pair_4mp_sliced", 2, 48, 12, 128, 512, 128, 128, dtype="bf16",
                mode="dense", seed=5, gate=True, q_len=4096, qk_fp32_accumulate=True)


ALL_CASES = {c().name: c for c in (tiny_dense, dense_1mp, scanline_1mp, tilemix_band_4mp,
                                   cfg_pair_4mp_sliced)}
