"""The sequence <-> head exchange on one GPU with every rank emulated: each
rank's destination buffers live on this device and the exchange kernels run
once per emulated rank. They only store and never wait on another rank, so
running the ranks one after the other computes what concurrent ranks would.

The result must equal the unsharded call bit for bit: the QK prologue of a row
does not depend on which rank computes it, every head of the core is
independent, and the TileMix key mean sums fixed 128-token chunks in fp64
whatever the head count. Each case also holds the exchanged result itself
against the oracle's own chain (QK prologue, rounding to the input dtype,
attention) on sampled rows at every shard's edges and middle, at the bounds the
other parity tests use. The decomposition itself is checked against the oracle
on CPU ranks in test_dist.py. Destinations start as NaN, so a row the exchange
failed to write breaks the equality."""
import numpy as np
import pytest
import torch

from oracle import krea_oracle as ko

import diffusion_transformer_attention_bidirectional_b200 as K
from diffusion_transformer_attention_bidirectional_b200 import seqpar
from synth import inputs as S

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def nan_buffers(world, shape, dtype, pad_heads=0):
    """world buffers of `shape`; with pad_heads, each a head-slice view of a wider
    tensor, so the destination strides differ from the contiguous ones."""
    B, L, H, d = shape
    bufs = [torch.full((B, L, H + pad_heads, d), float("nan"), dtype=dtype, device="cuda") for _ in range(world)]
    return [b[:, :, :H] for b in bufs]


def mode_opts(c):
    if c.mode == "scanline":
        return {"window": c.window, "tile_aligned": c.tile_aligned}
    if c.mode == "tilemix":
        return {"pattern": c.pattern, "percentage": c.percentage, "smooth_k": c.smooth_k}
    return {}


def run_case(c, world, pad_heads=0, out_dtype=torch.float32):
    q, k, v, g = (None if t is None else t.cuda() for t in S.make_inputs(c))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    assert L % world == 0
    Ls = L // world
    dt = q.dtype
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, "cuda"), head_dim=d)
    gq = torch.linspace(0.5, 1.5, d, device="cuda")
    gk = torch.linspace(1.25, 0.75, d, device="cuda")

    qh = nan_buffers(world, (B, L, Hq // world, d), dt, pad_heads)
    kh = nan_buffers(world, (B, L, Hkv // world, d), dt, pad_heads)
    vh = nan_buffers(world, (B, L, Hkv // world, d), dt, pad_heads)
    gh = nan_buffers(world, (B, L, Hq // world, d), dt, pad_heads) if g is not None else None
    for r in range(world):
        t0, t1 = seqpar.token_range(Ls, r)
        seqpar.qk_prologue_to_heads(q[:, t0:t1], table, seqpar.Destinations.of(qh), r, gq)
        seqpar.qk_prologue_to_heads(k[:, t0:t1], table, seqpar.Destinations.of(kh), r, gk)
        seqpar.seq_to_heads(v[:, t0:t1], seqpar.Destinations.of(vh), r)
        if g is not None:
            seqpar.seq_to_heads(g[:, t0:t1], seqpar.Destinations.of(gh), r)

    qn = K.qk_prologue(q, table, gq)
    kn = K.qk_prologue(k, table, gk)
    for j in range(world):
        a, b = seqpar.head_range(Hq, world, j)
        ka, kb = seqpar.head_range(Hkv, world, j)
        assert torch.equal(qh[j], qn[:, :, a:b]), j
        assert torch.equal(kh[j], kn[:, :, ka:kb]), j
        assert torch.equal(vh[j], v[:, :, ka:kb]), j
        if g is not None:
            assert torch.equal(gh[j], g[:, :, a:b]), j

    geo = dict(text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode=c.mode, out_dtype=out_dtype)
    oh = [K.attention(qh[j], kh[j], vh[j], None if g is None else gh[j], **geo, **mode_opts(c))
          for j in range(world)]
    out_s = nan_buffers(world, (B, Ls, Hq, d), out_dtype, pad_heads)
    for j in range(world):
        seqpar.heads_to_seq(oh[j], seqpar.Destinations.of(out_s), j)
    out = torch.cat(out_s, dim=1)
    ref = K.attention(qn, kn, v, g, **geo, **mode_opts(c))
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    check_against_oracle(c, out, world, gq, gk)


def check_against_oracle(c, out, world, gq, gk):
    """The exchanged output on sampled rows (the first, middle and last rows of every
    shard) and heads against the oracle's prologue -> attention chain."""
    q, k, v, g = S.make_inputs(c)
    L = c.seq_len
    Ls = L // world
    rows = sorted({t for r in range(world) for t in (r * Ls, r * Ls + 1, r * Ls + Ls // 2, (r + 1) * Ls - 1)})
    Hq = q.shape[2]
    heads = sorted({0, Hq // 2, Hq - 1})
    pos = ko.rope_positions(c.text_len, c.grid_h, c.grid_w)
    td = TDT[c.dtype]
    qo = torch.from_numpy(ko.qk_prologue(q, pos, gamma=gq.cpu().numpy())).to(td)
    ko_ = torch.from_numpy(ko.qk_prologue(k, pos, gamma=gk.cpu().numpy())).to(td)
    want = ko.attention(c, qo, ko_, v, g, rows=rows, heads=heads)["out"][:, :, heads]
    got = out.float().cpu().numpy()[:, rows][:, :, heads]
    if c.mode == "tilemix" and c.pattern != "zero":
        tol = 8e-3
    elif out.dtype == torch.float16:
        tol = 5e-4 + 2.0 ** -11  # fp16 output rounding of unit-scale values
    else:
        tol = 2e-3 if c.dtype == "bf16" else 5e-4
    err = float(np.max(np.abs(got - want)))
    print(f"[parity] exchange {c.name} over {world} ranks: max |gpu - oracle| = {err:.3e} (tol {tol:.1e})")
    assert err <= tol * max(1.0, float(np.max(np.abs(want))))


def test_scanline_1mp_over_four_ranks():
    # 48/12 heads split 12/3 per rank, 1152 tokens per rank
    c = S.Case("sp_scan", 1, 48, 12, 128, 512, 64, 64, dtype="bf16", mode="scanline", seed=201, window=11,
               gate=True, prologue=True)
    run_case(c, 4)


def test_dense_ragged_shards_strided_destinations():
    # 40 tokens per rank (no 128 alignment), d = 64, fp16, bf16-free output dtype
    c = S.Case("sp_dense", 2, 4, 2, 64, 16, 8, 8, dtype="f16", mode="dense", seed=203, gate=True, prologue=True)
    run_case(c, 2, pad_heads=3, out_dtype=torch.float16)


def test_tilemix_band_over_two_ranks():
    c = S.Case("sp_tm", 1, 48, 12, 128, 256, 32, 32, dtype="f16", mode="tilemix", seed=205, pattern="band",
               percentage=0.5, smooth_k=True, qk_dist="normal_koffset", prologue=True)
    run_case(c, 2)


def test_six_ranks_token_rule():
    c = S.Case("sp_tok", 1, 48, 12, 128, 96, 20, 24, dtype="bf16", mode="scanline", seed=207, window=5,
               tile_aligned=False, gate=True, prologue=True)
    run_case(c, 6)


def test_sequence_parallel_attention_one_rank():
    c = S.Case("sp_one", 1, 48, 12, 128, 512, 32, 32, dtype="bf16", mode="scanline", seed=209, window=11,
               gate=True, prologue=True)
    q, k, v, g = (t.cuda() for t in S.make_inputs(c))
    B, L, Hq, d = q.shape
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, "cuda"))
    spa = seqpar.SequenceParallelAttention(B, L, Hq, k.shape[2], d, dtype=torch.bfloat16)
    assert spa.world == 1
    out = spa(q, k, v, g, table, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode="scanline",
              window=11)
    ref = K.attention(K.qk_prologue(q, table), K.qk_prologue(k, table), v, g, text_len=c.text_len,
                      grid_h=c.grid_h, grid_w=c.grid_w, mode="scanline", window=11)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
