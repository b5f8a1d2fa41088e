"""krea_attn_fwd_rope_q: the attention on raw query projections, with the query
half of the QK prologue (RMSNorm, then the 3-axis RoPE: "Krea 2 TileMix Attention
(FP16/INT8 tiles)", section "What it actually patches") applied to each Q tile
in shared memory instead of in a separate pass over HBM.

The fused step repeats the standalone prologue kernel's arithmetic in the same
order, so the fused call must equal qk_prologue followed by attention bit for
bit, on every shape the core takes (ragged tails, text padding, query slices,
d = 64, rotary axes that leave channels unturned). The 1 MP configuration is
also held against the oracle's own chain (fp64 prologue, rounding to the input
dtype, fp64 attention) on sampled rows, at the FP16-tile bounds of the other
parity tests."""
import ctypes

import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from diffusion_transformer_attention_bidirectional_b200 import _lib
from oracle import krea_oracle as ko
from synth import inputs as S

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}
DEV = torch.device("cuda:0")


def mode_opts(c):
    if c.mode == "scanline":
        return {"window": c.window, "tile_aligned": c.tile_aligned, "text_pad": c.text_pad}
    return {}


def both(c, gamma=True, rope=None, **extra):
    """(fused output, chained output, fused lse, chained lse) of one case."""
    q, k, v, g = (None if t is None else t.to(DEV) for t in S.make_inputs(c))
    d = c.head_dim
    rope = rope if rope is not None else K.rope_params(d)
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, DEV), rope=rope, head_dim=d)
    gq = torch.linspace(0.5, 1.5, d, device=DEV) if gamma else None
    gk = torch.linspace(1.25, 0.75, d, device=DEV)
    kn = K.qk_prologue(k, table, gk, rope=rope)
    geo = dict(text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode=c.mode, **mode_opts(c), **extra)
    B, L, Hq, _ = q.shape
    lse_f = torch.full((B, Hq, L), float("nan"), dtype=torch.float32, device=DEV)
    lse_c = torch.full_like(lse_f, float("nan"))
    fused = K.attention_rope_q(q, kn, v, g, table, gq, rope, lse=lse_f, **geo)
    chained = K.attention(K.qk_prologue(q, table, gq, rope=rope), kn, v, g, lse=lse_c, **geo)
    torch.cuda.synchronize()
    return fused, chained, lse_f, lse_c


CASES = [
    S.Case("rq_scan_pad", 1, 8, 2, 128, 300, 60, 60, dtype="bf16", mode="scanline", seed=301, window=11,
           gate=True, prologue=True),
    S.Case("rq_scan_token", 1, 4, 2, 128, 100, 20, 20, dtype="f16", mode="scanline", seed=302, window=5,
           tile_aligned=False, prologue=True),
    S.Case("rq_dense_d64", 2, 4, 2, 64, 77, 9, 13, dtype="f16", mode="dense", seed=303, gate=True, prologue=True),
    S.Case("rq_dense_bf16", 1, 6, 3, 128, 16, 8, 8, dtype="bf16", mode="dense", seed=304, prologue=True),
]


@pytest.mark.parametrize("c", CASES, ids=[c.name for c in CASES])
def test_fused_equals_prologue_then_attention(c):
    fused, chained, lse_f, lse_c = both(c)
    assert torch.equal(fused, chained), float((fused - chained).abs().max())
    assert torch.equal(lse_f.nan_to_num(0.0), lse_c.nan_to_num(0.0))


def test_fused_query_slice_and_no_gamma():
    c = S.Case("rq_slice", 1, 4, 2, 128, 200, 16, 16, dtype="bf16", mode="dense", seed=305, gate=True,
               prologue=True)
    fused, chained, _, _ = both(c, gamma=False, q_start=128, q_len=300)
    rows = slice(128, 428)
    assert torch.equal(fused[:, rows], chained[:, rows])


def test_fused_partial_rotary_axes():
    # axes (16, 24, 24) turn 32 pairs; channels 64 .. 127 only go through RMSNorm
    c = S.Case("rq_axes", 1, 4, 1, 128, 40, 10, 10, dtype="f16", mode="dense", seed=306, prologue=True)
    rope = K.rope_params(128, axes_dim=(16, 24, 24))
    fused, chained, _, _ = both(c, rope=rope)
    assert torch.equal(fused, chained)


@pytest.mark.parametrize("dtype,tol", [("bf16", 2e-3), ("f16", 5e-4)])
def test_fused_1mp_matches_oracle_chain(dtype, tol):
    # the 1 MP configuration (48/12 heads, d = 128, 512 text + 64 x 64, gate) on raw projections
    c = S.dense_1mp()
    c = S.Case(c.name, c.batch, c.q_heads, c.kv_heads, c.head_dim, c.text_len, c.grid_h, c.grid_w, dtype=dtype,
               mode="dense", seed=c.seed, gate=True, prologue=True)
    q, k, v, g = S.make_inputs(c)
    d = c.head_dim
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, DEV))
    gq = torch.linspace(0.5, 1.5, d, device=DEV)
    gk = torch.linspace(1.25, 0.75, d, device=DEV)
    kn = K.qk_prologue(k.to(DEV), table, gk)
    out = K.attention_rope_q(q.to(DEV), kn, v.to(DEV), g.to(DEV), table, gq, text_len=c.text_len,
                             grid_h=c.grid_h, grid_w=c.grid_w)
    torch.cuda.synchronize()
    L = c.seq_len
    rows = [0, 1, 255, 511, 512, 513, 2000, 3071, L // 2 + 77, L - 129, L - 1]
    heads = [0, 5, 23, 47]
    pos = ko.rope_positions(c.text_len, c.grid_h, c.grid_w)
    qo = torch.from_numpy(ko.qk_prologue(q, pos, gamma=gq.cpu().numpy())).to(TDT[dtype])
    ko_ = torch.from_numpy(ko.qk_prologue(k, pos, gamma=gk.cpu().numpy())).to(TDT[dtype])
    want = ko.attention(c, qo, ko_, v, g, rows=rows, heads=heads)["out"][:, :, heads]
    got = out.cpu().numpy()[:, rows][:, :, heads]
    err = float(np.max(np.abs(got - want)))
    print(f"[parity] fused q prologue, 1 MP {dtype}: max |gpu - oracle| = {err:.3e} (tol {tol:.1e})")
    assert err <= tol


def _call(q, table, rope, k, mode, p):
    return _lib.lib().krea_attn_fwd_rope_q(q.data_ptr(), None, table, ctypes.byref(rope), k.data_ptr(),
                                           k.data_ptr(), None, q.data_ptr(), 16, 8, 8, _lib.MODE[mode],
                                           ctypes.byref(p), torch.cuda.current_stream().cuda_stream)


def test_fused_refusals():
    q = torch.zeros(1, 80, 4, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 80, 2, 128, dtype=torch.bfloat16, device=DEV)
    table = K.rope_table(K.rope_positions(16, 8, 8, DEV))
    p = K.make_params(1, 4, 2, 128, 16, 8, 8, in_dtype="bf16", out_dtype="bf16")
    rope = K.rope_params(128)
    assert _call(q, table.data_ptr(), rope, k, "tilemix", p) == _lib.ERR_UNSUPPORTED
    assert _call(q, table.data_ptr() + 4, rope, k, "dense", p) == _lib.ERR_INVALID_ARG
    assert _call(q, None, rope, k, "dense", p) == _lib.ERR_INVALID_ARG
    bad = K.rope_params(128, axes_dim=(30, 48, 48))  # sum 126: not a multiple of 4
    assert _call(q, table.data_ptr(), bad, k, "dense", p) == _lib.ERR_INVALID_ARG
    torch.cuda.synchronize()
