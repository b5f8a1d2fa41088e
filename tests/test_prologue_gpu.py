"""The QK prologue kernel (RMSNorm + 3-axis RoPE in one pass, optional INT8
codes) against the oracle's fp64 restatement, and the prologue followed by the
attention core against the oracle's chain."""
import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from oracle import krea_oracle as ko
from synth import inputs as S

pytestmark = pytest.mark.gpu

FRAC = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}  # half an ulp, relative
TDT = {"bf16": torch.bfloat16, "f16": torch.float16}


def raw(case):
    q, k, _, _ = S.make_inputs(case)
    return q, k


def round_to(x64, dtype):
    return torch.from_numpy(x64).to(TDT[dtype]).float().numpy()


def test_rope_table_matches_oracle():
    pos = K.rope_positions(300, 20, 24)
    tab = K.rope_table(pos.cuda()).cpu().numpy()
    ang = ko.rope_angles(ko.rope_positions(300, 20, 24), ko.default_axes(128))
    assert tab.shape == (300 + 480, 64, 2)
    assert np.max(np.abs(tab[..., 0] - np.cos(ang))) <= 6e-8
    assert np.max(np.abs(tab[..., 1] - np.sin(ang))) <= 6e-8


@pytest.mark.parametrize("dtype,d,use_gamma", [("bf16", 128, True), ("f16", 128, False), ("bf16", 64, False),
                                               ("f16", 64, True)])
def test_prologue_matches_oracle(dtype, d, use_gamma):
    c = S.Case("pro", 2, 6, 2, d, 77, 9, 13, dtype=dtype, mode="dense", seed=61 + d, prologue=True)
    q, _ = raw(c)
    pos = ko.rope_positions(c.text_len, c.grid_h, c.grid_w)
    gamma = np.random.default_rng(7).uniform(0.5, 1.5, d).astype(np.float32) if use_gamma else None
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, "cuda"), head_dim=d)
    y = K.qk_prologue(q.cuda(), table, torch.from_numpy(gamma).cuda() if use_gamma else None)
    torch.cuda.synchronize()
    got = y.float().cpu().numpy()
    ref64 = ko.qk_prologue(q, pos, gamma)
    ref = round_to(ref64, dtype)
    # fp32 arithmetic rounded once to the dtype: within one ulp of the fp64 value rounded,
    # and equal to it except where the fp64 value sits next to a rounding boundary
    assert np.all(np.abs(got - ref) <= 2 * FRAC[dtype] * np.abs(ref64) + 1e-7)
    assert np.mean(got == ref) >= 0.99


def test_prologue_in_place_strided_and_codes():
    c = S.Case("pro2", 1, 8, 2, 128, 130, 10, 20, dtype="f16", mode="dense", seed=71, prologue=True)
    q, k = raw(c)
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, "cuda"))
    # q and k as views of one packed projection output, transformed in place
    packed = torch.cat([q, k], dim=2).cuda()
    qv, kv = packed[:, :, :8], packed[:, :, 8:]
    want_q = K.qk_prologue(qv.contiguous(), table)
    want_k = K.qk_prologue(kv.contiguous(), table)
    K.qk_prologue(qv, table, out=qv)
    K.qk_prologue(kv, table, out=kv)
    torch.cuda.synchronize()
    assert torch.equal(packed[:, :, :8], want_q) and torch.equal(packed[:, :, 8:], want_k)
    # the fused INT8 codes are the quantiser's decisions on the stored values
    y, codes, scales = K.qk_prologue(q.cuda(), table, with_codes=True)
    torch.cuda.synchronize()
    q8, sq = ko.quantize_blocks(y.float().cpu().numpy(), "f32")
    assert np.array_equal(codes.cpu().numpy(), q8)
    assert np.array_equal(scales.cpu().numpy(), sq)


def test_prologue_then_attention_matches_oracle_chain():
    c = S.Case("chain", 1, 8, 2, 128, 100, 16, 16, dtype="bf16", mode="scanline", seed=81, window=5, gate=True,
               prologue=True)
    q, k, v, g = S.make_inputs(c)
    dev = torch.device("cuda:0")
    table = K.rope_table(K.rope_positions(c.text_len, c.grid_h, c.grid_w, dev))
    qp = K.qk_prologue(q.to(dev), table)
    kp = K.qk_prologue(k.to(dev), table)
    out = K.attention(qp, kp, v.to(dev), g.to(dev), text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w,
                      mode="scanline", window=5)
    torch.cuda.synchronize()
    pos = ko.rope_positions(c.text_len, c.grid_h, c.grid_w)
    qo = torch.from_numpy(ko.qk_prologue(q, pos)).to(torch.bfloat16)
    ko_ = torch.from_numpy(ko.qk_prologue(k, pos)).to(torch.bfloat16)
    ref = ko.attention(c, qo, ko_, v, g)["out"]
    err = float(np.max(np.abs(out.cpu().numpy() - ref)))
    print(f"[parity] prologue -> scanline attention chain: max |gpu - oracle| = {err:.3e} (tol 2e-3)")
    # the FP16-tile bound; q and k may differ from the oracle's rounded values by one ulp
    assert err <= 2e-3, err
