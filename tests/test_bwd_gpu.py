"""The backward kernels (prep + tcgen05 dq/dk/dv) against the oracle's fp64
gradients. The GPU rounds P, dS and dO to the input dtype for the tensor-core
products (relative error eps = 2^-9 bf16, 2^-11 fp16 per operand); every
gradient entry is a sum of such products, so |gpu - exact| stays within a few
eps of the largest entry: the bound used is 8 eps * max|exact| (fp32 accumulate)."""
import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from oracle import krea_oracle as ko
from synth import inputs as S

pytestmark = pytest.mark.gpu

EPS = {"bf16": 2.0 ** -9, "f16": 2.0 ** -11}


def run_case(c, with_gate):
    q, k, v, g = S.make_inputs(c, with_gate=with_gate)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    gd = g.to(dev) if g is not None else None
    opts = dict(window=c.window, tile_aligned=c.tile_aligned, text_pad=c.text_pad)
    lse = torch.empty(c.batch, c.q_heads, c.seq_len, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = K.attention(qd, kd, vd, gd, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode=c.mode,
                      lse=lse, status=status, debug_wait_limit=400_000_000, **opts)
    w = torch.from_numpy(np.random.default_rng(c.seed).standard_normal(out.shape).astype(np.float32))
    dq, dk, dv, dgate = K.attention_backward(qd, kd, vd, gd, out, w.to(dev), lse, text_len=c.text_len,
                                             grid_h=c.grid_h, grid_w=c.grid_w, mode=c.mode, status=status,
                                             debug_wait_limit=400_000_000, **opts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = ko.attention_backward(c, q, k, v, g, w)
    got = {"dq": dq, "dk": dk, "dv": dv, "dgate": dgate}
    for name in ("dq", "dk", "dv") + (("dgate",) if with_gate else ()):
        r = ref[name]
        x = got[name].cpu().numpy()
        err = float(np.max(np.abs(x - r)))
        bound = 8 * EPS[c.dtype] * float(np.max(np.abs(r)))
        assert err <= bound, f"{c.name} {name}: {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("dtype,d,Hq,Hkv,gate", [("bf16", 128, 4, 1, True), ("f16", 128, 4, 2, False),
                                                 ("bf16", 64, 2, 1, False), ("f16", 64, 4, 1, True)])
def test_backward_dense(dtype, d, Hq, Hkv, gate):
    c = S.Case("bwd_dense", 1, Hq, Hkv, d, 70, 9, 15, dtype=dtype, mode="dense", seed=101 + d)  # L = 205, ragged
    run_case(c, gate)


@pytest.mark.parametrize("ta", [True, False])
def test_backward_scanline(ta):
    c = S.Case("bwd_scan", 2, 4, 1, 128, 100, 12, 20, dtype="bf16", mode="scanline", seed=111, window=3,
               tile_aligned=ta)
    run_case(c, True)


def test_backward_full_size_one_group():
    # the dense 1 MP workload (48/12 heads) through the backward; kv-head groups are
    # independent, so group 5 must equal the oracle run on that group alone
    c = S.dense_1mp()
    q, k, v, g = S.make_inputs(c)
    dev = torch.device("cuda:0")
    lse = torch.empty(1, 48, c.seq_len, dtype=torch.float32, device=dev)
    qd, kd, vd, gd = q.to(dev), k.to(dev), v.to(dev), g.to(dev)
    out = K.attention(qd, kd, vd, gd, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, lse=lse)
    w = torch.from_numpy(np.random.default_rng(3).standard_normal(out.shape).astype(np.float32))
    dq, dk, dv, dgate = K.attention_backward(qd, kd, vd, gd, out, w.to(dev), lse, text_len=c.text_len,
                                             grid_h=c.grid_h, grid_w=c.grid_w)
    torch.cuda.synchronize()
    grp = 5
    hs = slice(4 * grp, 4 * grp + 4)
    sub = S.Case("grp", 1, 4, 1, 128, c.text_len, c.grid_h, c.grid_w, dtype="bf16", mode="dense", seed=0)
    ref = ko.attention_backward(sub, q[:, :, hs], k[:, :, grp:grp + 1], v[:, :, grp:grp + 1], g[:, :, hs],
                                w[:, :, hs])
    for name, x in (("dq", dq[:, :, hs]), ("dk", dk[:, :, grp:grp + 1]), ("dv", dv[:, :, grp:grp + 1]),
                    ("dgate", dgate[:, :, hs])):
        r = ref[name]
        err = float(np.max(np.abs(x.cpu().numpy() - r)))
        assert err <= 8 * EPS["bf16"] * float(np.max(np.abs(r))), (name, err)
