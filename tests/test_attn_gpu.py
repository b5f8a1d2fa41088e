"""Parity of the CUDA attention path (through the C ABI) with the fp64 oracle.

Small cases are compared element by element on every output; the full-size
workloads on sampled query tiles (whole 128-row tiles, several heads) that the
oracle computes row by row. Tolerances (max |gpu - oracle| on unit-scale
outputs), the ones the specification states: 8e-3 when INT8 tiles are present;
2e-3 for FP16 tiles; 5e-4 with fp32 QK accumulation (calls that set
qk_fp32_accumulate) and for fp16 inputs. The P operand of the PV product has the
type of V, so with bf16 inputs each softmax weight is rounded to 8 significant
bits (relative error 2^-9); over the thousand-plus keys of a long row those
errors average out well below 2e-3, and rows of at most eight key tiles carry P
to 16 bits (a second bf16 term) so that short rows, where single weights
dominate, stay inside the bound too. Every comparison prints its observed error.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from oracle import krea_oracle as ko
from synth import inputs as S

pytestmark = pytest.mark.gpu

TOL_FP = 5e-4     # fp32 QK accumulation, fp16 inputs
TOL_FP16_TILES = 2e-3
TOL_INT8 = 8e-3


def gpu_run(case, q, k, v, g, **extra):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    gd = g.to(dev) if g is not None else None
    opts = dict(softmax_scale=case.softmax_scale, pattern=case.pattern, percentage=case.percentage,
                band_blocks=case.band_blocks, smooth_k=case.smooth_k, window=case.window,
                tile_aligned=case.tile_aligned, text_pad=case.text_pad)
    opts.update(extra)
    own_status = "status" not in opts
    if own_status:
        opts["status"] = torch.zeros(1, dtype=torch.int32, device=dev)
    if "debug_wait_limit" not in opts:
        opts["debug_wait_limit"] = 400_000_000  # ~0.2 s: a stuck pipeline fails fast
    out = K.attention(qd, kd, vd, gd, text_len=case.text_len, grid_h=case.grid_h, grid_w=case.grid_w,
                      mode=case.mode, **opts)
    torch.cuda.synchronize()
    if own_status:
        assert int(opts["status"].item()) == 0, "device status"
    return out


def compare(case, out_gpu, q, k, v, g, rows=None, heads=None, tol=None):
    if tol is None:
        if case.mode == "tilemix" and case.pattern != "zero":
            tol = TOL_INT8
        elif case.dtype == "bf16" and not case.qk_fp32_accumulate:
            tol = TOL_FP16_TILES
        else:
            tol = TOL_FP
    ref = ko.attention(case, q, k, v, g, rows=rows, heads=heads)["out"]
    got = out_gpu.float().cpu().numpy()
    if rows is not None:
        got = got[:, rows]
    if heads is not None:
        ref = ref[:, :, heads]
        got = got[:, :, heads]
    assert np.all(np.isfinite(got))
    err = np.max(np.abs(got - ref))
    scale = max(1.0, float(np.max(np.abs(ref))))
    print(f"[parity] {case.name} {case.mode} {case.dtype} T={case.text_len} {case.grid_h}x{case.grid_w}: "
          f"max |gpu - oracle| = {err:.3e} (tol {tol * scale:.3e})")
    assert err <= tol * scale, f"max abs err {err:.3e} > {tol * scale:.3e}"
    return err


def tile_rows(L, tiles):
    rows = []
    for t in tiles:
        rows.extend(range(t * 128, min(L, t * 128 + 128)))
    return np.array(sorted(set(rows)))


# ---------------------------------------------------------------------------- small cases, every output

def test_tiny_dense_full():
    c = S.tiny_dense()
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    compare(c, out, q, k, v, g)


@pytest.mark.parametrize("T,H,W,d,Hq,Hkv,dtype,gate", [
    (16, 8, 8, 64, 4, 1, "bf16", True),
    (0, 9, 9, 128, 2, 2, "f16", False),        # L = 81, rep 1
    (1, 1, 128, 128, 6, 2, "bf16", True),      # L = 129, rep 3
    (100, 13, 12, 128, 8, 2, "f16", True),     # L = 256
    (300, 30, 30, 64, 4, 2, "bf16", False),    # L = 1200, ragged
    (77, 31, 33, 128, 4, 1, "f16", True),      # L = 1100
])
def test_dense_shapes(T, H, W, d, Hq, Hkv, dtype, gate):
    c = S.Case("shape", 1, Hq, Hkv, d, T, H, W, dtype=dtype, mode="dense", seed=T + H + d, gate=gate)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    compare(c, out, q, k, v, g)


def test_batch_and_out_dtype():
    c = S.Case("b2", 2, 4, 2, 128, 200, 20, 20, dtype="bf16", mode="dense", seed=9, gate=True)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g, out_dtype=torch.bfloat16)
    assert out.dtype == torch.bfloat16
    compare(c, out, q, k, v, g, tol=4e-3)  # 2e-3 FP16-tile bound + 2^-9 rounding of the bf16 output


def test_strided_inputs():
    # q, k, v as views of one packed [B, L, Hq + 2 Hkv, d] projection output
    c = S.Case("strided", 1, 8, 2, 128, 128, 16, 16, dtype="bf16", mode="dense", seed=21)
    q, k, v, _ = S.make_inputs(c)
    packed = torch.cat([q, k, v], dim=2).cuda()
    qv, kv, vv = packed[:, :, :8], packed[:, :, 8:10], packed[:, :, 10:12]
    out = K.attention(qv, kv, vv, None, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w)
    torch.cuda.synchronize()
    compare(c, out, q, k, v, None)


@pytest.mark.parametrize("T,H,W,window,ta,pad", [
    (16, 8, 8, 3, True, 0),
    (16, 8, 8, 3, False, 0),
    (300, 20, 24, 5, True, 0),
    (300, 20, 24, 5, False, 0),
    (130, 16, 40, 1, False, 256),
    (0, 12, 50, 3, True, 0),
])
def test_scanline_small(T, H, W, window, ta, pad):
    c = S.Case("scan", 1, 4, 2, 128, T, H, W, dtype="bf16", mode="scanline", seed=5 + T, window=window,
               tile_aligned=ta, text_pad=pad, gate=True)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    compare(c, out, q, k, v, g)


@pytest.mark.parametrize("pattern,pct", [("zero", 0.5), ("band", 0.5), ("one", 0.5), ("band", 0.75)])
def test_tilemix_small(pattern, pct):
    c = S.Case("tm", 1, 4, 2, 128, 200, 30, 30, dtype="f16", mode="tilemix", seed=17,
               qk_dist="normal_koffset", pattern=pattern, percentage=pct, band_blocks=1, smooth_k=True)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    compare(c, out, q, k, v, g)


def test_tilemix_smooth_k_off():
    c = S.Case("tm", 1, 4, 2, 128, 64, 24, 24, dtype="bf16", mode="tilemix", seed=18,
               qk_dist="normal_koffset", pattern="one", smooth_k=False, band_blocks=1)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    compare(c, out, q, k, v, g)


# ---------------------------------------------------------------------------- quantiser

def test_quantizer_matches_oracle_fp32_decisions():
    c = S.Case("q", 2, 8, 2, 128, 150, 17, 19, dtype="f16", mode="tilemix", seed=3, qk_dist="normal_koffset")
    q, k, _, _ = S.make_inputs(c)
    res = K.quantize(q.cuda(), k.cuda(), text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, smooth_k=True)
    torch.cuda.synchronize()
    kd = k.double().numpy()
    kc32, mu32 = ko.centred_keys(kd, "f32")
    k8, sk = ko.quantize_blocks(kc32, "f32")
    q8, sq = ko.quantize_blocks(q.float().numpy(), "f32")
    assert np.array_equal(res["mu"].cpu().numpy(), mu32)
    assert np.array_equal(res["sk"].cpu().numpy(), sk)
    assert np.array_equal(res["sq"].cpu().numpy(), sq)
    assert np.array_equal(res["k8"].cpu().numpy(), k8)
    assert np.array_equal(res["q8"].cpu().numpy(), q8)
    kc_ref = torch.from_numpy(kc32).to(torch.float16).numpy()
    assert np.array_equal(res["kc"].cpu().numpy(), kc_ref)


# ---------------------------------------------------------------------------- full-size workloads, sampled

def test_config_dense_1mp():
    c = S.dense_1mp()
    q, k, v, g = S.make_inputs(c)
    # raw projections through the oracle's QK prologue (RMSNorm + 3-axis RoPE), rounded to bf16
    pos = ko.rope_positions(c.text_len, c.grid_h, c.grid_w)
    q = torch.from_numpy(ko.qk_prologue(q, pos)).to(torch.bfloat16)
    k = torch.from_numpy(ko.qk_prologue(k, pos)).to(torch.bfloat16)
    out = gpu_run(c, q, k, v, g)
    rows = tile_rows(c.seq_len, [0, 3, 4, 17, 35])
    # thousands of keys per row: the bf16 rounding of P averages out below 5e-4
    compare(c, out, q, k, v, g, rows=rows, heads=[0, 1, 2, 3, 22, 47], tol=TOL_FP)


@pytest.mark.parametrize("T,H,W", [(512, 64, 64), (300, 64, 64), (300, 60, 60)])
def test_config_scanline_1mp(T, H, W):
    c = S.scanline_1mp()
    c.text_len, c.grid_h, c.grid_w = T, H, W
    c.text_pad = 512
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    L = c.seq_len
    rows = np.unique(np.r_[np.arange(0, 8), np.arange(T - 4, T + 130), np.arange(2000, 2140), np.arange(L - 200, L)])
    compare(c, out, q, k, v, g, rows=rows, heads=[0, 5, 47])


def test_config_scanline_1mp_token_rule():
    # tile_aligned off: each image query admits exactly the keys within five rows
    # (64-token rows, two per tile, so boundary tiles become masked tiles)
    c = S.scanline_1mp()
    c.tile_aligned = False
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    L = c.seq_len
    rows = np.unique(np.r_[np.arange(0, 4), np.arange(508, 700), np.arange(2500, 2600), np.arange(L - 130, L)])
    compare(c, out, q, k, v, g, rows=rows, heads=[0, 7, 47])


def test_config_tilemix_band_4mp():
    c = S.tilemix_band_4mp()
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g)
    rows = tile_rows(c.seq_len, [0, 4, 60, 131])
    compare(c, out, q, k, v, g, rows=rows, heads=[0, 1, 46])


def test_config_cfg_pair_4mp_sliced_bit_identical():
    c = S.cfg_pair_4mp_sliced()
    q, k, v, g = S.make_inputs(c)
    dev = torch.device("cuda:0")
    qd, kd, vd, gd = q.to(dev), k.to(dev), v.to(dev), g.to(dev)
    L = c.seq_len
    full = K.attention(qd, kd, vd, gd, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w)
    sliced = torch.full_like(full, float("nan"))
    for s in range(0, L, c.q_len):
        K.attention(qd, kd, vd, gd, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, out=sliced,
                    q_start=s, q_len=min(c.q_len, L - s))
    torch.cuda.synchronize()
    assert torch.equal(full, sliced)
    rows = tile_rows(L, [0, 33, 131])
    compare(c, full, q, k, v, g, rows=rows, heads=[0, 13, 47], tol=TOL_FP)  # fp32-accumulate bound


def test_slices_write_only_their_rows():
    c = S.Case("sl", 1, 4, 2, 128, 100, 20, 20, dtype="bf16", mode="scanline", seed=4, window=5)
    q, k, v, g = S.make_inputs(c)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    full = K.attention(qd, kd, vd, None, text_len=100, grid_h=20, grid_w=20, mode="scanline", window=5)
    part = torch.full_like(full, 7.0)
    K.attention(qd, kd, vd, None, text_len=100, grid_h=20, grid_w=20, mode="scanline", window=5, out=part,
                q_start=128, q_len=200)
    torch.cuda.synchronize()
    assert torch.equal(part[:, 128:328], full[:, 128:328])
    assert torch.all(part[:, :128] == 7.0) and torch.all(part[:, 328:] == 7.0)


# ---------------------------------------------------------------------------- failure detection

def test_bounded_wait_reports_timeout_and_context_survives():
    c = S.Case("t", 1, 4, 2, 128, 64, 16, 16, dtype="bf16", mode="dense", seed=2)
    q, k, v, g = S.make_inputs(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    gpu_run(c, q, k, v, g, status=status, debug_flags=1, debug_wait_limit=2_000_000)
    assert int(status.item()) == -5
    status.zero_()
    out = gpu_run(c, q, k, v, g, status=status)
    assert int(status.item()) == 0
    compare(c, out, q, k, v, g)


def test_errors_are_reported_not_hidden():
    q = torch.zeros(1, 80, 4, 64, dtype=torch.float32, device="cuda:0")
    with pytest.raises(K.KreaError) as e:
        K.attention(q, q[:, :, :1], q[:, :, :1], text_len=16, grid_h=8, grid_w=8)
    assert e.value.code == -2  # fp32 inputs are unsupported
    qh = q.half()
    with pytest.raises(K.KreaError) as e:
        K.attention(qh, qh[:, :, :1], qh[:, :, :1], text_len=16, grid_h=8, grid_w=8, q_start=64)
    assert e.value.code == -1  # slice start not a multiple of 128


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_polynomial_exp2_path(dtype):
    # every exponential through the FMA-pipe polynomial (normally one in four):
    # its error (1.2e-4 relative for bf16, 2.9e-6 for fp16) stays inside the tolerance
    c = S.Case("poly", 1, 4, 2, 128, 100, 20, 20, dtype=dtype, mode="scanline", seed=31, window=3,
               tile_aligned=False, gate=True)
    q, k, v, g = S.make_inputs(c)
    out = gpu_run(c, q, k, v, g, debug_flags=2)
    compare(c, out, q, k, v, g)
    base = gpu_run(c, q, k, v, g)
    assert float((out - base).abs().max()) < 4e-3


def test_head_shards_equal_full_call():
    # the multi-GPU split: each rank's call on views of its kv heads (here run one
    # after the other on one GPU) fills exactly the rows of the full call
    from diffusion_transformer_attention_bidirectional_b200 import shard

    c = S.Case("shards", 1, 48, 12, 128, 256, 24, 24, dtype="bf16", mode="scanline", seed=51, window=7,
               gate=True)
    q, k, v, g = (t.cuda() for t in S.make_inputs(c))
    full = K.attention(q, k, v, g, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode="scanline",
                       window=7)
    out = torch.full_like(full, float("nan"))
    for rank in range(3):
        qs, ks, vs, gs, os_ = shard.shard_views(q, k, v, g, out, rank, 3)
        K.attention(qs, ks, vs, gs, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, mode="scanline",
                    window=7, out=os_)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


# ---------------------------------------------------------------------------- closed forms on the GPU path

def test_single_admitted_key_returns_its_value():
    # scanline, no text, one token per image row, window 1, token rule: every query
    # admits exactly itself, so out = sigmoid(gate) * v (and v without a gate)
    c = S.Case("one_key", 1, 4, 2, 128, 0, 300, 1, dtype="bf16", mode="scanline", seed=91, window=1,
               tile_aligned=False)
    q, k, v, _ = S.make_inputs(c)
    out = gpu_run(c, q, k, v, None).cpu().numpy()
    want = np.repeat(v.float().numpy(), 2, axis=2)  # q head h reads kv head h // 2
    assert np.max(np.abs(out - want)) <= 1e-6 * max(1.0, float(np.max(np.abs(want))))
    g = torch.from_numpy(np.random.default_rng(5).standard_normal(q.shape).astype(np.float32)).to(torch.bfloat16)
    out_g = gpu_run(c, q, k, v, g).cpu().numpy()
    sig = 1.0 / (1.0 + np.exp(-g.double().numpy()))
    assert np.max(np.abs(out_g - sig * want)) <= 1e-5


@pytest.mark.parametrize("mode,ta", [("dense", True), ("scanline", False), ("scanline", True)])
def test_zero_queries_give_the_mean_of_admitted_values(mode, ta):
    # q = 0: every admitted score is 0, every weight 1/|A(q)|; the admitted sets are
    # written out here from the rule (text global, image rows within window // 2)
    T, H, W, win = 130, 12, 20, 5
    c = S.Case("qzero", 1, 2, 1, 128, T, H, W, dtype="bf16", mode=mode, seed=93, window=win, tile_aligned=ta)
    _, k, v, _ = S.make_inputs(c)
    q = torch.zeros(1, c.seq_len, 2, 128, dtype=torch.bfloat16)
    out = gpu_run(c, q, k, v, None).cpu().numpy()[0, :, 0]
    vv = v.double().numpy()[0, :, 0]
    L = c.seq_len
    for t in [0, 1, T - 1, T, T + 7, T + W * 5 + 3, L - 1]:
        if mode == "dense" or t < T:
            idx = np.arange(L)
        else:
            r = (t - T) // W
            if ta:  # tile-aligned: every valid key of every active 128-tile pair
                idx = None
            else:
                rows = range(max(0, r - win // 2), min(H, r + win // 2 + 1))
                idx = np.r_[np.arange(T), [T + rr * W + cc for rr in rows for cc in range(W)]].astype(int)
        if idx is None:
            continue  # covered by the oracle comparisons; the rule above is per token
        assert np.max(np.abs(out[t] - vv[idx].mean(axis=0))) <= 2e-6, t


@pytest.mark.parametrize("mode", ["dense", "scanline", "tilemix"])
def test_lse_matches_oracle(mode):
    # the softmax normaliser ln sum_j exp(scale s_ij) per valid query row, written
    # when asked for (the quantity a backward pass recomputes P from)
    extra = dict(window=5, tile_aligned=False) if mode == "scanline" else {}
    if mode == "tilemix":
        extra = dict(pattern="band", percentage=0.5, band_blocks=1, smooth_k=True, qk_dist="normal_koffset")
    c = S.Case("lse", 1, 4, 2, 128, 150, 14, 22, dtype="f16", mode=mode, seed=97, gate=True, **extra)
    q, k, v, g = S.make_inputs(c)
    lse = torch.full((1, 4, c.seq_len), float("nan"), dtype=torch.float32, device="cuda")
    out = gpu_run(c, q, k, v, g, lse=lse)
    ref = ko.attention(c, q, k, v, g)
    tol = 1e-3 if mode == "tilemix" else 1e-4
    assert np.max(np.abs(lse.cpu().numpy() - ref["lse"])) <= tol
    # a slice writes only its own rows
    lse2 = torch.full_like(lse, float("nan"))
    gpu_run(c, q, k, v, g, lse=lse2, q_start=128, q_len=200)
    got = lse2.cpu().numpy()
    assert np.all(np.isnan(got[..., :128])) and np.all(np.isnan(got[..., 328:]))
    assert np.max(np.abs(got[..., 128:328] - ref["lse"][..., 128:328])) <= tol
