"""Pins for the oracle: each test checks it against something other than its
own code -- brute force on tiny inputs, a library routine (torch SDPA in fp64),
closed forms, the pages' invariants and the numbers the pages print."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import krea_oracle as ko
from synth.inputs import Case, make_inputs, tiny_dense

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(t):
    return t.double().numpy()


def small_case(mode="dense", **kw):
    base = dict(name="s", batch=1, q_heads=8, kv_heads=2, head_dim=64, text_len=40, grid_h=12, grid_w=12,
                dtype="f16", mode=mode, seed=11)
    base.update(kw)
    return Case(**base)


def token_rule_mask(T, H, W, window):
    """Admission by the scanline token rule, written from the page: text tokens see
    everything and are seen by everyone; an image token sees image tokens whose grid
    row is at most window // 2 away."""
    L = T + H * W
    m = np.zeros((L, L), dtype=bool)
    row = [None] * T + [i // W for i in range(H * W)]
    for a in range(L):
        for b in range(L):
            if a < T or b < T:
                m[a, b] = True
            else:
                m[a, b] = abs(row[a] - row[b]) <= window // 2
    return m


# --------------------------------------------------------------------------- brute force

def brute_force(q, k, v, gate, scale, allowed):
    """Per (head, row) loops over keys with math.exp, K/V expanded by repeat_interleave."""
    B, L, Hq, d = q.shape
    rep = Hq // k.shape[2]
    ke = np.repeat(k, rep, axis=2)  # repeat_interleave order: head h -> kv head h // rep
    ve = np.repeat(v, rep, axis=2)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            for t in range(L):
                keys = [j for j in range(L) if allowed[t, j]]
                s = [scale * float(np.dot(q[b, t, h], ke[b, j, h])) for j in keys]
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                z = sum(w)
                o = sum(wi / z * ve[b, j, h] for wi, j in zip(w, keys))
                if gate is not None:
                    o = o / (1.0 + np.exp(-gate[b, t, h]))
                out[b, t, h] = o
    return out


def test_brute_force_tiny_dense():
    c = tiny_dense()
    q, k, v, _ = make_inputs(c)
    ref = ko.attention(c, q, k, v)["out"]
    L = c.seq_len
    bf = brute_force(f64(q), f64(k), f64(v), None, 1 / 8, np.ones((L, L), bool))
    assert np.max(np.abs(ref - bf)) < 1e-12


def test_brute_force_scanline_token_rule_with_gate():
    c = small_case("scanline", text_len=20, grid_h=6, grid_w=7, window=3, tile_aligned=False,
                   q_heads=4, kv_heads=2, gate=True)
    q, k, v, g = make_inputs(c)
    ref = ko.attention(c, q, k, v, g)["out"]
    allowed = token_rule_mask(c.text_len, c.grid_h, c.grid_w, c.window)
    bf = brute_force(f64(q), f64(k), f64(v), f64(g), 1 / math.sqrt(64), allowed)
    assert np.max(np.abs(ref - bf)) < 1e-12


# --------------------------------------------------------------------------- library routine

def sdpa_ref(q, k, v, mask, scale):
    """torch.nn.functional.scaled_dot_product_attention in fp64 with expanded K/V."""
    rep = q.shape[2] // k.shape[2]
    qt = q.double().permute(0, 2, 1, 3)
    kt = k.double().repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    vt = v.double().repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask),
                                                          scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def test_dense_equals_sdpa():
    c = small_case("dense", batch=2)
    q, k, v, _ = make_inputs(c)
    ref = ko.attention(c, q, k, v)["out"]
    L = c.seq_len
    lib = sdpa_ref(q, k, v, np.ones((L, L), bool), 1 / 8)
    assert np.max(np.abs(ref - lib)) < 1e-10


def test_scanline_token_rule_equals_masked_sdpa():
    c = small_case("scanline", window=5, tile_aligned=False, grid_h=14, grid_w=11, text_len=77)
    q, k, v, _ = make_inputs(c)
    ref = ko.attention(c, q, k, v)["out"]
    lib = sdpa_ref(q, k, v, token_rule_mask(c.text_len, c.grid_h, c.grid_w, c.window), 1 / 8)
    assert np.max(np.abs(ref - lib)) < 1e-10


def test_scanline_tile_aligned_equals_sdpa_on_active_tiles():
    # tile_aligned: a pair is admitted iff both tokens are real and their logical
    # 128-slot tiles form an active tile pair (one holding a pair the rule admits)
    T, H, W, win = 200, 24, 20, 3
    c = small_case("scanline", window=win, tile_aligned=True, grid_h=H, grid_w=W, text_len=T)
    q, k, v, _ = make_inputs(c)
    ref = ko.attention(c, q, k, v)["out"]
    rule = token_rule_mask(T, H, W, win)
    Pt = 512
    slot = np.array([t if t < T else Pt + t - T for t in range(T + H * W)])
    tile = slot // 128
    nt = tile.max() + 1
    active = np.zeros((nt, nt), bool)
    for a in range(T + H * W):
        for b in np.nonzero(rule[a])[0]:
            active[tile[a], tile[b]] = True
    mask = active[tile[:, None], tile[None, :]]
    lib = sdpa_ref(q, k, v, mask, 1 / 8)
    assert np.max(np.abs(ref - lib)) < 1e-10


# --------------------------------------------------------------------------- closed forms

def _q_zero_case(**kw):
    c = small_case(**kw)
    q, k, v, _ = make_inputs(c)
    L = c.seq_len
    q = torch.zeros_like(q)
    vv = torch.zeros_like(v)
    vv[..., 0] = 1.0
    vv[..., 1] = torch.arange(L, dtype=torch.float64).to(v.dtype)[None, :, None]  # exact up to 2048 in f16
    return c, q, k, vv


def test_q_zero_gives_mean_of_admitted_values_dense():
    c, q, k, v = _q_zero_case(mode="dense")
    out = ko.attention(c, q, k, v)["out"]
    L = c.seq_len
    assert np.allclose(out[..., 0], 1.0, atol=1e-13)
    assert np.allclose(out[..., 1], (L - 1) / 2, atol=1e-10)


def test_q_zero_scanline_window_closed_form():
    T, H, W, win = 30, 9, 10, 3
    c, q, k, v = _q_zero_case(mode="scanline", text_len=T, grid_h=H, grid_w=W, window=win,
                              tile_aligned=False)
    out = ko.attention(c, q, k, v)["out"][0, :, 0, 1]
    L = T + H * W
    for t in range(L):
        if t < T:
            expect = (L - 1) / 2
        else:
            r = (t - T) // W
            rows = range(max(0, r - win // 2), min(H, r + win // 2 + 1))
            idx = list(range(T)) + [T + rr * W + cc for rr in rows for cc in range(W)]
            expect = sum(idx) / len(idx)
        assert abs(out[t] - expect) < 1e-9, t


def test_constant_values_and_gate():
    c = small_case("dense", gate=True)
    q, k, v, g = make_inputs(c)
    v = torch.full_like(v, 0.75)
    out = ko.attention(c, q, k, v, g)["out"]
    sig = 1 / (1 + np.exp(-f64(g)))
    assert np.max(np.abs(out - 0.75 * sig)) < 1e-12
    g0 = torch.zeros_like(g)
    out0 = ko.attention(c, q, k, v, g0)["out"]
    assert np.max(np.abs(out0 - 0.375)) < 1e-12


def test_dominant_key():
    c = small_case("dense", text_len=8, grid_h=4, grid_w=4, q_heads=2, kv_heads=1)
    q, k, v, _ = make_inputs(c)
    qd = f64(q)
    j = 13
    qd[0, 5, 0] = 40.0 * f64(k)[0, j, 0]
    out = ko.attention(c, torch.from_numpy(qd), k, v)["out"]
    assert np.max(np.abs(out[0, 5, 0] - f64(v)[0, j, 0])) < 1e-6


def test_gqa_equals_explicit_expansion():
    c = small_case("dense", q_heads=8, kv_heads=2)
    q, k, v, _ = make_inputs(c)
    out = ko.attention(c, q, k, v)["out"]
    ce = small_case("dense", q_heads=8, kv_heads=8)
    out_e = ko.attention(ce, q, k.repeat_interleave(4, dim=2), v.repeat_interleave(4, dim=2))["out"]
    assert np.max(np.abs(out - out_e)) < 1e-13


def test_probabilities_rows_sum_to_one_masked_zero():
    c = small_case("scanline", window=3, tile_aligned=False, text_len=20, grid_h=6, grid_w=9)
    q, k, v, _ = make_inputs(c)
    P = ko.attention(c, q, k, v, return_probs=True)["probs"]
    assert np.allclose(P.sum(-1), 1.0, atol=1e-13)
    allowed = token_rule_mask(c.text_len, c.grid_h, c.grid_w, c.window)
    assert np.all(P[:, :, ~allowed] == 0.0)
    assert np.all(P[:, :, allowed] > 0.0)


# --------------------------------------------------------------------------- invariants

def test_wide_window_equals_dense():
    T, H, W = 50, 7, 13
    for ta in (True, False):
        c = small_case("scanline", text_len=T, grid_h=H, grid_w=W, window=2 * H - 1, tile_aligned=ta)
        q, k, v, _ = make_inputs(c)
        out = ko.attention(c, q, k, v)["out"]
        cd = small_case("dense", text_len=T, grid_h=H, grid_w=W)
        outd = ko.attention(cd, q, k, v)["out"]
        assert np.max(np.abs(out - outd)) < 1e-12


def test_smooth_k_is_exact_for_fp16_tiles():
    c = small_case("tilemix", pattern="zero", smooth_k=True, qk_dist="normal_koffset")
    q, k, v, _ = make_inputs(c)
    on = ko.attention(c, q, k, v)["out"]
    c.smooth_k = False
    off = ko.attention(c, q, k, v)["out"]
    assert np.max(np.abs(on - off)) < 1e-12


def test_pattern_zero_equals_dense():
    c = small_case("tilemix", pattern="zero")
    q, k, v, _ = make_inputs(c)
    a = ko.attention(c, q, k, v)["out"]
    b = ko.attention(small_case("dense"), q, k, v)["out"]
    assert np.max(np.abs(a - b)) < 1e-12


def test_tilemix_map_rules():
    T, H, W, band = 300, 40, 40, 2
    zero = ko.tilemix_map(T, H, W, "zero", 0.5, band).kind
    one = ko.tilemix_map(T, H, W, "one", 0.5, band).kind
    assert np.array_equal(ko.tilemix_map(T, H, W, "band", 0.0, band).kind, zero)
    assert np.array_equal(ko.tilemix_map(T, H, W, "band", 1.0, band).kind, one)
    nt = zero.shape[0]
    text = [a * 128 < T for a in range(nt)]
    for p in (0.25, 0.5, 0.75):
        kind = ko.tilemix_map(T, H, W, "band", p, band).kind
        for a in range(nt):
            n_left = sum(1 for b in range(nt) if not text[a] and not text[b] and abs(a - b) > band)
            assert (kind[a] & ko.KIND_INT8 > 0).sum() == math.floor(p * n_left + 0.5)
            for b in range(nt):
                if text[a] or text[b] or abs(a - b) <= band:
                    assert not kind[a, b] & ko.KIND_INT8
        # farthest tiles go first: within a row, every INT8 tile is at least as
        # far from the diagonal as every FP16 left-over tile
        for a in range(nt):
            d8 = [abs(a - b) for b in range(nt) if kind[a, b] & ko.KIND_INT8]
            d16 = [abs(a - b) for b in range(nt)
                   if not text[a] and not text[b] and abs(a - b) > band and not kind[a, b] & ko.KIND_INT8]
            if d8 and d16:
                assert min(d8) >= max(d16)


def test_int8_score_error_bound():
    c = small_case("tilemix", pattern="one", qk_dist="normal_koffset", head_dim=64, text_len=0,
                   grid_h=16, grid_w=16, q_heads=2, kv_heads=1)
    q, k, _, _ = make_inputs(c)
    qd, kd = f64(q), f64(k)
    kc, _ = ko.centred_keys(kd)
    q8, sq = ko.quantize_blocks(qd)
    k8, sk = ko.quantize_blocks(kc)
    L = c.seq_len
    blk = np.arange(L) // 128
    for h in range(2):
        Sq = sq[0, h, blk][:, None]
        Sk = sk[0, 0, blk][None, :]
        s8 = (q8[0, :, h].astype(np.float64) @ k8[0, :, 0].astype(np.float64).T) * Sq * Sk
        exact = qd[0, :, h] @ kc[0, :, 0].T
        bound = (np.abs(qd[0, :, h]).sum(1)[:, None] * Sk / 2 + np.abs(kc[0, :, 0]).sum(1)[None, :] * Sq / 2
                 + 64 * Sq * Sk / 4)
        assert np.all(np.abs(s8 - exact) <= bound + 1e-12)
    # dequantisation error is at most half a step
    step = sq[0][:, blk].T[:, :, None]                       # [L, Hq, 1]
    assert np.all(np.abs(q8[0].astype(np.float64) * step - qd[0]) <= step / 2 + 1e-15)


def test_quantize_golden_example():
    g = json.load(open(os.path.join(GOLDEN, "quant_example.json")))
    x = np.zeros(g["shape"])
    rows = np.array(g["block0_first_rows"])
    x[0, :3, 0, :] = rows
    for prec in ("f64", "f32"):
        codes, scales = ko.quantize_blocks(x.astype(np.float32) if prec == "f32" else x, prec)
        assert np.array_equal(codes[0, :3, 0, :], np.array(g["block0_codes"]))
        assert np.all(codes[0, 3:] == 0)
        assert float(scales[0, 0, 0]) == g["block0_scale"]
        assert float(scales[0, 0, 1]) == g["block1_scale"]


# --------------------------------------------------------------------------- the pages' numbers

def test_pages_grid_and_window():
    f = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    side = f["image_px"] // 8 // 2           # VAE latent /8, then halved by the wrapper
    assert f["image_px"] // 8 == f["latent_side_at_1024"]
    assert side == f["token_grid_side_at_1024"]
    assert f["window_default"] // 2 == f["rows_each_side_at_window_11"]
    assert f["q_heads"] * 128 == f["hidden"]
    assert abs(128 * 128 + 512 - f["tokens_at_4mp_approx"]) < 1000
    # an image token in the middle of the 64x64 grid sees exactly rows r-5 .. r+5
    T, H, W = 16, side, side
    c, q, k, v = _q_zero_case(mode="scanline", text_len=T, grid_h=H, grid_w=W, window=f["window_default"],
                              tile_aligned=False, q_heads=1, kv_heads=1, head_dim=64)
    rows_q = np.array([T + 32 * W + 7])
    P = ko.attention(c, q, k, v, rows=rows_q, return_probs=True)["probs"][0, 0, 0]
    seen_rows = sorted({(j - T) // W for j in np.nonzero(P)[0] if j >= T})
    assert seen_rows == list(range(32 - 5, 32 + 5 + 1))
    assert np.all(P[:T] > 0)


def test_scanline_padding_layout():
    f = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    phys = ko.logical_layout(300, 64, 64, "scanline")
    assert ko.text_slot(300) == f["text_pad"]
    assert phys.shape[0] % 128 == 0
    assert np.all(phys[:300] == np.arange(300)) and np.all(phys[300:512] == -1)
    assert phys[512] == 300 and phys[512 + 4095] == 300 + 4095


def _window_rows(H, half):
    """Rows within `half` of each of H rows, counted row by row."""
    return [min(H - 1, r + half) - max(0, r - half) + 1 for r in range(H)]


def test_admitted_pair_counts_closed_form():
    # Scanline at 1 MP ("Krea 2 Scanline Attention", What the mask actually is: a
    # 64x64 latent grid, window 11 = five rows up and five down, text global both
    # ways). Counted here from the rule itself, independently of the oracle's maps:
    #   text queries see all L keys, image queries see the T text keys, and
    #   token rule: an image query sees the W tokens of each row within 5 rows;
    #   tile-aligned: with W = 64 a 128-token tile holds two rows, so image tiles a, b
    #   are active iff the nearest rows are <= 5 apart (|a - b| <= 3), and every pair
    #   of an active tile is admitted.
    T, H, W = 512, 64, 64
    L, N = T + H * W, H * W
    text = T * L + N * T
    token = text + sum(_window_rows(H, 5)) * W * W
    tiles = H * W // 128
    active = sum(min(tiles - 1, a + 3) - max(0, a - 3) + 1 for a in range(tiles))
    aligned = text + active * 128 * 128
    assert (token, aligned) == (7217152, 7929856)
    base = dict(window=11, text_pad=512)
    assert ko.admitted_pairs(Case("s", 1, 1, 1, 128, T, H, W, mode="scanline", tile_aligned=False, **base)) == token
    assert ko.admitted_pairs(Case("s", 1, 1, 1, 128, T, H, W, mode="scanline", tile_aligned=True, **base)) == aligned
    # dense: every pair of real tokens
    assert ko.admitted_pairs(Case("d", 1, 1, 1, 128, T, H, W, mode="dense")) == L * L


# ---------------------------------------------------------------------------- QK prologue pins

def test_rms_norm_closed_forms():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 5, 3, 128)) * 3.0
    y = ko.rms_norm(x, eps=0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, atol=1e-13)     # unit RMS per vector
    assert np.allclose(ko.rms_norm(7.5 * x, eps=0.0), y, atol=1e-13)  # scale invariance
    g = rng.standard_normal(128)
    assert np.allclose(ko.rms_norm(x, g, eps=0.0), y * g, atol=1e-13)  # one weight per channel
    # eps enters under the root: mean(y^2) = m / (m + eps), m = mean(x^2)
    m = np.mean(x * x, axis=-1)
    ye = ko.rms_norm(x, eps=0.5)
    assert np.allclose(np.mean(ye * ye, axis=-1), m / (m + 0.5), atol=1e-13)


def test_rope_positions_layout():
    pos = ko.rope_positions(2, 2, 3)
    assert pos.tolist() == [[0, 0, 0], [1, 0, 0], [0, 0, 0], [0, 0, 1], [0, 0, 2], [0, 1, 0], [0, 1, 1], [0, 1, 2]]
    assert ko.default_axes(128) == (32, 48, 48) and ko.default_axes(64) == (16, 24, 24)


def test_rope_worked_example_and_frequencies():
    # d = 4, axes (2, 2, 0): pair 0 turns by p0 * theta^0, pair 1 by p1 * theta^0
    x = np.array([1.0, 0.0, 1.0, 0.0]).reshape(1, 1, 1, 4)
    pos = np.array([[1, 2, 0]])
    y = ko.rope_rotate(x, ko.rope_angles(pos, (2, 2, 0)))[0, 0, 0]
    assert np.allclose(y, [math.cos(1), math.sin(1), math.cos(2), math.sin(2)], atol=1e-15)
    # pair i of an axis of n channels turns at theta^(-2i/n) radians per position step
    ang = ko.rope_angles(np.array([[0, 1, 0]]), (32, 48, 48))[0]
    assert np.all(ang[:16] == 0) and np.all(ang[40:] == 0)
    assert np.allclose(ang[16:40], [10000.0 ** (-2.0 * i / 48) for i in range(24)], rtol=1e-15)


def test_rope_rotation_identities():
    rng = np.random.default_rng(5)
    L, d = 6, 128
    axes = ko.default_axes(d)
    q = rng.standard_normal((1, L, 1, d))
    k = rng.standard_normal((1, L, 1, d))
    p1 = rng.integers(0, 50, size=(L, 3))
    p2 = rng.integers(0, 50, size=(L, 3))
    r = lambda x, p: ko.rope_rotate(x, ko.rope_angles(p, axes))
    assert np.allclose(r(q, np.zeros((L, 3), dtype=np.int64)), q, atol=0)           # position 0: identity
    pair = lambda x: x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    assert np.allclose(pair(r(q, p1)), pair(q), atol=1e-12)                          # a rotation per pair
    assert np.allclose(r(r(q, p1), p2), r(q, p1 + p2), atol=1e-11)                   # angles add
    # relative position: <R(a) q, R(b) k> = <R(a - b) q, k>
    lhs = np.sum(r(q, p1) * r(k, p2), axis=-1)
    rhs = np.sum(r(q, p1 - p2) * k, axis=-1)
    assert np.allclose(lhs, rhs, atol=1e-11)


def test_qk_prologue_is_norm_then_rope():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((1, 12, 2, 64))
    pos = ko.rope_positions(4, 2, 4)
    g = rng.uniform(0.5, 1.5, 64)
    y = ko.qk_prologue(x, pos, g)
    # rotation keeps each pair's length, so the RMS of y is that of the normalised x
    assert np.allclose(np.mean(y * y, -1), np.mean(ko.rms_norm(x, g) ** 2, -1), atol=1e-12)
    assert np.allclose(y[:, 0], ko.rms_norm(x, g)[:, 0], atol=0)  # token 0 sits at (0, 0, 0)


# ---------------------------------------------------------------------------- backward pins

def _loss(c, q, k, v, g, w):
    return float(np.sum(ko.attention(c, q, k, v, g)["out"] * w))


@pytest.mark.parametrize("mode,extra", [("dense", {}), ("scanline", dict(window=3, tile_aligned=False)),
                                        ("scanline", dict(window=3, tile_aligned=True))])
def test_backward_matches_central_differences(mode, extra):
    # d/dx of sum(out * w) by central differences on a tiny case, every input entry
    # of a few sampled coordinates: pins every term of the backward formulas
    c = Case("bw", 1, 2, 1, 8, 3, 3, 4, mode=mode, seed=12, softmax_scale=0.7, **extra)
    rng = np.random.default_rng(4)
    L = c.seq_len
    q, k, v = (rng.standard_normal((1, L, h, 8)) for h in (2, 1, 1))
    g = rng.standard_normal((1, L, 2, 8))
    w = rng.standard_normal((1, L, 2, 8))
    grads = ko.attention_backward(c, q, k, v, g, w)
    eps = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v), ("dgate", g)):
        idx = [tuple(rng.integers(0, n) for n in x.shape) for _ in range(12)]
        for ix in idx:
            xp, xm = x.copy(), x.copy()
            xp[ix] += eps
            xm[ix] -= eps
            args = {"dq": (xp, k, v, g), "dk": (q, xp, v, g), "dv": (q, k, xp, g), "dgate": (q, k, v, xp)}[name]
            argm = {"dq": (xm, k, v, g), "dk": (q, xm, v, g), "dv": (q, k, xm, g), "dgate": (q, k, v, xm)}[name]
            num = (_loss(c, *args, w) - _loss(c, *argm, w)) / (2 * eps)
            assert abs(num - grads[name][ix]) <= 1e-6 * max(1.0, abs(num)), (name, ix, num, grads[name][ix])


def test_backward_closed_forms():
    # dV_j = sum_i P_ij dO_i: with q = 0 (dense) every weight is 1 / L, so every row of
    # dV is the sum of dO over all queries and both heads of the group, divided by L
    c = Case("bw2", 1, 2, 1, 8, 0, 4, 5, mode="dense", seed=13)
    rng = np.random.default_rng(6)
    L = c.seq_len
    q = np.zeros((1, L, 2, 8))
    k, v = rng.standard_normal((1, L, 1, 8)), rng.standard_normal((1, L, 1, 8))
    w = rng.standard_normal((1, L, 2, 8))
    gr = ko.attention_backward(c, q, k, v, None, w)
    want_dv = (w[0, :, 0, :].sum(0) + w[0, :, 1, :].sum(0)) / L
    assert np.allclose(gr["dv"][0, :, 0, :], want_dv[None, :], atol=1e-12)
    # a row's weights do not change when every key moves by the same vector (each
    # score of the row shifts by one constant): sum_j dS_ij = 0, so sum_j dK_j = 0
    assert np.allclose(gr["dk"].sum(axis=1), 0.0, atol=1e-12)


# --------------------------------------------------------------------------- INT8 tiles and the key mean

def _brute_int8_attention(q, k, v, T, band_blocks, int8_tile, smooth_k, scale):
    """TileMix attention written out per query row and key tile, straight from the
    definitions ("Krea 2 TileMix Attention (FP16/INT8 tiles)", sections "What it
    actually patches" and "The inputs that matter", with the symmetric
    per-(batch, head, 128-token block) absmax/127 scheme the specification fixes):

      mu[b, g, c] = (1 / L) sum_t k[b, t, g, c]        (smooth_k; 0 otherwise)
      kc = k - mu                                      (used by FP16 and INT8 tiles)
      S(block) = max |x| over the block's tokens and channels / 127
      X8 = round_half_even(x / S) clamped to [-127, 127]   (0 when S = 0)
      s(t, j) = S_q(t) S_k(j) sum_c Q8[t, c] K8[j, c]   on an INT8 tile
              = sum_c q[t, c] kc[j, c]                 on an FP16 tile
      out[t] = sum_j softmax_j(scale s(t, j)) v[j]      (every key admitted)

    Each piece is computed here on its own, with loops over tokens, blocks and
    tiles; int8_tile(a, b) says whether tile (query tile a, key tile b) is INT8."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    rep = Hq // Hkv
    mu = np.zeros((B, Hkv, d))
    if smooth_k:
        for b in range(B):
            for g in range(Hkv):
                acc = np.zeros(d)
                for t in range(L):
                    acc += k[b, t, g]
                mu[b, g] = acc / L
    kc = k - mu[:, None]

    def codes_and_scales(x):
        _, _, H, _ = x.shape
        nb = (L + 127) // 128
        c8 = np.zeros(x.shape)
        sc = np.zeros((B, H, nb))
        for b in range(B):
            for h in range(H):
                for j in range(nb):
                    blk = x[b, 128 * j:128 * j + 128, h]
                    amax = max(abs(float(e)) for e in blk.ravel())
                    s = amax / 127.0
                    sc[b, h, j] = s
                    if s > 0:
                        for r in range(blk.shape[0]):
                            for c in range(d):
                                c8[b, 128 * j + r, h, c] = min(127, max(-127, round(float(blk[r, c]) / s)))
        return c8, sc

    q8, sq = codes_and_scales(q)
    k8, sk = codes_and_scales(kc)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            for t in range(L):
                a = t // 128
                s = np.empty(L)
                for kb in range(0, L, 128):
                    j = np.arange(kb, min(L, kb + 128))
                    if int8_tile(a, kb // 128):
                        s[j] = sq[b, h, a] * sk[b, g, kb // 128] * (k8[b, j, g] @ q8[b, t, h])
                    else:
                        s[j] = kc[b, j, g] @ q[b, t, h]
                s = scale * s
                w = np.exp(s - s.max())
                out[b, t, h] = (w / w.sum()) @ v[b, :, g]
    return out


@pytest.mark.parametrize("pattern,smooth_k", [("one", True), ("one", False), ("band", True)])
def test_int8_tiles_brute_force(pattern, smooth_k):
    # 20 text tokens + 24 x 24 image tokens = 596 tokens: 5 tiles, the last one a
    # ragged tail (84 tokens) that is both INT8 and masked in the exported map.
    # K carries a per-channel offset, so the centring moves the INT8 codes.
    c = Case("i8", 1, 2, 1, 16, 20, 24, 24, dtype="f16", mode="tilemix", seed=41, qk_dist="normal_koffset",
             pattern=pattern, percentage=0.5, band_blocks=0, smooth_k=smooth_k)
    q, k, v, _ = make_inputs(c)
    qd, kd, vd = f64(q), f64(k), f64(v)
    kind = ko.tile_map(c).kind
    assert kind[1, 4] == ko.KIND_INT8 | ko.KIND_MASKED  # the ragged tail tile is both
    if pattern == "one":
        # written from the page: text tiles and the band (here the diagonal) stay FP16,
        # every other image-image tile goes to INT8
        def int8_tile(a, b):
            return a != 0 and b != 0 and a != b
    else:
        def int8_tile(a, b):
            return bool(kind[a, b] & ko.KIND_INT8)
    n8 = sum(int8_tile(a, b) for a in range(5) for b in range(5))
    assert n8 == (12 if pattern == "one" else 8)
    want = _brute_int8_attention(qd, kd, vd, c.text_len, c.band_blocks, int8_tile, smooth_k, 1 / math.sqrt(16))
    got = ko.attention(c, q, k, v)["out"]
    assert np.max(np.abs(got - want)) <= 1e-12
    # and the INT8 tiles really change the result: with every tile FP16 the rows
    # whose tiles hold INT8 scores differ by the quantisation error
    zero = ko.attention(Case(**{**c.__dict__, "pattern": "zero"}), q, k, v)["out"]
    assert np.max(np.abs(zero[:, 128:] - want[:, 128:])) > 1e-4
    assert np.max(np.abs(zero[:, :128] - want[:, :128])) <= 1e-12  # text query tile: all FP16


def test_key_mean_closed_form():
    # keys c + (-1)^t x over an even number of tokens: the +x and -x rows cancel, so
    # the mean over tokens is exactly c and the centred keys are (-1)^t x
    rng = np.random.default_rng(3)
    B, L, Hkv, d = 2, 10, 3, 8
    cvec = rng.standard_normal((B, Hkv, d))
    x = rng.standard_normal((B, 1, Hkv, d))
    sign = np.array([(-1.0) ** t for t in range(L)])[None, :, None, None]
    k = cvec[:, None] + sign * x
    assert np.max(np.abs(ko.key_mean(k) - cvec)) <= 1e-15
    kc, mu = ko.centred_keys(k, "f64")
    assert np.max(np.abs(mu - cvec)) <= 1e-15
    assert np.max(np.abs(kc - sign * x)) <= 1e-15
    # a constant key sequence has itself as mean and centres to zero
    kconst = np.broadcast_to(cvec[:, None], (B, 7, Hkv, d))
    assert np.max(np.abs(ko.centred_keys(kconst, "f64")[0])) <= 1e-15
