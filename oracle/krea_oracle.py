"""Oracle for the Krea 2 bidirectional attention core -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU restatement of what the attention core computes, written
from the pages' descriptions. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import it; the product path never does. It shares no code,
table or constant with the CUDA library: the two meet only in the seeded inputs
drawn by ``synth.inputs``.

Sources (page title, section):

* [TM]  "Krea 2 TileMix Attention (FP16/INT8 tiles)"
        - "What it actually patches": bidirectional (non-causal) online-softmax
          attention; every score tile goes to FP16 or INT8 by a static map; both
          feed one softmax state; text tiles and a diagonal band of key blocks
          stay FP16; the INT8 share counts only the left-over image-image tiles;
          GQA 48 q heads / 12 KV heads resolved in-kernel (repeat_interleave order).
        - "The inputs that matter": patterns band / one / zero, percentage,
          smooth_k (per-head K mean-centring before quantisation, exact for
          softmax), qk_fp32_accumulate.
* [SL]  "Krea 2 Scanline Attention"
        - "What the mask actually is": text is global both ways; an image token
          sees image tokens within window // 2 rows; text padded to 512 and the
          tail to multiples of 128; padding masked; block mask over 128 tiles;
          tile_aligned admits every valid pair inside an active tile.
* [LS]  "LayerStream: Krea2 Chunking"
        - "What the node does to the block": queries in slices against full K/V,
          with the attention gate; "Be clear about exactness": one slice is exact.

Readings taken where the pages are silent (each is listed in the design notes):

* Softmax scale 1/sqrt(head_dim) unless given.
* Scanline text slot P_t = max(512, ceil128(T)) unless given; a tile is active
  iff it holds at least one valid (query, key) pair the token rule admits.
* TileMix tiles run over the unpadded sequence; a tile holding any text token is
  a text tile; the band is |a - b| <= band_blocks; `band` routes the first
  floor(p * n + 0.5) of a query-tile row's n left-over tiles to INT8, farthest
  from the diagonal first, ties to the smaller key tile.
* INT8 scheme (the pages give none): symmetric, one scale per (batch, head,
  128-token block) = absmax / 127, codes round-half-even clamped to +-127, Q not
  centred, K centred by its per-(batch, kv head, channel) mean over all tokens
  when smooth_k; the centred K is used by the FP16 tiles too.

QK prologue ([TM] "What it actually patches": QK RMSNorm and 3-axis RoPE are the
steps right before the attention core; the pages name them and give no formula).
Readings, each listed in the design notes: RMSNorm y = x * gamma / sqrt(mean(x^2)
+ eps) per (token, head) vector, gamma one weight per channel shared by the
heads, eps 1e-6; then a rotary embedding over three consecutive channel groups
of axes_dim channels (default d/4, 3d/8, 3d/8 = 32, 48, 48 at d = 128), adjacent
channel pairs (2i, 2i+1) of group a turned by pos_a * theta^(-2i / axes_dim[a]),
theta = 10000; positions: text token t at (t, 0, 0), image token at grid (r, c)
at (0, r, c). Parity of this step is pinned by the closed forms and the
rotation identities in the tests.

Parity note: the INT8 quantisation scheme is fixed by the specification, not by
the pages. The INT8 branch of `attention` is pinned by a per-row, per-tile
brute force of that scheme (centring, block scales, round-half-even codes, the
dequantised INT8 scores mixed with FP16 scores in one softmax), the key mean by
a closed form, and both by the pages' invariants (pattern zero equals dense,
smooth_k leaves FP16 results unchanged) and the per-pair INT8 error bound.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

TILE = 128

# Tile kinds in an exported map: bit 0 = some pair in the tile is masked,
# bit 1 = the tile's scores are computed from INT8 codes.
KIND_MASKED = 1
KIND_INT8 = 2

MODES = {"dense": 0, "tilemix": 1, "scanline": 2}


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# ----------------------------------------------------------------------------
# Token layout
# ----------------------------------------------------------------------------

def text_slot(text_len: int, text_pad: int = 0) -> int:
    """[SL] "What the mask actually is": text padded out to 512, or to the next
    multiple of 128 when longer; an explicit slot size overrides."""
    if text_pad:
        return text_pad
    return max(512, ceil_div(text_len, TILE) * TILE)


def logical_layout(text_len: int, grid_h: int, grid_w: int, mode: str, text_pad: int = 0):
    """Map logical slots to physical tokens (-1 = padding slot).

    dense / tilemix: slots are the tokens themselves, the last tile padded.
    scanline ([SL]): text at slots [0, T), padding up to P_t, the image at the
    128-aligned offset P_t, the tail padded to a multiple of 128.
    """
    T = text_len
    N = grid_h * grid_w
    L = T + N
    if mode == "scanline":
        Pt = text_slot(T, text_pad)
        Lp = Pt + ceil_div(N, TILE) * TILE
        phys = np.full(Lp, -1, dtype=np.int64)
        phys[:T] = np.arange(T)
        phys[Pt:Pt + N] = T + np.arange(N)
    else:
        Lp = ceil_div(L, TILE) * TILE
        phys = np.full(Lp, -1, dtype=np.int64)
        phys[:L] = np.arange(L)
    return phys


def scanline_token_rule(tq: np.ndarray, tk: np.ndarray, text_len: int, grid_w: int,
                        window: int) -> np.ndarray:
    """[SL] "What the mask actually is": text tokens see everything and are
    seen by everyone; image tokens see image tokens within window // 2 rows.
    `tq`, `tk` are physical token indices (broadcastable)."""
    q_text = tq < text_len
    k_text = tk < text_len
    rq = (tq - text_len) // grid_w
    rk = (tk - text_len) // grid_w
    return q_text | k_text | (np.abs(rq - rk) <= window // 2)


# ----------------------------------------------------------------------------
# Tile maps
# ----------------------------------------------------------------------------

class TileMap:
    """kind[a, b] for every (query tile a, key tile b); -1 = tile skipped."""

    def __init__(self, kind: np.ndarray):
        self.kind = kind

    @property
    def n_tiles(self) -> int:
        return self.kind.shape[0]

    def csr(self):
        """Row pointers, key tiles and kinds, key tiles ascending in every row."""
        row_ptr = [0]
        cols, kinds = [], []
        for a in range(self.n_tiles):
            for b in range(self.kind.shape[1]):
                if self.kind[a, b] >= 0:
                    cols.append(b)
                    kinds.append(int(self.kind[a, b]))
            row_ptr.append(len(cols))
        return (np.array(row_ptr, dtype=np.int32), np.array(cols, dtype=np.int32),
                np.array(kinds, dtype=np.uint8))


def admitted_matrix_scanline(text_len, grid_h, grid_w, window, tile_aligned, text_pad=0):
    """Boolean [Lp, Lp] over logical slots: is the pair (query slot, key slot)
    admitted?  Brute force over every pair, straight from [SL]."""
    phys = logical_layout(text_len, grid_h, grid_w, "scanline", text_pad)
    Lp = phys.shape[0]
    nt = Lp // TILE
    valid = phys >= 0
    rule = scanline_token_rule(phys[:, None], phys[None, :], text_len, grid_w, window)
    pair_ok = valid[:, None] & valid[None, :] & rule
    active = pair_ok.reshape(nt, TILE, nt, TILE).any(axis=(1, 3))
    if tile_aligned:
        # every valid pair inside an active tile is admitted
        tile_on = np.repeat(np.repeat(active, TILE, axis=0), TILE, axis=1)
        adm = valid[:, None] & valid[None, :] & tile_on
    else:
        adm = pair_ok
    return phys, active, adm


def _kind_from_admission(active: np.ndarray, adm: np.ndarray, valid_q: np.ndarray) -> np.ndarray:
    """A tile is 'masked' unless every valid query row admits all 128 key slots."""
    nt = active.shape[0]
    # padding query rows never count against a tile being full
    adm_rows = adm | ~valid_q[:, None]
    full = adm_rows.reshape(nt, TILE, nt, TILE).all(axis=(1, 3))
    kind = np.where(full, 0, KIND_MASKED).astype(np.int16)
    return np.where(active, kind, -1).astype(np.int16)


def scanline_map(text_len, grid_h, grid_w, window, tile_aligned=True, text_pad=0) -> TileMap:
    """[SL] block mask at 128 tiles: active tiles only, inactive ones skipped.

    Same brute force as `admitted_matrix_scanline`, one query tile at a time so
    that 4 MP grids stay within memory."""
    phys = logical_layout(text_len, grid_h, grid_w, "scanline", text_pad)
    Lp = phys.shape[0]
    nt = Lp // TILE
    valid = phys >= 0
    kind = np.full((nt, nt), -1, dtype=np.int16)
    for a in range(nt):
        pq = phys[a * TILE:(a + 1) * TILE]
        vq = valid[a * TILE:(a + 1) * TILE]
        if not vq.any():
            continue
        rule = scanline_token_rule(pq[:, None], phys[None, :], text_len, grid_w, window)
        pair_ok = vq[:, None] & valid[None, :] & rule                  # [128, Lp]
        active = pair_ok.reshape(TILE, nt, TILE).any(axis=(0, 2))       # [nt]
        if tile_aligned:
            adm = vq[:, None] & valid[None, :] & np.repeat(active, TILE)[None, :]
        else:
            adm = pair_ok
        full = (adm | ~vq[:, None]).reshape(TILE, nt, TILE).all(axis=(0, 2))
        kind[a] = np.where(active, np.where(full, 0, KIND_MASKED), -1)
    return TileMap(kind)


def dense_map(text_len, grid_h, grid_w) -> TileMap:
    """Every tile over the unpadded sequence; the tail tile's padded keys are masked."""
    L = text_len + grid_h * grid_w
    nt = ceil_div(L, TILE)
    kind = np.zeros((nt, nt), dtype=np.int16)
    if L % TILE:
        kind[:, nt - 1] = KIND_MASKED
    return TileMap(kind)


def tilemix_map(text_len, grid_h, grid_w, pattern="band", percentage=0.5,
                band_blocks=2) -> TileMap:
    """[TM] "What it actually patches" / "The inputs that matter".

    FP16 whatever the settings: tiles reading a text key block or writing a text
    query row, and key blocks within `band_blocks` of the query block. The rest
    (image-image, off the band) are the candidates: `zero` keeps them FP16,
    `one` sends them all to INT8, `band` sends a `percentage` share of each
    query-tile row to INT8, farthest from the diagonal first."""
    L = text_len + grid_h * grid_w
    nt = ceil_div(L, TILE)
    kind = np.zeros((nt, nt), dtype=np.int16)
    is_text = np.array([a * TILE < text_len for a in range(nt)])
    for a in range(nt):
        cand = [b for b in range(nt)
                if not (is_text[a] or is_text[b] or abs(a - b) <= band_blocks)]
        if pattern == "zero":
            chosen = []
        elif pattern == "one":
            chosen = cand
        elif pattern == "band":
            cand.sort(key=lambda b: (-abs(a - b), b))
            n8 = int(math.floor(percentage * len(cand) + 0.5))
            chosen = cand[:n8]
        else:
            raise ValueError(pattern)
        for b in chosen:
            kind[a, b] = KIND_INT8
    if L % TILE:
        kind[:, nt - 1] |= KIND_MASKED
    return TileMap(kind)


def tile_map(case_like) -> TileMap:
    c = case_like
    if c.mode == "scanline":
        return scanline_map(c.text_len, c.grid_h, c.grid_w, c.window, c.tile_aligned, c.text_pad)
    if c.mode == "tilemix":
        return tilemix_map(c.text_len, c.grid_h, c.grid_w, c.pattern, c.percentage, c.band_blocks)
    return dense_map(c.text_len, c.grid_h, c.grid_w)


# ----------------------------------------------------------------------------
# smooth_k and the INT8 scheme
# ----------------------------------------------------------------------------

def key_mean(k: np.ndarray) -> np.ndarray:
    """[TM] smooth_k: mean of K over all tokens, per (batch, kv head, channel)."""
    return k.mean(axis=1)                                  # [B, Hkv, d]


def quantize_blocks(x: np.ndarray, precision: str = "f64"):
    """Symmetric INT8 codes with one scale per (batch, head, 128-token block).

    scale = absmax / 127; code = clamp(round_half_even(x / scale), -127, 127);
    a block whose absmax is 0 gets scale 0 and codes 0.

    precision "f64": the definition, in fp64.
    precision "f32": the same steps with every operation rounded to fp32 in the
    order inv = 127 / absmax, code = rne(x * inv) -- the precision in which the
    kernel takes the integer decision, so codes can be compared bit for bit.
    x: [B, L, H, d] (for "f32" already an fp32-representable array).
    Returns codes int8 [B, L, H, d] and scales [B, H, nblocks].
    """
    B, L, H, d = x.shape
    nb = ceil_div(L, TILE)
    codes = np.zeros((B, L, H, d), dtype=np.int8)
    ft = np.float64 if precision == "f64" else np.float32
    scales = np.zeros((B, H, nb), dtype=ft)
    for j in range(nb):
        blk = x[:, j * TILE:(j + 1) * TILE].astype(ft)      # [B, n, H, d]
        amax = np.abs(blk).max(axis=(1, 3))                 # [B, H]
        if precision == "f64":
            s = amax / 127.0
            with np.errstate(divide="ignore", invalid="ignore"):
                r = blk / s[:, None, :, None]
        else:
            s = (amax / np.float32(127.0)).astype(np.float32)
            with np.errstate(divide="ignore", invalid="ignore"):
                inv = (np.float32(127.0) / amax).astype(np.float32)
                r = (blk * inv[:, None, :, None]).astype(np.float32)
        r = np.where((amax > 0)[:, None, :, None], r, 0)
        c = np.clip(np.rint(r), -127, 127).astype(np.int8)  # rint: half to even
        codes[:, j * TILE:(j + 1) * TILE] = c
        scales[:, :, j] = s
    return codes, scales


def centred_keys(k: np.ndarray, precision: str = "f64"):
    """K - mean(K) per (batch, kv head, channel).  In "f32" precision the mean is
    rounded to fp32 once and the subtraction is one fp32 operation."""
    mu = key_mean(k)
    if precision == "f64":
        return k - mu[:, None], mu
    mu32 = mu.astype(np.float32)
    return (k.astype(np.float32) - mu32[:, None]).astype(np.float32), mu32


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------

def _as_f64(t) -> Optional[np.ndarray]:
    if t is None:
        return None
    if hasattr(t, "detach"):
        return t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def attention(case, q, k, v, gate=None, rows: Optional[Sequence[int]] = None,
              batches: Optional[Sequence[int]] = None, heads: Optional[Sequence[int]] = None,
              return_probs: bool = False) -> Dict[str, np.ndarray]:
    """out[b, t, h, :] = sigmoid(gate[b, t, h, :]) * sum_{j in A(t)} softmax_j(scale * s(t, j)) v[b, j, h // rep, :]

    Two-pass softmax (row max, exponentials, sum, divide) over the admitted
    keys A(t) only. Scores s are FP16-tile scores q . k~ (k~ = centred keys
    under TileMix smooth_k) or INT8-tile scores s_q s_k (Q8 . K8), tile by tile
    as the map says. `rows` are physical query tokens (default: all).
    Returns {"out": [B, R, Hq, d], "lse": [B, Hq, R]} (+ "probs" [B, Hq, R, L] if
    asked); lse = log sum_{j in A(t)} exp(scale * s(t, j)), the softmax normaliser.
    """
    c = case
    qd, kd, vd, gd = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(gate)
    B, L, Hq, d = qd.shape
    Hkv = kd.shape[2]
    rep = Hq // Hkv
    scale = c.softmax_scale if c.softmax_scale else 1.0 / math.sqrt(d)
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    batches = range(B) if batches is None else batches
    heads = range(Hq) if heads is None else heads

    tm = tile_map(c)
    mode = c.mode
    # per physical token: its tile (query side and key side use the same layout)
    phys = logical_layout(c.text_len, c.grid_h, c.grid_w, mode, c.text_pad)
    slot_of = np.empty(L, dtype=np.int64)
    slot_of[phys[phys >= 0]] = np.nonzero(phys >= 0)[0]
    tile_of = slot_of // TILE
    kind_tok = tm.kind[tile_of[rows][:, None], tile_of[None, :]]        # [R, L]
    if mode == "scanline":
        if c.tile_aligned:
            adm = kind_tok >= 0
        else:
            adm = (kind_tok >= 0) & scanline_token_rule(rows[:, None], np.arange(L)[None, :],
                                                        c.text_len, c.grid_w, c.window)
    else:
        adm = np.ones((rows.shape[0], L), dtype=bool)
    int8_tile = (kind_tok >= 0) & ((kind_tok & KIND_INT8) != 0)
    any_int8 = bool(int8_tile.any())

    kk = kd
    if mode == "tilemix" and c.smooth_k:
        kk, _ = centred_keys(kd, "f64")
    if any_int8:
        q8, sq = quantize_blocks(qd, "f64")
        k8, sk = quantize_blocks(kk, "f64")

    out = np.zeros((B, rows.shape[0], Hq, d))
    probs = np.zeros((B, Hq, rows.shape[0], L)) if return_probs else None
    lse = np.zeros((B, Hq, rows.shape[0]))
    for b in batches:
        for h in heads:
            g = h // rep                                   # repeat_interleave order
            s = qd[b, rows, h, :] @ kk[b, :, g, :].T        # [R, L]
            if any_int8:
                s8 = (q8[b, rows, h, :].astype(np.float64) @ k8[b, :, g, :].astype(np.float64).T)
                s8 *= sq[b, h, rows // TILE][:, None] * sk[b, g, np.arange(L) // TILE][None, :]
                s = np.where(int8_tile, s8, s)
            s = scale * s
            s = np.where(adm, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            assert np.all(np.isfinite(m)), "a query row admits no key"
            p = np.exp(s - m)
            z = p.sum(axis=1, keepdims=True)
            lse[b, h] = (m + np.log(z))[:, 0]
            p /= z
            o = p @ vd[b, :, g, :]
            if gd is not None:
                o = o * sigmoid(gd[b, rows, h, :])
            out[b, :, h, :] = o
            if return_probs:
                probs[b, h] = p
    res = {"out": out, "lse": lse}
    if return_probs:
        res["probs"] = probs
    return res


def attention_backward(case, q, k, v, gate, dout) -> Dict[str, np.ndarray]:
    """Gradients of out = sigmoid(gate) * softmax(scale * q k^T over A) v with respect
    to q, k, v and gate, given dout [B, L, Hq, d]; FP16-tile scores only (dense and
    scanline: the INT8 codes of TileMix have no gradient).

    With P the softmax weights over the admitted keys and O = P v (before the gate):
      dO = dout * sigmoid(g);  dgate = dout * O * sigmoid(g) (1 - sigmoid(g))
      dV_j = sum_i P_ij dO_i;   dP_ij = dO_i . v_j;   D_i = sum_j P_ij dP_ij = dO_i . O_i
      dS_ij = P_ij (dP_ij - D_i);  dQ_i = scale sum_j dS_ij k_j;  dK_j = scale sum_i dS_ij q_i
    summed over the rep query heads that share a kv head for dK and dV.
    """
    c = case
    assert c.mode != "tilemix" or c.pattern == "zero", "INT8 tiles have no gradient"
    qd, kd, vd, gd, dod = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(gate), _as_f64(dout)
    B, L, Hq, d = qd.shape
    rep = Hq // kd.shape[2]
    scale = c.softmax_scale if c.softmax_scale else 1.0 / math.sqrt(d)
    fwd = attention(c, q, k, v, None, return_probs=True)
    O = fwd["out"]                                   # before the gate
    P = fwd["probs"]                                 # [B, Hq, L, L], zero off the admitted set
    dq, dk, dv = np.zeros_like(qd), np.zeros_like(kd), np.zeros_like(vd)
    sg = sigmoid(gd) if gd is not None else None
    dO = dod * sg if gd is not None else dod
    dgate = dod * O * sg * (1.0 - sg) if gd is not None else None
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            p = P[b, h]
            dv[b, :, g, :] += p.T @ dO[b, :, h, :]
            dp = dO[b, :, h, :] @ vd[b, :, g, :].T
            Dr = np.sum(dO[b, :, h, :] * O[b, :, h, :], axis=1, keepdims=True)
            ds = p * (dp - Dr)
            dq[b, :, h, :] = scale * ds @ kd[b, :, g, :]
            dk[b, :, g, :] += scale * ds.T @ qd[b, :, h, :]
    return {"dq": dq, "dk": dk, "dv": dv, "dgate": dgate}


# ----------------------------------------------------------------------------
# QK prologue: RMSNorm, then the 3-axis rotary embedding
# ----------------------------------------------------------------------------

def default_axes(head_dim: int):
    """Channel groups of the three rotary axes: d/4, 3d/8, 3d/8."""
    return (head_dim // 4, 3 * head_dim // 8, 3 * head_dim // 8)


def rope_positions(text_len: int, grid_h: int, grid_w: int) -> np.ndarray:
    """[L, 3] positions: text token t at (t, 0, 0); image token (r, c) at (0, r, c)."""
    L = text_len + grid_h * grid_w
    pos = np.zeros((L, 3), dtype=np.int64)
    pos[:text_len, 0] = np.arange(text_len)
    for i in range(grid_h * grid_w):
        pos[text_len + i, 1] = i // grid_w
        pos[text_len + i, 2] = i % grid_w
    return pos


def rope_angles(pos: np.ndarray, axes_dim, theta: float = 10000.0) -> np.ndarray:
    """[L, sum(axes_dim) / 2] rotation angles, pair by pair, axis by axis."""
    cols = []
    for a, n in enumerate(axes_dim):
        for i in range(n // 2):
            cols.append(pos[:, a].astype(np.float64) * theta ** (-2.0 * i / n))
    return np.stack(cols, axis=1) if cols else np.zeros((pos.shape[0], 0))


def rms_norm(x: np.ndarray, gamma: Optional[np.ndarray] = None, eps: float = 1e-6) -> np.ndarray:
    """x [..., d] -> x * gamma / sqrt(mean over d of x^2 + eps), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / r
    return y if gamma is None else y * np.asarray(gamma, dtype=np.float64)


def rope_rotate(x: np.ndarray, ang: np.ndarray) -> np.ndarray:
    """x [B, L, H, d]; ang [L, n] turns channel pairs (2j, 2j+1), j < n; the rest pass."""
    x = np.array(x, dtype=np.float64)
    n = ang.shape[1]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    x0 = x[..., 0:2 * n:2].copy()
    x1 = x[..., 1:2 * n:2].copy()
    x[..., 0:2 * n:2] = x0 * c - x1 * s
    x[..., 1:2 * n:2] = x0 * s + x1 * c
    return x


def qk_prologue(x, pos: np.ndarray, gamma: Optional[np.ndarray] = None, axes_dim=None,
                theta: float = 10000.0, eps: float = 1e-6) -> np.ndarray:
    """rope(rms_norm(x)) for x [B, L, H, d] (torch or numpy), in fp64."""
    x = _as_f64(x)
    d = x.shape[-1]
    axes = default_axes(d) if axes_dim is None else tuple(axes_dim)
    return rope_rotate(rms_norm(x, gamma, eps), rope_angles(pos, axes, theta))


def admitted_pairs(case) -> int:
    """Number of (query, key) pairs the attention admits over all valid tokens,
    per (batch, q head): the FLOP count is 4 * B * Hq * d * this."""
    L = case.text_len + case.grid_h * case.grid_w
    if case.mode != "scanline":
        return L * L
    phys = logical_layout(case.text_len, case.grid_h, case.grid_w, "scanline", case.text_pad)
    valid = phys >= 0
    nt = phys.shape[0] // TILE
    kind = tile_map(case).kind
    total = 0
    for a in range(nt):
        pq = phys[a * TILE:(a + 1) * TILE]
        vq = valid[a * TILE:(a + 1) * TILE]
        on = np.repeat(kind[a] >= 0, TILE)
        adm = vq[:, None] & valid[None, :] & on[None, :]
        if not case.tile_aligned:
            adm &= scanline_token_rule(pq[:, None], phys[None, :], case.text_len,
                                       case.grid_w, case.window)
        total += int(adm.sum())
    return total
