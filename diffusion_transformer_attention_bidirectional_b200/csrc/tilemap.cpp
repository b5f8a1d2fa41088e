// Tile-map builder of the Krea 2 attention core: which 128x128 score tiles a
// query tile visits, in which order, and how each is computed.
//
// Built on the host by interval arithmetic over whole tiles (no per-pair
// enumeration): at 4 MP a map has 132^2 = 17424 tile pairs. Maps are cached by
// api.cpp, so the build cost is paid once per geometry, as with the block-mask
// cache of "Krea 2 Scanline Attention", section "Where people get burned".
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "krea_internal.h"

namespace krea {

namespace {

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Per-tile summary of the logical slots it holds.
struct TileInfo {
  bool text = false;       // holds at least one text token
  bool image = false;      // holds at least one image token
  bool all_valid = false;  // all 128 slots are real tokens (no padding)
  int r0 = 0, r1 = -1;     // first / last image row it holds
};

TileInfo tile_info(const Geometry& g, int a) {
  TileInfo t;
  const long s0 = (long)a * kTile, s1 = s0 + kTile;  // slots [s0, s1)
  t.text = s0 < g.T;
  const long i0 = std::max<long>(s0, g.Pt), i1 = std::min<long>(s1, (long)g.Pt + g.N);
  t.image = i0 < i1;
  if (t.image) {
    t.r0 = (int)((i0 - g.Pt) / g.W);
    t.r1 = (int)((i1 - 1 - g.Pt) / g.W);
  }
  // valid slots are [0, T) and [Pt, Pt + N)
  t.all_valid = (s1 <= g.T) || (s0 >= g.Pt && s1 <= (long)g.Pt + g.N);
  return t;
}

// Scanline ("Krea 2 Scanline Attention", section "What the mask actually is"):
// text is global both ways; an image query sees image keys within window/2 rows.
// A tile pair is active when some valid pair inside it is admitted by that rule.
void build_scanline(const Geometry& g, HostMap* m) {
  const int nt = g.n_tiles;
  const int wh = g.window / 2;
  std::vector<TileInfo> info(nt);
  for (int a = 0; a < nt; ++a) info[a] = tile_info(g, a);
  m->row_ptr.assign(1, 0);
  for (int a = 0; a < nt; ++a) {
    const TileInfo& A = info[a];
    for (int b = 0; b < nt; ++b) {
      const TileInfo& Bk = info[b];
      const bool a_valid = A.text || A.image, b_valid = Bk.text || Bk.image;
      if (!a_valid || !b_valid) continue;
      bool active = A.text || Bk.text;
      if (!active && A.image && Bk.image) {
        const int gap = std::max({0, Bk.r0 - A.r1, A.r0 - Bk.r1});  // nearest row distance
        active = gap <= wh;
      }
      if (!active) continue;
      bool full;
      if (g.tile_aligned) {
        full = Bk.all_valid;  // every valid pair of an active tile is admitted
      } else {
        // every valid query of tile a must admit every slot of tile b
        if (!Bk.all_valid) full = false;
        else if (Bk.text || !A.image) full = true;  // text keys, or text-only queries
        else full = std::max(Bk.r1 - A.r0, A.r1 - Bk.r0) <= wh;  // farthest row pair
      }
      m->entries.push_back((b << 2) | (full ? 0 : KREA_KIND_MASKED));
    }
    m->row_ptr.push_back((int32_t)m->entries.size());
  }
}

// TileMix ("Krea 2 TileMix Attention (FP16/INT8 tiles)", sections "What it
// actually patches" and "The inputs that matter"): tiles reading a text key
// block or writing a text query row, and key blocks within band_blocks of the
// diagonal, stay FP16; of the rest, `zero` keeps all FP16, `one` sends all to
// INT8, `band` sends floor(p * n + 0.5) of each row's n left-over tiles to INT8,
// farthest from the diagonal first, the smaller key tile first on ties.
void build_tilemix(const Geometry& g, HostMap* m) {
  const int nt = g.n_tiles;
  const bool ragged = (g.L % kTile) != 0;
  m->row_ptr.assign(1, 0);
  std::vector<int> kinds(nt);
  std::vector<int> cand;
  for (int a = 0; a < nt; ++a) {
    const bool a_text = (long)a * kTile < g.T;
    cand.clear();
    for (int b = 0; b < nt; ++b) {
      kinds[b] = (ragged && b == nt - 1) ? KREA_KIND_MASKED : 0;
      const bool b_text = (long)b * kTile < g.T;
      if (!a_text && !b_text && std::abs(a - b) > g.band_blocks) cand.push_back(b);
    }
    int n8 = 0;
    if (g.pattern == KREA_PATTERN_ONE) n8 = (int)cand.size();
    else if (g.pattern == KREA_PATTERN_BAND)
      n8 = (int)std::floor((double)g.percentage * (double)cand.size() + 0.5);
    // farthest first: distance descending, then key tile ascending
    std::stable_sort(cand.begin(), cand.end(), [a](int x, int y) {
      const int dx = std::abs(a - x), dy = std::abs(a - y);
      return dx != dy ? dx > dy : x < y;
    });
    for (int i = 0; i < n8; ++i) kinds[cand[i]] |= KREA_KIND_INT8;
    for (int b = 0; b < nt; ++b) {
      m->entries.push_back((b << 2) | kinds[b]);
      if (kinds[b] & KREA_KIND_INT8) m->n_int8++;
    }
    m->row_ptr.push_back((int32_t)m->entries.size());
  }
}

void build_dense(const Geometry& g, HostMap* m) {
  const int nt = g.n_tiles;
  const bool ragged = (g.L % kTile) != 0;
  m->row_ptr.assign(1, 0);
  for (int a = 0; a < nt; ++a) {
    for (int b = 0; b < nt; ++b)
      m->entries.push_back((b << 2) | ((ragged && b == nt - 1) ? KREA_KIND_MASKED : 0));
    m->row_ptr.push_back((int32_t)m->entries.size());
  }
}

}  // namespace

int make_geometry(int text_len, int grid_h, int grid_w, int mode, const krea_attn_params_t* p,
                  Geometry* g) {
  if (!p || !g) return KREA_ERR_INVALID_ARG;
  if (text_len < 0 || grid_h < 0 || grid_w < 0) return KREA_ERR_INVALID_ARG;
  if ((grid_h == 0) != (grid_w == 0)) return KREA_ERR_INVALID_ARG;
  const long N = (long)grid_h * grid_w;
  const long L = text_len + N;
  if (L <= 0 || L > (1L << 24)) return KREA_ERR_INVALID_ARG;
  g->T = text_len;
  g->H = grid_h;
  g->W = grid_w > 0 ? grid_w : 1;
  g->N = (int)N;
  g->L = (int)L;
  g->mode = mode;
  if (mode == KREA_MODE_SCANLINE) {
    if (p->window < 1 || p->window > 255 || (p->window % 2) == 0) return KREA_ERR_INVALID_ARG;
    int Pt = p->text_pad;
    if (Pt == 0) Pt = std::max(512, ceil_div(text_len, kTile) * kTile);
    if (Pt % kTile != 0 || Pt < text_len) return KREA_ERR_INVALID_ARG;
    g->Pt = Pt;
    g->n_tiles = (Pt + ceil_div((int)N, kTile) * kTile) / kTile;
    g->window = p->window;
    g->tile_aligned = p->tile_aligned ? 1 : 0;
  } else if (mode == KREA_MODE_DENSE || mode == KREA_MODE_TILEMIX) {
    g->Pt = text_len;
    g->n_tiles = ceil_div((int)L, kTile);
    if (mode == KREA_MODE_TILEMIX) {
      if (p->pattern < KREA_PATTERN_ZERO || p->pattern > KREA_PATTERN_ONE) return KREA_ERR_INVALID_ARG;
      if (!(p->percentage >= 0.0f && p->percentage <= 1.0f)) return KREA_ERR_INVALID_ARG;
      g->pattern = p->pattern;
      g->percentage = p->percentage;
      g->band_blocks = p->band_blocks < 0 ? 2 : p->band_blocks;
    }
  } else {
    return KREA_ERR_INVALID_ARG;
  }
  return KREA_OK;
}

namespace {

// KREA_ATTN_LOG set to anything but "0": one line on stderr per map built, the
// counterpart of the pages' console lines that confirm the path is active.
bool log_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("KREA_ATTN_LOG");
    return e != nullptr && *e != '\0' && std::strcmp(e, "0") != 0;
  }();
  return on;
}

void log_map(const Geometry& g, const HostMap& m) {
  long masked = 0;
  for (int32_t e : m.entries) masked += (e & KREA_KIND_MASKED) ? 1 : 0;
  const long pairs = (long)m.n_tiles * m.n_tiles;
  const long active = (long)m.entries.size();
  char extra[96] = "";
  if (g.mode == KREA_MODE_SCANLINE)
    std::snprintf(extra, sizeof(extra), " text_pad=%d window=%d tile_aligned=%d", g.Pt, g.window, g.tile_aligned);
  else if (g.mode == KREA_MODE_TILEMIX)
    std::snprintf(extra, sizeof(extra), " pattern=%s percentage=%g band=%d",
                  g.pattern == KREA_PATTERN_ZERO ? "zero" : g.pattern == KREA_PATTERN_ONE ? "one" : "band",
                  (double)g.percentage, g.band_blocks);
  const char* name = g.mode == KREA_MODE_SCANLINE ? "scanline" : g.mode == KREA_MODE_TILEMIX ? "tilemix" : "dense";
  std::fprintf(stderr,
               "[krea_attn] map %s T=%d grid=%dx%d%s: %dx%d tiles, %ld active (%.1f%%), %d int8, %ld masked\n",
               name, g.T, g.H, g.W, extra, m.n_tiles, m.n_tiles, active,
               pairs > 0 ? 100.0 * (double)active / (double)pairs : 0.0, m.n_int8, masked);
}

}  // namespace

long tilemix_int8_tiles(const Geometry& g) {
  if (g.mode != KREA_MODE_TILEMIX || g.pattern == KREA_PATTERN_ZERO) return 0;
  const int nt = g.n_tiles, t0 = ceil_div(g.T, kTile);  // tiles holding a text token come first
  long total = 0;
  for (int a = t0; a < nt; ++a) {
    // off-band image key tiles left and right of the diagonal
    const long n = std::max(0, a - g.band_blocks - t0) + std::max(0, nt - 1 - a - g.band_blocks);
    total += g.pattern == KREA_PATTERN_ONE ? n : (long)std::floor((double)g.percentage * (double)n + 0.5);
  }
  return total;
}

int build_map(const Geometry& g, HostMap* out, bool quiet) {
  if (!out) return KREA_ERR_INVALID_ARG;
  out->row_ptr.clear();
  out->entries.clear();
  out->n_int8 = 0;
  out->n_tiles = g.n_tiles;
  if ((long)g.n_tiles * g.n_tiles > (1L << 28)) return KREA_ERR_INVALID_ARG;
  switch (g.mode) {
    case KREA_MODE_SCANLINE: build_scanline(g, out); break;
    case KREA_MODE_TILEMIX: build_tilemix(g, out); break;
    default: build_dense(g, out); break;
  }
  // the closed-form count that callers without a host map rely on must agree
  if (out->n_int8 != tilemix_int8_tiles(g)) return KREA_ERR_INVALID_ARG;
  if (!quiet && log_enabled()) log_map(g, *out);
  return KREA_OK;
}

}  // namespace krea
