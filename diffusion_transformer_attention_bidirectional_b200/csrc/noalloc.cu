// Allocation-free variant of krea_attn_fwd (declared in include/krea_attn.h).
//
// Some callers cannot allocate device memory while they run: code inside a
// memory-pool or arena that forbids cudaMalloc/cudaFree (both synchronise the
// device and can stall every stream), plugins of a host framework that owns all
// device memory, or a serving loop that must never block on the allocator. For
// them this entry point runs the same kernels as krea_attn_fwd but keeps every
// piece of scratch -- the tile map and, for TileMix, the quantiser workspace
// (centred keys, INT8 codes, scales, key mean, partial sums) -- in one fixed
// array in device memory that the library declares at file scope. Nothing is
// allocated, cached or freed per call; the caller passes only inputs and outputs.
//
// The array costs kScratchBytes of memory on every GPU that loads the library,
// until the process exits. Shapes whose map and workspace do not fit are
// rejected with KREA_ERR_TOO_LARGE before anything is launched.
//
// All calls share the one array and each call overwrites what it needs (the
// map is copied in, the quantiser writes every workspace word it later reads;
// nothing must start at zero). Calls whose work overlaps on the GPU -- on two
// streams, or two threads sharing a device -- race on the array and must not be
// issued; calls on one stream are ordered and safe.
//
// The first call on a device looks the array's device address up with
// cudaGetSymbolAddress (the array's name in host code is only a host-side
// stand-in, not a device address); make that first call before any CUDA graph
// capture on that device.
#include <algorithm>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "krea_internal.h"

namespace {

using namespace krea;

constexpr size_t kScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per device.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KREA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return KREA_ERR_CUDA;
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return KREA_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
int bytes_of(int dt) { return dt == KREA_F32 ? 4 : 2; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool strides_ok(const int64_t s[3], int es) {
  for (int i = 0; i < 3; ++i)
    if (s[i] <= 0 || (s[i] * es) % 16 != 0) return false;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B, L, H, d] with element strides -> 4-D map (d, H, L, B), box (inner, 1, 128, 1), 128-byte swizzle.
bool tmap(CUtensorMap* tm, const void* base, CUtensorMapDataType dt, int es, int d, int H, int L, int B,
          const int64_t s[3], int inner) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t str[3] = {(cuuint64_t)(s[2] * es), (cuuint64_t)(s[1] * es), (cuuint64_t)(s[0] * es)};
  cuuint32_t box[4] = {(cuuint32_t)inner, 1, (cuuint32_t)kTile, 1};
  cuuint32_t one[4] = {1, 1, 1, 1};
  return enc(tm, dt, 4, const_cast<void*>(base), dims, str, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int krea_attn_fwd_noalloc(const void* q, const void* k, const void* v, const void* gate, void* out,
                                     int text_len, int grid_h, int grid_w, int mode,
                                     const krea_attn_params_t* p, void* stream) {
  // ---- the argument checks of krea_attn_fwd
  if (!p || p->abi_version != KREA_ATTN_ABI_VERSION) return KREA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1) return KREA_ERR_INVALID_ARG;
  if (p->batch > 65535 || p->num_q_heads > 65535) return KREA_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return KREA_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return KREA_ERR_UNSUPPORTED;
  if (p->in_dtype == KREA_F32) return KREA_ERR_UNSUPPORTED;
  if (p->in_dtype != KREA_F16 && p->in_dtype != KREA_BF16) return KREA_ERR_INVALID_ARG;
  if (p->out_dtype != KREA_F32 && p->out_dtype != p->in_dtype) return KREA_ERR_INVALID_ARG;
  Geometry g;
  int rc = make_geometry(text_len, grid_h, grid_w, mode, p, &g);
  if (rc != KREA_OK) return rc;
  const int es = bytes_of(p->in_dtype), oes = bytes_of(p->out_dtype);
  if (!q || !k || !v || !out) return KREA_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || (gate && !al16(gate))) return KREA_ERR_INVALID_ARG;
  if (!strides_ok(p->q_stride, es) || !strides_ok(p->k_stride, es) || !strides_ok(p->v_stride, es) ||
      !strides_ok(p->out_stride, oes) || (gate && !strides_ok(p->gate_stride, es)))
    return KREA_ERR_INVALID_ARG;
  if (p->q_start < 0 || p->q_start % kTile != 0 || p->q_start >= g.L || p->q_len < 0) return KREA_ERR_INVALID_ARG;
  const int q_len = p->q_len == 0 ? g.L - p->q_start : p->q_len;
  if ((long)p->q_start + q_len > g.L) return KREA_ERR_INVALID_ARG;
  int dev = -1, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return KREA_ERR_NO_DEVICE;
  }

  // ---- tile map (host) and the scratch layout: map, then the TileMix workspace
  HostMap hm;
  rc = build_map(g, &hm);
  if (rc != KREA_OK) return rc;
  const int d = p->head_dim, B = p->batch, Hq = p->num_q_heads, Hkv = p->num_kv_heads;
  const bool use_int8 = mode == KREA_MODE_TILEMIX && hm.n_int8 > 0;
  const bool centred = mode == KREA_MODE_TILEMIX && p->smooth_k;
  if (use_int8 && d != 128) return KREA_ERR_UNSUPPORTED;
  const size_t off_rows = 0;
  const size_t off_entries = up256(hm.row_ptr.size() * sizeof(int32_t));
  const size_t off_ws = up256(off_entries + hm.entries.size() * sizeof(int32_t));
  WsLayout w;
  size_t need = off_ws;
  if (use_int8 || centred) {
    w = workspace_layout(B, g.L, Hq, Hkv, d, es, p->smooth_k);
    need = off_ws + w.total;
  }
  if (need > kScratchBytes) return KREA_ERR_TOO_LARGE;

  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != KREA_OK) return rc;
  char* sc = static_cast<char*>(scratch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(sc + off_rows, hm.row_ptr.data(), hm.row_ptr.size() * sizeof(int32_t),
                      cudaMemcpyHostToDevice, s) != cudaSuccess ||
      (!hm.entries.empty() && cudaMemcpyAsync(sc + off_entries, hm.entries.data(),
                                              hm.entries.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                                              s) != cudaSuccess))
    return KREA_ERR_CUDA;

  // ---- quantiser into the array (TileMix)
  const bool bf16 = p->in_dtype == KREA_BF16;
  const CUtensorMapDataType tdt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const void* k_src = k;
  int64_t kstr[3] = {p->k_stride[0], p->k_stride[1], p->k_stride[2]};
  const float* sq = nullptr;
  const float* sk = nullptr;
  if (use_int8 || centred) {
    char* ws = sc + off_ws;
    QuantDevParams qp;
    std::memset(&qp, 0, sizeof(qp));
    qp.q = q;
    qp.k = k;
    for (int i = 0; i < 3; ++i) {
      qp.q_stride[i] = p->q_stride[i];
      qp.k_stride[i] = p->k_stride[i];
    }
    qp.kc = p->smooth_k ? ws + w.kc : nullptr;
    qp.q8 = reinterpret_cast<int8_t*>(ws + w.q8);
    qp.k8 = reinterpret_cast<int8_t*>(ws + w.k8);
    qp.sq = reinterpret_cast<float*>(ws + w.sq);
    qp.sk = reinterpret_cast<float*>(ws + w.sk);
    qp.mu = reinterpret_cast<float*>(ws + w.mu);
    qp.part = reinterpret_cast<double*>(ws + w.part);
    qp.B = B;
    qp.L = g.L;
    qp.Hq = Hq;
    qp.Hkv = Hkv;
    qp.d = d;
    qp.nt = (g.L + kTile - 1) / kTile;
    qp.n_chunks = w.n_chunks;
    qp.chunk_tokens = w.chunk_tokens;
    qp.smooth_k = p->smooth_k ? 1 : 0;
    qp.quant_q = use_int8 ? 1 : 0;
    rc = launch_quantize(qp, bf16, stream);
    if (rc != KREA_OK) return rc;
    if (centred) {
      k_src = ws + w.kc;
      const int64_t cs[3] = {(int64_t)g.L * Hkv * d, (int64_t)Hkv * d, d};
      for (int i = 0; i < 3; ++i) kstr[i] = cs[i];
    }
    if (use_int8) {
      const int64_t s8q[3] = {(int64_t)g.L * Hq * d, (int64_t)Hq * d, d};
      const int64_t s8k[3] = {(int64_t)g.L * Hkv * d, (int64_t)Hkv * d, d};
      if (!tmap(&maps.q8, ws + w.q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Hq, g.L, B, s8q, 128) ||
          !tmap(&maps.k8, ws + w.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Hkv, g.L, B, s8k, 128))
        return KREA_ERR_INVALID_ARG;
      sq = reinterpret_cast<const float*>(ws + w.sq);
      sk = reinterpret_cast<const float*>(ws + w.sk);
    }
  }
  if (!tmap(&maps.q, q, tdt, es, d, Hq, g.L, B, p->q_stride, 64) ||
      !tmap(&maps.k, k_src, tdt, es, d, Hkv, g.L, B, kstr, 64) ||
      !tmap(&maps.v, v, tdt, es, d, Hkv, g.L, B, p->v_stride, 64))
    return KREA_ERR_INVALID_ARG;
  bool tma_out = tmap(&maps.out, out, p->out_dtype == KREA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : tdt, oes, d,
                      Hq, g.L, B, p->out_stride, p->out_dtype == KREA_F32 ? 32 : 64);
  if (tma_out && gate) tma_out = tmap(&maps.gate, gate, tdt, es, d, Hq, g.L, B, p->gate_stride, 64);

  // ---- the attention kernel, map and workspace in the array
  AttnDevParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.row_ptr = reinterpret_cast<const int32_t*>(sc + off_rows);
  ap.entries = reinterpret_cast<const int32_t*>(sc + off_entries);
  ap.gate = gate;
  ap.out = out;
  ap.sq = sq;
  ap.sk = sk;
  ap.status = p->status;
  for (int i = 0; i < 3; ++i) {
    ap.gate_stride[i] = p->gate_stride[i];
    ap.out_stride[i] = p->out_stride[i];
  }
  ap.B = B;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.d = d;
  ap.rep = Hq / Hkv;
  ap.nh = (ap.rep % 2 == 0) ? 2 : 1;
  ap.npairs = ap.rep / ap.nh;
  ap.T = g.T;
  ap.N = g.N;
  ap.Pt = g.Pt;
  ap.L = g.L;
  ap.W = g.W;
  ap.H = g.H;
  ap.window_half = g.window / 2;
  ap.tile_aligned = (mode != KREA_MODE_SCANLINE) || g.tile_aligned;
  ap.n_tiles = g.n_tiles;
  ap.q_lo = p->q_start;
  ap.q_hi = p->q_start + q_len;
  auto slot_of = [&](int t) { return t < g.T ? t : t - g.T + g.Pt; };
  ap.tile_begin = slot_of(ap.q_lo) / kTile;
  ap.n_slice_tiles = slot_of(ap.q_hi - 1) / kTile - ap.tile_begin + 1;
  // Scanline: text query rows see every key tile, image rows only the text and their
  // window, so the text tiles' CTAs go first and no long row starts in the last wave.
  {
    const int text_tiles = (g.T + kTile - 1) / kTile;
    ap.n_heavy = mode == KREA_MODE_SCANLINE
                     ? std::max(0, std::min(ap.tile_begin + ap.n_slice_tiles, text_tiles) - ap.tile_begin)
                     : 0;
  }
  ap.nt_scale = (g.L + kTile - 1) / kTile;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt((float)d);
  ap.scale_log2 = scale * 1.4426950408889634f;
  ap.has_gate = gate != nullptr;
  ap.out_f32 = p->out_dtype == KREA_F32;
  ap.tma_out = tma_out ? 1 : 0;
  ap.wait_limit = p->debug_wait_limit > 0 ? p->debug_wait_limit : (long long)2000000000LL;
  ap.debug_flags = p->debug_flags;
  if (p->lse && (reinterpret_cast<uintptr_t>(p->lse) & 3)) return KREA_ERR_INVALID_ARG;
  ap.lse = p->lse;
  return launch_attention(ap, maps, bf16, stream);
}
