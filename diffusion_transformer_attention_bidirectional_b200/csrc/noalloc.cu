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
// allocated, cached or freed per call, and nothing is copied from the host: the
// tile map is built into the array by the device map builder on the caller's
// stream. The caller passes only inputs and outputs.
//
// The array costs kScratchBytes of memory on every GPU that loads the library,
// until the process exits. Shapes whose map and workspace do not fit are
// rejected with KREA_ERR_TOO_LARGE before anything is launched.
//
// All calls share the one array and each call overwrites what it reads (the map
// builder writes every row pointer and listed entry, the quantiser every
// workspace word it later reads; nothing must start at zero). Calls whose work
// overlaps on the GPU -- on two streams, or two threads sharing a device -- race
// on the array and must not be issued; calls on one stream are ordered and safe.
//
// The first call on a device looks the array's device address up with
// cudaGetSymbolAddress (the array's name in host code is only a host-side
// stand-in, not a device address); make that first call before any CUDA stream
// capture on that device.
#include <cuda_runtime.h>

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

}  // namespace

extern "C" int krea_attn_fwd_noalloc(const void* q, const void* k, const void* v, const void* gate, void* out,
                                     int text_len, int grid_h, int grid_w, int mode,
                                     const krea_attn_params_t* p, void* stream) {
  // the argument checks of krea_attn_fwd
  int rc = check_params(p);
  if (rc != KREA_OK) return rc;
  Geometry g;
  rc = make_geometry(text_len, grid_h, grid_w, mode, p, &g);
  if (rc != KREA_OK) return rc;
  int q_len = 0;
  rc = check_forward(q, k, v, gate, out, g, p, &q_len);
  if (rc != KREA_OK) return rc;
  rc = check_device_sm100();
  if (rc != KREA_OK) return rc;

  // scratch layout: row pointers, packed map entries (n_tiles^2 always suffice),
  // then the TileMix workspace
  const bool use_int8 = tilemix_int8_tiles(g) > 0;
  const bool centred = mode == KREA_MODE_TILEMIX && p->smooth_k;
  const size_t nt = (size_t)g.n_tiles;
  const size_t off_entries = up256((nt + 1) * sizeof(int32_t));
  const size_t off_ws = up256(off_entries + nt * nt * sizeof(int32_t));
  size_t need = off_ws;
  if (use_int8 || centred)
    need += workspace_layout(p->batch, g.L, p->num_q_heads, p->num_kv_heads, p->head_dim,
                             p->in_dtype == KREA_F32 ? 4 : 2, p->smooth_k)
                .total;
  if (need > kScratchBytes) return KREA_ERR_TOO_LARGE;

  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != KREA_OK) return rc;
  char* sc = static_cast<char*>(scratch);
  int32_t* row_ptr = reinterpret_cast<int32_t*>(sc);
  int32_t* entries = reinterpret_cast<int32_t*>(sc + off_entries);
  // the tile map, built on the stream into the array (bit-identical to the map
  // krea_attn_fwd caches)
  rc = launch_build_map(g, row_ptr, entries, nullptr, nullptr, (int)(nt * nt), p->status, stream);
  if (rc != KREA_OK) return rc;
  // the attention reads the map just built on the stream: it never overlaps it
  krea_attn_params_t pa = *p;
  pa.overlap_previous = 0;
  return launch_forward(q, k, v, gate, out, g, &pa, q_len, row_ptr, entries, use_int8, sc + off_ws,
                        kScratchBytes - off_ws, stream);
}
