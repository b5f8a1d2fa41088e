// Sequence <-> head exchange for callers that split the joint [text, image]
// sequence by token across ranks. The attention heads are independent and query
// head h reads kv head h / rep ("Krea 2 TileMix Attention (FP16/INT8 tiles)",
// section "What it actually patches"), so a rank can run the core on a slice of
// the heads over the whole sequence; these copies move rows between the two
// splits.
//
// A push over peer memory: every rank stores its rows straight into the
// destination buffer of the rank that owns them (an NVLink peer mapping, or this
// GPU's own memory), in the destination's final layout. Nothing is packed and no
// library collective runs; the caller's stream-ordered barrier before the
// consumer's first read is the only synchronisation. Bound by HBM reads and
// NVLink (or HBM) writes: every byte moves once.
#include <cuda_runtime.h>

#include "krea_internal.h"

namespace krea {
namespace {

// Grid (x, B). Batch b's rows (t, h) in source order, 2^chunk_shift pieces of 16
// bytes each, are numbered i = ((t * Hs + h) << chunk_shift) + piece; thread i
// of a grid-stride loop moves piece i, four pieces (one grid stride apart) per
// iteration with the loads issued before the stores. Consecutive threads read
// consecutive source bytes, and a destination row stays contiguous.
__global__ void __launch_bounds__(256) exchange_kernel(ExchangeDevParams p) {
  constexpr int U = 4;
  const int b = blockIdx.y;
  const unsigned n = ((unsigned)p.Ls * (unsigned)p.Hs) << p.chunk_shift;
  const unsigned stride = gridDim.x * blockDim.x;
  const unsigned mask = (1u << p.chunk_shift) - 1u;
  const char* src = static_cast<const char*>(p.src) + (long long)b * p.s_stride[0] * p.es;
  for (unsigned base = blockIdx.x * blockDim.x + threadIdx.x; base < n; base += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const unsigned i = base + u * stride;
      if (i < n) {
        const unsigned row = i >> p.chunk_shift;
        const unsigned t = row / (unsigned)p.Hs, h = row - t * (unsigned)p.Hs;
        v[u] = __ldg(reinterpret_cast<const uint4*>(src + ((long long)t * p.s_stride[1] + (long long)h * p.s_stride[2]) * p.es +
                                                    16u * (i & mask)));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const unsigned i = base + u * stride;
      if (i < n) {
        const unsigned row = i >> p.chunk_shift;
        const int t = (int)(row / (unsigned)p.Hs), h = (int)(row - (unsigned)t * (unsigned)p.Hs);
        int peer, td, hd;
        if (p.to_heads) {
          peer = h / p.heads_per_rank;
          hd = h - peer * p.heads_per_rank;
          td = p.rank * p.tokens_per_rank + t;
        } else {
          peer = t / p.tokens_per_rank;
          td = t - peer * p.tokens_per_rank;
          hd = p.rank * p.Hs + h;
        }
        char* dst = static_cast<char*>(p.dst[peer]);
        *reinterpret_cast<uint4*>(dst + ((long long)b * p.d_stride[0] + (long long)td * p.d_stride[1] +
                                         (long long)hd * p.d_stride[2]) * p.es + 16u * (i & mask)) = v[u];
      }
    }
  }
  // the stores into a peer's memory are performed before this grid completes
  __threadfence_system();
}

}  // namespace

int launch_exchange(const ExchangeDevParams& p, void* stream) {
  const unsigned long long n = ((unsigned long long)p.Ls * (unsigned long long)p.Hs) << p.chunk_shift;
  if (n == 0) return KREA_OK;
  // about 8 CTAs of 256 threads per SM (148 SMs) over the whole grid, split
  // across the batch; each thread moves 4 pieces per loop iteration
  const unsigned long long per_b = (n + 256ull * 4 - 1) / (256ull * 4);
  const unsigned long long total = per_b * (unsigned long long)p.B;
  const unsigned long long target = total < 1184ull ? total : 1184ull;
  unsigned gx = (unsigned)((target + p.B - 1) / p.B);
  if (gx == 0) gx = 1;
  exchange_kernel<<<dim3(gx, (unsigned)p.B), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace krea
