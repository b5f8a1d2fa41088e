// TileMix quantiser of the Krea 2 attention core ("Krea 2 TileMix Attention
// (FP16/INT8 tiles)", section "The inputs that matter": smooth_k mean-centres K
// per head before quantisation).
//
// Steps, all memory-bound:
//   1. key mean: per (batch, kv head, channel), a fixed-order two-stage sum in
//      fp64 (chunks of 128 tokens, then the chunks in order), rounded once to fp32;
//   2. centred keys  k - mean  (one fp32 subtraction), stored in the input dtype
//      for the FP16 tiles, and quantised for the INT8 tiles;
//   3. INT8 codes, one symmetric scale per (batch, head, 128-token block):
//      scale = absmax / 127, code = rint(x * (127 / absmax)) clamped to +-127,
//      each operation rounded to fp32 (IEEE division and multiply).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "krea_internal.h"

namespace krea {
namespace {

template <bool BF16>
__device__ __forceinline__ float to_f(uint16_t u) {
  if constexpr (BF16) return __bfloat162float(__ushort_as_bfloat16(u));
  else return __half2float(__ushort_as_half(u));
}

template <bool BF16>
__device__ __forceinline__ uint16_t from_f(float x) {
  if constexpr (BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
  else return __half_as_ushort(__float2half_rn(x));
}

// Stage 1 of the key mean: grid (n_chunks, B). Each thread owns 8 consecutive
// channels (one 16-byte load per token, coalesced across the warp) and sums the
// chunk's tokens in fp64. Channels are (kv head, dim) pairs, Hkv * d of them.
template <bool BF16>
__global__ void __launch_bounds__(256) kmean_partial_kernel(QuantDevParams p) {
  const int chunk = blockIdx.x, b = blockIdx.y;
  const int C = p.Hkv * p.d;
  const int t0 = chunk * p.chunk_tokens;
  const int t1 = min(p.L, t0 + p.chunk_tokens);
  const uint16_t* k = static_cast<const uint16_t*>(p.k);
  for (int c8 = threadIdx.x; c8 < C / 8; c8 += blockDim.x) {
    const int c = c8 * 8;
    const int h = c / p.d, x = c % p.d;
    const uint16_t* src = k + b * p.k_stride[0] + h * p.k_stride[2] + x;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int t = t0; t < t1; ++t) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + (long long)t * p.k_stride[1]);
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += (double)to_f<BF16>(e[j]);
    }
    double* dst = p.part + ((long long)chunk * p.B + b) * C + c;
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = acc[j];
  }
}

// Stage 2: grid (ceil(C / 128), B), one thread per channel: the chunks in
// order, divided by L, rounded to fp32.
__global__ void __launch_bounds__(128) kmean_final_kernel(QuantDevParams p) {
  const int b = blockIdx.y;
  const int C = p.Hkv * p.d;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  double acc = 0.0;
  for (int j = 0; j < p.n_chunks; ++j) acc += p.part[((long long)j * p.B + b) * C + c];
  p.mu[(long long)b * C + c] = (float)(acc / (double)p.L);
}

// One 128-token block of one head: grid (nt, H, B), 128 threads, thread = token
// (each thread streams its own 256-byte row with 16-byte loads; measured faster
// on B200 than splitting rows across a warp).
// IS_KEY: subtract the mean (smooth_k), store the centred keys, quantise.
template <bool BF16, bool IS_KEY>
__global__ void __launch_bounds__(128) quant_block_kernel(QuantDevParams p) {
  constexpr int D = 128;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = blk * kTile + threadIdx.x;
  const bool live = t < p.L;
  const int H = IS_KEY ? p.Hkv : p.Hq;
  const long long* st = IS_KEY ? p.k_stride : p.q_stride;
  const uint16_t* src = static_cast<const uint16_t*>(IS_KEY ? p.k : p.q) + b * st[0] + h * st[2];
  __shared__ float mu[D];
  __shared__ float red[4];
  if (IS_KEY) {
    mu[threadIdx.x] = p.smooth_k ? p.mu[((long long)b * p.Hkv + h) * D + threadIdx.x] : 0.f;
    __syncthreads();
  }
  float x[D];
  float amax = 0.f;
  if (live) {
    const uint4* row = reinterpret_cast<const uint4*>(src + (long long)t * st[1]);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      uint4 u = row[i];
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = to_f<BF16>(e[j]);
        if (IS_KEY) v = __fsub_rn(v, mu[i * 8 + j]);
        x[i * 8 + j] = v;
        amax = fmaxf(amax, fabsf(v));
      }
    }
    if (IS_KEY && p.kc) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.kc) +
                                            (((long long)b * p.L + t) * p.Hkv + h) * D);
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        uint4 u;
        uint16_t* e = reinterpret_cast<uint16_t*>(&u);
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = from_f<BF16>(x[i * 8 + j]);
        dst[i] = u;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) x[i] = 0.f;
  }
  // block absmax
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float scale = __fdiv_rn(amax, 127.0f);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
  if (threadIdx.x == 0) {
    float* sc = IS_KEY ? p.sk : p.sq;
    sc[((long long)b * H + h) * p.nt + blk] = scale;
  }
  if (live) {
    int8_t* dst8 = (IS_KEY ? p.k8 : p.q8) + (((long long)b * p.L + t) * H + h) * D;
    uint4* d4 = reinterpret_cast<uint4*>(dst8);
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      uint4 u;
      int8_t* e = reinterpret_cast<int8_t*>(&u);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float r = rintf(__fmul_rn(x[i * 16 + j], inv));
        r = fminf(fmaxf(r, -127.f), 127.f);
        e[j] = (int8_t)(int)r;
      }
      d4[i] = u;
    }
  }
}

template <bool BF16>
int run(const QuantDevParams& p, cudaStream_t s) {
  if (p.d != 128) return KREA_ERR_UNSUPPORTED;
  if (p.smooth_k) {
    kmean_partial_kernel<BF16><<<dim3(p.n_chunks, p.B), 256, 0, s>>>(p);
    kmean_final_kernel<<<dim3((p.Hkv * p.d + 127) / 128, p.B), 128, 0, s>>>(p);
  }
  quant_block_kernel<BF16, true><<<dim3(p.nt, p.Hkv, p.B), 128, 0, s>>>(p);
  if (p.quant_q) quant_block_kernel<BF16, false><<<dim3(p.nt, p.Hq, p.B), 128, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace

int launch_quantize(const QuantDevParams& p, bool bf16, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return bf16 ? run<true>(p, s) : run<false>(p, s);
}

}  // namespace krea
