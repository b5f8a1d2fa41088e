// QK prologue of the Krea 2 attention core: RMSNorm then the 3-axis rotary
// embedding, the two steps that run on q and k right before attention
// ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What it actually
// patches"), in one pass over HBM instead of one pass each.
//
//   y = rope(x * gamma / sqrt(mean(x^2) + eps))   per (batch, token, head) vector
//
// rope turns adjacent channel pairs (2i, 2i+1) of three consecutive channel
// groups (axes_dim[0..2] channels) by pos[t][a] * theta^(-2i / axes_dim[a]).
// The cos/sin of every (token, pair) come from a table built once per geometry
// (rope_table_kernel, fp64 angles and trigonometry rounded to fp32): the 28
// blocks of the model and both q and k share it.
//
// Optionally the same pass writes the TileMix INT8 codes of y and their
// per-(batch, head, 128-token block) scales, decided exactly as the quantiser in
// quant.cu decides them from the stored y (absmax / 127, IEEE division and
// multiply, round half to even, clamp to +-127), so the two agree bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "krea_internal.h"

namespace krea {
namespace {

template <bool BF16>
__device__ __forceinline__ float ld_f(uint16_t u) {
  if constexpr (BF16) return __bfloat162float(__ushort_as_bfloat16(u));
  else return __half2float(__ushort_as_half(u));
}

template <bool BF16>
__device__ __forceinline__ uint16_t st_f(float x) {
  if constexpr (BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
  else return __half_as_ushort(__float2half_rn(x));
}

// One thread per (token, pair): the pair's axis and index within the axis, the
// angle and its cos/sin in fp64, rounded once to fp32.
__global__ void __launch_bounds__(256) rope_table_kernel(const int32_t* pos, int tokens, int n0, int n1, int n2,
                                                         double theta, float2* table) {
  const int np = (n0 + n1 + n2) / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)tokens * np) return;
  const int t = (int)(idx / np), j = (int)(idx % np);
  int a, i, n;
  if (j < n0 / 2) {
    a = 0; i = j; n = n0;
  } else if (j < (n0 + n1) / 2) {
    a = 1; i = j - n0 / 2; n = n1;
  } else {
    a = 2; i = j - (n0 + n1) / 2; n = n2;
  }
  const double ang = (double)pos[3 * (long long)t + a] * pow(theta, -2.0 * i / n);
  double s, c;
  sincos(ang, &s, &c);
  table[idx] = make_float2((float)c, (float)s);
}

// Grid (ceil(L / 128), H, B), 128 threads: thread = token, its whole row in registers.
template <bool BF16, int D>
__global__ void __launch_bounds__(128) prologue_kernel(PrologueDevParams p) {
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = blk * kTile + threadIdx.x;
  const bool live = t < p.L;
  __shared__ float red[4];
  float x[D];
  float amax = 0.f;
  if (live) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + b * p.x_stride[0] +
                                                      (long long)t * p.x_stride[1] + h * p.x_stride[2]);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const uint4 u = src[i];
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        x[8 * i + j] = ld_f<BF16>(e[j]);
        ss = __fmaf_rn(x[8 * i + j], x[8 * i + j], ss);
      }
    }
    // 1 / sqrt(mean + eps), each step rounded once (IEEE)
    const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)D), p.eps));
#pragma unroll
    for (int c = 0; c < D; ++c) x[c] = p.gamma ? __fmul_rn(__fmul_rn(x[c], r), p.gamma[c]) : __fmul_rn(x[c], r);
    const float4* tab = reinterpret_cast<const float4*>(p.table + 2LL * t * p.n_pairs);  // (cos, sin) pairs
#pragma unroll
    for (int j2 = 0; j2 < D / 4; ++j2) {  // two pairs per 16-byte table load
      if (2 * j2 >= p.n_pairs) break;
      const float4 cs = tab[j2];
      const float c0 = cs.x, s0 = cs.y, c1 = cs.z, s1 = cs.w;
      const float a0 = x[4 * j2], a1 = x[4 * j2 + 1];
      x[4 * j2] = __fmaf_rn(a0, c0, -__fmul_rn(a1, s0));
      x[4 * j2 + 1] = __fmaf_rn(a0, s0, __fmul_rn(a1, c0));
      if (2 * j2 + 1 < p.n_pairs) {
        const float b0 = x[4 * j2 + 2], b1 = x[4 * j2 + 3];
        x[4 * j2 + 2] = __fmaf_rn(b0, c1, -__fmul_rn(b1, s1));
        x[4 * j2 + 3] = __fmaf_rn(b0, s1, __fmul_rn(b1, c1));
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + b * p.y_stride[0] +
                                          (long long)t * p.y_stride[1] + h * p.y_stride[2]);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      uint4 u;
      uint16_t* e = reinterpret_cast<uint16_t*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        e[j] = st_f<BF16>(x[8 * i + j]);
        x[8 * i + j] = ld_f<BF16>(e[j]);  // the codes below are decided on the stored values
        amax = fmaxf(amax, fabsf(x[8 * i + j]));
      }
      dst[i] = u;
    }
  }
  if (!p.codes) return;  // uniform over the grid
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float scale = __fdiv_rn(amax, 127.0f);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
  if (threadIdx.x == 0) p.scales[((long long)b * p.H + h) * p.nt + blk] = scale;
  if (live) {
    int8_t* dst8 = p.codes + (((long long)b * p.L + t) * p.H + h) * D;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      uint4 u;
      int8_t* e = reinterpret_cast<int8_t*>(&u);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float q = rintf(__fmul_rn(x[16 * i + j], inv));
        q = fminf(fmaxf(q, -127.f), 127.f);
        e[j] = (int8_t)(int)q;
      }
      reinterpret_cast<uint4*>(dst8)[i] = u;
    }
  }
}

}  // namespace

int launch_rope_table(const int32_t* pos, int tokens, const int axes[3], double theta, float* table, void* stream) {
  const int np = (axes[0] + axes[1] + axes[2]) / 2;
  if (np == 0) return KREA_OK;
  const long long n = (long long)tokens * np;
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      pos, tokens, axes[0], axes[1], axes[2], theta, reinterpret_cast<float2*>(table));
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

int launch_prologue(const PrologueDevParams& p, bool bf16, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid((unsigned)p.nt, (unsigned)p.H, (unsigned)p.B);
  if (p.d == 128) {
    if (bf16) prologue_kernel<true, 128><<<grid, 128, 0, s>>>(p);
    else prologue_kernel<false, 128><<<grid, 128, 0, s>>>(p);
  } else if (p.d == 64) {
    if (bf16) prologue_kernel<true, 64><<<grid, 128, 0, s>>>(p);
    else prologue_kernel<false, 64><<<grid, 128, 0, s>>>(p);
  } else {
    return KREA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace krea
