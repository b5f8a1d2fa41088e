// QK prologue of the Krea 2 attention core: RMSNorm then the 3-axis rotary
// embedding, the two steps that run on q and k right before attention
// ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What it actually
// patches"), in one pass over HBM instead of one pass each.
//
//   y = rope(x * gamma / sqrt(mean(x^2) + eps))   per (batch, token, head) vector
//
// in fp32 (pairs of channels per packed instruction), the reciprocal square
// root to within 2^-22 relative, rounded once to the input dtype.
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
#include "ptx_sm100.cuh"

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

// 512 threads = 16 warps. A row (token, head) of d channels is held by d/8
// lanes, 8 channels (16 bytes) each, so one warp access covers RPW = 32 / (d/8)
// rows. Channel pairs (2i, 2i+1) never straddle lanes. Each thread makes STEPS =
// 8 / RPW accesses, every load issued before the first use:
//  - without codes, grid (ceil(L / (16 RPW)), ceil(H / STEPS), B): a thread keeps
//    one token and steps through STEPS consecutive heads, so its rotary table
//    entries are loaded once for all of them;
//  - with codes, grid (ceil(L / 128), H, B): the CTA holds one head's whole
//    128-token block (the scale is its absmax), a thread steps through tokens.
template <bool BF16, int D, bool CODES>
__global__ void __launch_bounds__(512, CODES ? 1 : 2) prologue_kernel(PrologueDevParams p) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp access
  constexpr int STEPS = 8 / RPW;   // accesses per thread
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  const int c0 = 8 * li;            // this lane's channels c0 .. c0 + 7
  const int pj0 = c0 / 2;           // and its rotary pairs pj0 .. pj0 + 3
  // the (token, head) of step st
  auto token_of = [&](int st) {
    return CODES ? (int)blockIdx.x * kTile + warp * 8 + st * RPW + sub : (int)blockIdx.x * (16 * RPW) + warp * RPW + sub;
  };
  auto head_of = [&](int st) { return CODES ? (int)blockIdx.y : (int)blockIdx.y * STEPS + st; };
  __shared__ float red[16];
  uint64_t g2[4];  // the weights as f32 pairs: the arithmetic below is packed (two lanes per op)
#pragma unroll
  for (int j = 0; j < 4; ++j)
    g2[j] = p.gamma ? ptx::f2(p.gamma[c0 + 2 * j], p.gamma[c0 + 2 * j + 1]) : ptx::f2(1.0f, 1.0f);
  float keep[CODES ? STEPS : 1][8];  // stored values, for the codes
  float amax = 0.f;
  uint4 raw[STEPS];
#pragma unroll
  for (int st = 0; st < STEPS; ++st) {
    const int t = token_of(st), hh = head_of(st);
    raw[st] = t < p.L && hh < p.H
                  ? *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + b * p.x_stride[0] +
                                                    (long long)t * p.x_stride[1] + hh * p.x_stride[2] + c0)
                  : make_uint4(0u, 0u, 0u, 0u);
  }
  // without codes every step has the same token: its table entries, once
  float4 cs_tok[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  if constexpr (!CODES) {
    const int t = token_of(0);
    if (t < p.L) {
      const float4* tab =
          reinterpret_cast<const float4*>(p.table + 2LL * (((long long)t + p.token_offset) * p.n_pairs + pj0));
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
        if (pj0 + 2 * q2 < p.n_pairs) cs_tok[q2] = tab[q2];
    }
  }
#pragma unroll
  for (int st = 0; st < STEPS; ++st) {
    const int t = token_of(st), hh = head_of(st);
    const bool live = t < p.L && hh < p.H;
    uint64_t x2[4];  // channel pairs (2j, 2j+1) of this lane, as f32 pairs
    float ss = 0.f;
    {
      const uint4 u = raw[st];  // zero for rows past L or H
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
      uint64_t acc = ptx::f2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x2[j] = ptx::f2(ld_f<BF16>(e[2 * j]), ld_f<BF16>(e[2 * j + 1]));
        acc = ptx::fma2(x2[j], x2[j], acc);
      }
      float s0, s1;
      ptx::unf2(acc, s0, s1);
      ss = s0 + s1;
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    if (live) {
      // 1 / sqrt(mean + eps): 1/D is a power of two (exact), rsqrt to within 2^-22
      const float r = rsqrtf(__fadd_rn(ss * (1.0f / (float)D), p.eps));
      const uint64_t r2 = ptx::f2(r, r);
#pragma unroll
      for (int j = 0; j < 4; ++j) x2[j] = ptx::mul2(ptx::mul2(x2[j], r2), g2[j]);
      const long long tg = (long long)t + p.token_offset;  // token in the whole sequence
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {  // two pairs per 16-byte table entry
        if (pj0 + 2 * q2 >= p.n_pairs) break;
        const float4 cs =
            CODES ? reinterpret_cast<const float4*>(p.table + 2LL * (tg * p.n_pairs + pj0))[q2] : cs_tok[q2];
        // (a0, a1) -> (a0 c - a1 s, a0 s + a1 c) = (a0, a0) (c, s) + (a1, a1) (-s, c)
        float a0, a1, b0, b1;
        ptx::unf2(x2[2 * q2], a0, a1);
        ptx::unf2(x2[2 * q2 + 1], b0, b1);
        x2[2 * q2] = ptx::fma2(ptx::f2(a1, a1), ptx::f2(-cs.y, cs.x), ptx::mul2(ptx::f2(a0, a0), ptx::f2(cs.x, cs.y)));
        x2[2 * q2 + 1] =
            ptx::fma2(ptx::f2(b1, b1), ptx::f2(-cs.w, cs.z), ptx::mul2(ptx::f2(b0, b0), ptx::f2(cs.z, cs.w)));
      }
      // where this head's row goes: y, or a peer's buffer of the sequence <-> head exchange
      uint16_t* ybase = static_cast<uint16_t*>(p.y);
      int hy = hh;
      if (p.heads_per_peer > 0) {
        const int j = hh / p.heads_per_peer;
        ybase = static_cast<uint16_t*>(p.y_peer[j]);
        hy = hh - j * p.heads_per_peer;
      }
      float x[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) ptx::unf2(x2[j], x[2 * j], x[2 * j + 1]);
      uint4 u;
      uint16_t* e = reinterpret_cast<uint16_t*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        e[j] = st_f<BF16>(x[j]);
        if constexpr (CODES) {
          keep[st][j] = ld_f<BF16>(e[j]);  // the codes below are decided on the stored values
          amax = fmaxf(amax, fabsf(keep[st][j]));
        }
      }
      *reinterpret_cast<uint4*>(ybase + b * p.y_stride[0] + tg * p.y_stride[1] + hy * p.y_stride[2] + c0) = u;
    } else if constexpr (CODES) {
#pragma unroll
      for (int j = 0; j < 8; ++j) keep[st][j] = 0.f;
    }
  }
  if constexpr (!CODES) return;
  else {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 16; ++w) amax = fmaxf(amax, red[w]);
  const float scale = __fdiv_rn(amax, 127.0f);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
  const int h = blockIdx.y;
  if (threadIdx.x == 0) p.scales[((long long)b * p.H + h) * p.nt + blockIdx.x] = scale;
#pragma unroll
  for (int st = 0; st < STEPS; ++st) {
    const int t = token_of(st);
    if (t >= p.L) continue;
    uint2 u;
    int8_t* e = reinterpret_cast<int8_t*>(&u);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float q = rintf(__fmul_rn(keep[st][j], inv));
      q = fminf(fmaxf(q, -127.f), 127.f);
      e[j] = (int8_t)(int)q;
    }
    *reinterpret_cast<uint2*>(p.codes + (((long long)b * p.L + t) * p.H + h) * D + c0) = u;
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
  const bool codes = p.codes != nullptr;
  if (p.d != 128 && p.d != 64) return KREA_ERR_UNSUPPORTED;
  // rows per warp access 256 / d, accesses per thread 8 / that (see the kernel)
  const int rpw = 256 / p.d, steps = 8 / rpw;
  const dim3 grid = codes ? dim3((unsigned)p.nt, (unsigned)p.H, (unsigned)p.B)
                          : dim3((unsigned)((p.L + 16 * rpw - 1) / (16 * rpw)), (unsigned)((p.H + steps - 1) / steps),
                                 (unsigned)p.B);
  if (p.d == 128) {
    if (bf16) codes ? prologue_kernel<true, 128, true><<<grid, 512, 0, s>>>(p)
                    : prologue_kernel<true, 128, false><<<grid, 512, 0, s>>>(p);
    else codes ? prologue_kernel<false, 128, true><<<grid, 512, 0, s>>>(p)
               : prologue_kernel<false, 128, false><<<grid, 512, 0, s>>>(p);
  } else {
    if (bf16) codes ? prologue_kernel<true, 64, true><<<grid, 512, 0, s>>>(p)
                    : prologue_kernel<true, 64, false><<<grid, 512, 0, s>>>(p);
    else codes ? prologue_kernel<false, 64, true><<<grid, 512, 0, s>>>(p)
               : prologue_kernel<false, 64, false><<<grid, 512, 0, s>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace krea
