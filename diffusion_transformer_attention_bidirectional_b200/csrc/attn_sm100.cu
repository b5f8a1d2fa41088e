// Attention kernel of the Krea 2 core for B200 (sm_100a): bidirectional
// online-softmax attention over 128 x 128 score tiles listed by a tile map,
// FP16/BF16 or INT8 QK^T on tcgen05 tensor cores with TMEM accumulators,
// K/V tiles staged by TMA, sigmoid(gate) fused into the epilogue.
//
// What it computes ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What
// it actually patches"; "Krea 2 Scanline Attention", section "What the mask
// actually is"; "LayerStream: Krea2 Chunking", section "What the node does to
// the block"):
//   out[b,t,h,:] = sigmoid(gate[b,t,h,:]) * sum_j softmax_j(scale * s(t,j)) v[b,j,h/rep,:]
// over the key tiles of the query tile's map row, in ascending key-tile order;
// masked tiles apply the padding / scanline predicate per key slot, skipped
// tiles are never loaded.
//
// One CTA = one 128-row query tile of TWO query heads that share a kv head
// (GQA resolved by index: kv head = h / rep), so every K/V tile loaded from HBM
// feeds two 128 x 128 x d products. Warp roles (384 threads, 3 warpgroups):
//   warps 0-3  softmax for head 0 (thread = query row), epilogue
//   warps 4-7  softmax for head 1
//   warp  8    TMA producer: K_j, V_j into a 4-slot ring of 32 KB (thread 0 issues
//              Q and the first K, V right after setting up the barriers)
//   warp  9    TMEM allocator and the single thread issuing tcgen05.mma
//   warps 10-11 idle (they complete the third warpgroup)
// The launch gives 168 registers per thread; the producer/MMA warpgroup drops to
// 56 (setmaxnreg.dec) so the two softmax warpgroups can rise to 224 and keep a
// whole 128-score row in registers: 32*56 + 2*32*224 = 3*32*168 per SM
// sub-partition. The host refuses to launch unless the kernel was compiled to
// exactly 168 registers, so the raise can never wait for registers that are
// not there.
// TMEM (512 columns x 128 lanes): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512); P_i (16-bit, 64 columns) overwrites the first half of S_i.
// Per kv tile j and head i the MMA thread issues, in order,
//   PV_i(j-1) on keys 0..63 (as soon as the softmax has written that half of
//   P_i), PV_i(j-1) on keys 64..127 (when all of P_i is written), then
//   QK_i(j): S_i = Q_i K_j^T
// and commits S_i after QK_i(j); tcgen05 operations of one thread complete in
// issue order, so when softmax i sees S_i(j) complete, PV_i(j-1) is complete
// too and O_i may be rescaled in place before P_i(j) is released.
// The running max is only moved when it grows by more than 2^8 (lazy rescale):
// exact, since numerator and denominator share the stale maximum.
//
// Every barrier wait is bounded (p.wait_limit SM cycles): a wait that runs out
// sets a CTA abort flag and writes KREA_ERR_DEVICE_TIMEOUT to p.status; the
// producer then waits (bounded) for its own TMA copies in flight, the MMA thread
// for its own MMAs, and the CTA frees its TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "krea_internal.h"
#include "ptx_sm100.cuh"

namespace krea {
namespace {

constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
constexpr int kSlots = 4;
constexpr uint32_t kBox = 16384;       // one TMA box: 128 rows x 128 bytes
constexpr uint32_t kTileBytes = 32768; // 128 x 128 16-bit
constexpr uint32_t SM_Q = 0;           // 2 x 32 KB
constexpr uint32_t SM_Q8 = 65536;      // 2 x 16 KB
constexpr uint32_t SM_SLOT = 98304;    // kSlots x 32 KB
constexpr uint32_t SM_BAR = SM_SLOT + kSlots * kTileBytes;
constexpr int BAR_Q = 0,  // 2: Q of head i landed
              BAR_FULL = 2, BAR_EMPTY = BAR_FULL + kSlots, BAR_S = BAR_EMPTY + kSlots,
              BAR_P = BAR_S + 2, BAR_O = BAR_P + 2, BAR_DRAIN = BAR_O + 2, BAR_NEVER = BAR_DRAIN + 1,
              BAR_QFREE = BAR_NEVER + 1,  // the last QK^T finished: the Q area may be reused
              BAR_GATE = BAR_QFREE + 1,   // gate tiles landed in the Q area
              BAR_EPI = BAR_GATE + 1,     // 2 x 4: box x of head i staged for its TMA store (i * 4 + x)
              BAR_Q8 = BAR_EPI + 8,       // INT8 query codes landed (rows with INT8 tiles only)
              BAR_PH = BAR_Q8 + 1,        // 2: the first half of P_i (keys 0..63) written
              BAR_QN = BAR_PH + 2,        // 2: raw Q rows of head i normalised and rotated in place (q_rope)
              N_BARS = BAR_QN + 2;
constexpr uint32_t SM_TMEM_PTR = SM_BAR + 8 * N_BARS;
constexpr uint32_t SM_ABORT = SM_TMEM_PTR + 4;
constexpr uint32_t SMEM_USED = SM_BAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // slack to align the base to 1024 bytes
static_assert(8 * N_BARS + 8 <= 512, "barrier block overflow");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(kSlots == 4, "the staged epilogue places head 0's output in the even slots, head 1's in the odd");
constexpr long long kDrainLimit = 4000000000LL;
// Pairs of exponentials computed by the FMA-pipe polynomial: bit (i % 8) of
// kPolyMask for pair i. Measured on B200 inside this kernel: every offload
// fraction tried (1/4, 3/8) was slower than none, since the softmax warps are
// then bound by issue and latency rather than by the exponential unit; the
// polynomial stays available (debug_flags bit 1 runs every exponential on it).
constexpr uint32_t kPolyMask = 0x00u;
// bf16 query tiles whose map row lists at most this many key tiles (<= 1024 keys)
// take P to 16 bits: the 2^-9 relative rounding of single weights bounds the
// error of short rows near 2^-9 max|v|, and only averages out over longer rows.
constexpr int kSplitMaxTiles = 8;
constexpr float kNegInf = -INFINITY;

struct Ctl {
  volatile int* abort;
  int32_t* status;
  long long limit;
};

__device__ __forceinline__ void raise_timeout(const Ctl& c) {
  *c.abort = 1;
  if (c.status) atomicCAS(c.status, 0, KREA_ERR_DEVICE_TIMEOUT);
}

// Hardware suspend hint of every barrier wait (ns): a waiting thread parks until the
// phase completes instead of polling, leaving its sub-partition's issue slots to the
// warps that compute (measured: +3 to +5 % on the dense 4 MP call).
constexpr uint32_t kSuspendNs = 0x100000u;

// Single-thread bounded wait.
__device__ __forceinline__ bool wait1(const Ctl& c, uint32_t bar, uint32_t parity) {
  if (ptx::mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
  const long long t0 = clock64();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (*c.abort) return false;
    if (clock64() - t0 > c.limit) {
      raise_timeout(c);
      return false;
    }
  }
}

// Whole-warp bounded wait: every lane polls, the warp leaves together.
__device__ __forceinline__ bool wait_warp(const Ctl& c, uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    const bool done = ptx::mbar_try_wait_sleep(bar, parity, kSuspendNs);
    if (__all_sync(0xffffffffu, done)) return true;
    const bool stop = *c.abort || (clock64() - t0 > c.limit);
    if (__any_sync(0xffffffffu, stop)) {
      if ((threadIdx.x & 31) == 0 && !*c.abort) raise_timeout(c);
      return false;
    }
  }
}

// Wait used only on the abort path, for work this thread itself started.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kDrainLimit) return;
}

// First physical token of logical tile `tile` (text slots map to themselves,
// image slots start at Pt).
__device__ __forceinline__ int tile_row0(int tile, const AttnDevParams& p) {
  const int s0 = tile * kTile;
  return s0 < p.Pt ? s0 : s0 - p.Pt + p.T;
}

// Work item of CTA idx: (batch, kv head, head pair, query tile), query tile
// fastest; the slice's first n_heavy query tiles (the longest map rows) come
// first for every (batch, kv head, head pair), then the rest.
struct Item {
  int qt, pair, g, b;
};
__device__ __forceinline__ Item decode_item(int idx, const AttnDevParams& p) {
  const int heavy_ctas = p.B * p.Hkv * p.npairs * p.n_heavy;
  int ql;
  if (idx < heavy_ctas) {
    ql = idx % p.n_heavy;
    idx /= p.n_heavy;
  } else {
    idx -= heavy_ctas;
    const int n_light = p.n_slice_tiles - p.n_heavy;
    ql = p.n_heavy + idx % n_light;
    idx /= n_light;
  }
  Item it;
  it.qt = p.tile_begin + ql;
  it.pair = idx % p.npairs;
  idx /= p.npairs;
  it.g = idx % p.Hkv;
  it.b = idx / p.Hkv;
  return it;
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) return ptx::pack_bf16(lo, hi);
  else return ptx::pack_f16(lo, hi);
}

template <bool BF16>
__device__ __forceinline__ float h2f(uint16_t u) {
  if constexpr (BF16) return __uint_as_float((uint32_t)u << 16);
  else {
    float f;
    asm("{\n\t.reg .f16 t;\n\tmov.b16 t, %1;\n\tcvt.f32.f16 %0, t;\n\t}" : "=f"(f) : "h"(u));
    return f;
  }
}

// sigmoid(x) = 1 / (1 + 2^(-x log2 e)): two exponential-unit operations; x -> -inf
// gives 1/inf = 0, x -> +inf gives 1.
__device__ __forceinline__ float sigmoidf_(float x) {
  return ptx::rcp_approx(1.0f + ptx::ex2(x * -1.4426950408889634f));
}

// 2^x on the FMA pipe for a pair of values, so that part of the exponentials
// leaves the MUFU unit (whose 16 results per clock per SM would otherwise bound
// the softmax). Range reduction x = n + f with n = rint(x), f in [-1/2, 1/2]
// (rounding by adding 1.5 * 2^23), a polynomial for 2^f, and 2^n applied by
// adding n to the exponent field. The polynomial keeps p(0) = 1 exactly and is a
// minimax fit of the relative error of 2^f on [-1/2, 1/2] (Lawson's iteratively
// reweighted least squares): degree 3, max relative error 1.2e-4, for bf16
// probabilities (8-bit significand); degree 4, 2.9e-6, for fp16 (11-bit).
// x is clamped to -127, where the result is exactly 0 (masked keys stay 0).
template <bool BF16>
__device__ __forceinline__ void exp2_poly2(float& a, float& b) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  a = fmaxf(a, -127.0f);
  b = fmaxf(b, -127.0f);
  const uint64_t x = ptx::f2(a, b);
  const uint64_t j = ptx::add2(x, ptx::f2(kRound, kRound));
  const uint64_t n = ptx::add2(j, ptx::f2(-kRound, -kRound));
  const uint64_t f = ptx::fma2(n, ptx::f2(-1.0f, -1.0f), x);  // x - n
  uint64_t p;
  if constexpr (BF16) {
    p = ptx::fma2(ptx::f2(0.055417872965335846f, 0.055417872965335846f), f,
                  ptx::f2(0.242211252450943f, 0.242211252450943f));
    p = ptx::fma2(p, f, ptx::f2(0.6931995153427124f, 0.6931995153427124f));
  } else {
    p = ptx::fma2(ptx::f2(0.009585633873939514f, 0.009585633873939514f), f,
                  ptx::f2(0.05590590462088585f, 0.05590590462088585f));
    p = ptx::fma2(p, f, ptx::f2(0.2402404099702835f, 0.2402404099702835f));
    p = ptx::fma2(p, f, ptx::f2(0.6931242942810059f, 0.6931242942810059f));
  }
  p = ptx::fma2(p, f, ptx::f2(1.0f, 1.0f));
  float p0, p1, j0, j1;
  ptx::unf2(p, p0, p1);
  ptx::unf2(j, j0, j1);
  // the low mantissa bits of j hold n; shifting them into the exponent field
  a = __int_as_float(__float_as_int(p0) + (__float_as_int(j0) << 23));
  b = __int_as_float(__float_as_int(p1) + (__float_as_int(j1) << 23));
}

// The QK prologue on one head's raw Q tile in shared memory, in place, by the
// CTA's 256 softmax threads: RMSNorm then the 3-axis rotary turns ("Krea 2 TileMix
// Attention (FP16/INT8 tiles)", section "What it actually patches": both run on q
// right before the core). The work is split as krea_attn_qk_prologue splits it --
// D / 8 lanes per row, 8 channels (16 bytes) per lane, the sum of squares as an
// even/odd pair of fma chains per lane and then the lanes' butterfly, (x * r) *
// gamma, the same rotation, one rounding -- with every operation an explicitly
// rounded fp32 one, so the stored rows equal that pass's output bit for bit, and a
// row's rotary table entries are read by its lanes as one contiguous run. Row
// `row` of the 128-byte swizzled tile: 16-byte chunk c of the row (channels 8c ..
// 8c+7) sits in box c / 8 at chunk (c % 8) ^ (row % 8). The tile's rows are tokens
// qrow0 .. qrow0 + 127; rows past the sequence were zero-filled by the TMA unit
// and stay zero.
template <bool BF16, int D>
struct RopeQ {
  static constexpr int LPR = D / 8;                // lanes per row
  static constexpr int RPW = 32 / LPR;             // rows per warp step
  static constexpr int STEPS = kTile / (8 * RPW);  // steps of the eight warps over the 128 rows
  int li, sub, w, pj0;
  float4 cs[STEPS][2];  // this lane's table entries of every step: the same rows for every head

  // Everything that does not depend on Q: called before Q lands, so the table
  // loads' latency hides behind the Q copy.
  __device__ __forceinline__ void load_table(int qrow0, int tid, const AttnDevParams& p) {
    const int lane = tid & 31;
    w = tid >> 5;
    sub = lane / LPR;
    li = lane % LPR;
    pj0 = 4 * li;
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int tok = min(qrow0 + row_of(st), p.L - 1);
      const float4* tab = reinterpret_cast<const float4*>(p.q_table + 2LL * ((long long)tok * p.q_npairs + pj0));
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
        cs[st][q2] = pj0 + 2 * q2 < p.q_npairs ? __ldg(tab + q2) : make_float4(1.f, 0.f, 1.f, 0.f);
    }
  }
  __device__ __forceinline__ int row_of(int st) const { return (st * 8 + w) * RPW + sub; }
  __device__ __forceinline__ uint32_t chunk(uint32_t tile, int row) const {
    return tile + (uint32_t)(li >> 3) * kBox + (uint32_t)row * 128u + ((((uint32_t)li & 7u) ^ ((uint32_t)row & 7u)) << 4);
  }
  // One head's tile, in place.
  __device__ __forceinline__ void apply(uint32_t tile, int qrow0, const AttnDevParams& p) const {
    float gm[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) gm[j] = p.q_gamma ? p.q_gamma[8 * li + j] : 1.0f;
    uint4 raw[STEPS];
#pragma unroll
    for (int st = 0; st < STEPS; ++st) raw[st] = ptx::lds128(chunk(tile, row_of(st)));
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int row = row_of(st);
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&raw[st]);
      float x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = h2f<BF16>(e[j]);
      float se = 0.f, so = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        se = __fmaf_rn(x[2 * j], x[2 * j], se);
        so = __fmaf_rn(x[2 * j + 1], x[2 * j + 1], so);
      }
      float ss = __fadd_rn(se, so);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
      // a select for rows past the sequence (zero rows stay zero)
      const float r = qrow0 + row < p.L ? rsqrtf(__fadd_rn(ss * (1.0f / (float)D), p.q_eps)) : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(__fmul_rn(x[j], r), gm[j]);
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {  // pair pj0 + pp: (a0, a1) -> (a0 c - a1 s, a0 s + a1 c)
        if (pj0 + pp >= p.q_npairs) break;  // channels past the rotary axes pass unturned
        const float4 c4 = cs[st][pp >> 1];
        const float c = (pp & 1) ? c4.z : c4.x, sn = (pp & 1) ? c4.w : c4.y;
        const float a0 = x[2 * pp], a1 = x[2 * pp + 1];
        x[2 * pp] = __fmaf_rn(a1, -sn, __fmul_rn(a0, c));
        x[2 * pp + 1] = __fmaf_rn(a1, c, __fmul_rn(a0, sn));
      }
      ptx::sts128(chunk(tile, row), make_uint4(pack2<BF16>(x[0], x[1]), pack2<BF16>(x[2], x[3]),
                                               pack2<BF16>(x[4], x[5]), pack2<BF16>(x[6], x[7])));
    }
  }
};

// Online-softmax step of one 128-key tile for one query row held by this thread.
// v: the row of S (fp32 bits, or s32 for INT8 tiles), overwritten. mult: score
// scale in log2 units (softmax scale * log2 e, times s_q s_k for INT8 tiles).
// Key column c is admitted iff c < a1 or a2 <= c < a3 (masked tiles only).
// Writes P (16-bit pairs) over the first 64 columns of S, releasing the first 32
// (keys 0..63) on half_bar before the exponentials of keys 64..127 are taken, so
// that PV on those keys overlaps them; updates m, l and, when the running maximum
// moves, rescales O in TMEM (before either half of P is released).
// SPLIT (bf16 only): each weight p is also written as a second bf16 term
// p - bf16(p) over columns 64..127 of S (free once the row is in registers), so
// that two PV products give P to 16 significant bits instead of 8 (rows with few
// admitted keys, where the rounding of single weights does not average out).
template <bool BF16, bool IS8, bool MASKED, bool ALL_POLY, bool SPLIT>
__device__ __forceinline__ void softmax_tile(uint32_t (&v)[128], float mult, int a1, int a2, int a3, float& m,
                                             float& l, bool first, uint32_t tS, uint32_t tO, int d,
                                             uint32_t half_bar) {
  // INT8 tiles: an s32 sum x (|x| <= 128 * 127 * 127 < 2^21) becomes the float
  // 1.5 * 2^23 + x exactly by one integer add on its bits; the bias is taken out of the maximum below and folded
  // into the constant of the one FMA before each exponential
  constexpr float kBias = IS8 ? 12582912.0f : 0.0f;
#pragma unroll
  for (int c = 0; c < 128; ++c) {
    float r = IS8 ? __int_as_float((int)(v[c] + 0x4B400000u)) : __uint_as_float(v[c]);
    if constexpr (MASKED) r = ((c < a1) || (c >= a2 && c < a3)) ? r : kNegInf;
    v[c] = __float_as_uint(r);
  }
  float mx0 = kNegInf, mx1 = kNegInf, mx2 = kNegInf, mx3 = kNegInf;
#pragma unroll
  for (int c = 0; c < 128; c += 8) {  // four independent chains: short latency
    mx0 = ptx::max3(mx0, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
    mx1 = ptx::max3(mx1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
    mx2 = ptx::max3(mx2, __uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
    mx3 = ptx::max3(mx3, __uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
  }
  const float m_tile = (fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) - kBias) * mult;  // mult > 0; exact subtraction
  const float m_new = fmaxf(m, m_tile);
  if (first) {
    m = m_new;
  } else {
    const bool need = m_new > m + 8.0f;
    if (__any_sync(0xffffffffu, need)) {
      const float f = need ? ptx::ex2(m - m_new) : 1.0f;
      for (int j = 0; j < d / 32; ++j) {
        uint32_t o[32];
        __syncwarp();
        ptx::tmem_ld32(tO + 32u * j, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
        ptx::tmem_st32(tO + 32u * j, o);
      }
      if (need) {
        l *= f;
        m = m_new;
      }
    }
  }
  const float m_use = (m == kNegInf) ? 0.f : m;
  // (bias + x) mult - (bias mult + m) = x mult - m, the constant rounded once (INT8:
  // an error near 2^-24 * bias * mult, ~0.75 of one code unit's weight)
  const float c_use = IS8 ? __fmaf_rn(kBias, mult, m_use) : m_use;
  const uint64_t mult2 = ptx::f2(mult, mult), negm2 = ptx::f2(-c_use, -c_use);
  uint64_t acc0 = ptx::f2(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // 64 keys -> 32 columns of P per half
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c = 64 * h + 2 * i;
      const uint64_t x = ptx::fma2(ptx::f2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), mult2, negm2);
      float p0, p1;
      ptx::unf2(x, p0, p1);
      if (ALL_POLY || ((kPolyMask >> (i % 8)) & 1u)) {
        exp2_poly2<BF16>(p0, p1);
      } else {
        p0 = ptx::ex2(p0);
        p1 = ptx::ex2(p1);
      }
      if (i & 1) acc1 = ptx::add2(acc1, ptx::f2(p0, p1));
      else acc0 = ptx::add2(acc0, ptx::f2(p0, p1));
      pk[i] = pack2<BF16>(p0, p1);
      if constexpr (SPLIT) {  // the rounding residual, itself rounded to bf16
        const float r0 = p0 - __uint_as_float(pk[i] << 16), r1 = p1 - __uint_as_float(pk[i] & 0xffff0000u);
        v[64 * h + i] = pack2<BF16>(r0, r1);  // keys 64h .. 64h+63 of v are consumed: reuse their registers
      }
    }
    ptx::tmem_st32(tS + 32u * h, pk);
    if constexpr (SPLIT) ptx::tmem_st32(tS + 64u + 32u * h, *reinterpret_cast<const uint32_t(*)[32]>(&v[64 * h]));
    if (h == 0) {  // keys 0..63 of P are in TMEM: the tensor core may start on them
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(half_bar);
    }
  }
  float s0, s1, s2, s3;
  ptx::unf2(acc0, s0, s1);
  ptx::unf2(acc1, s2, s3);
  l += (s0 + s1) + (s2 + s3);
}

// The single thread that issues every tcgen05.mma of the CTA. Descriptors are
// built once and advanced by constant adds (the 14-bit start-address field
// cannot carry: shared addresses stay below 256 KB), and every K loop is
// unrolled, so that issuing keeps ahead of the tensor core (one 128x128x16 MMA
// completes every 64 cycles).
template <bool BF16, int D>
__device__ __forceinline__ void mma_thread(const AttnDevParams& p, uint32_t base, uint32_t tmem, int e0, int n,
                                           int nh, const Ctl& ctl, bool split) {
  auto bar = [&](int i) { return base + SM_BAR + 8u * (uint32_t)i; };
  constexpr uint32_t ab = BF16 ? 1u : 0u;
  constexpr uint32_t ID_QK = ptx::idesc(1, ab, 0, 0, 128, 128);
  constexpr uint32_t ID_QK8 = ptx::idesc(2, 1, 0, 0, 128, 128);
  constexpr uint32_t ID_PV = ptx::idesc(1, ab, 0, 1, D, 128);
  // low words of the shared-memory descriptors (start address >> 4 sits in bits 0..13)
  const uint32_t dq = ptx::sdesc_lo(base + SM_Q, 16);      // Q of head i: + i * 32 KB
  const uint32_t dq8 = ptx::sdesc_lo(base + SM_Q8, 16);    // Q codes of head i: + i * 16 KB
  const uint32_t dk = ptx::sdesc_lo(base + SM_SLOT, 16);   // slot s, K-major: + s * 32 KB
  const uint32_t dv = ptx::sdesc_lo(base + SM_SLOT, kBox); // slot s, MN-major (V)
  auto qk = [&](int i, int kind, uint32_t slot) {
    const uint32_t dS = tmem + (uint32_t)i * 128u;
    const uint32_t kd = dk + slot * (kTileBytes >> 4);
    if (kind & KREA_KIND_INT8) {
      const uint32_t qd = dq8 + (uint32_t)i * (kBox >> 4);
#pragma unroll
      for (int k = 0; k < 4; ++k)  // K = 32 bytes per step
        ptx::mma_i8_ss_lo(dS, qd + 2 * k, kd + 2 * k, ID_QK8, k > 0);
    } else {
      const uint32_t qd = dq + (uint32_t)i * (kTileBytes >> 4);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {  // K = 16 elements (32 bytes) per step
        constexpr uint32_t kb4 = kBox >> 4;
        const uint32_t off = (uint32_t)(k >> 2) * kb4 + (uint32_t)(k & 3) * 2u;
        ptx::mma_f16_ss_lo(dS, qd + off, kd + off, ID_QK, k > 0);
      }
    }
  };
  // PV over keys 64 half .. 64 half + 63 of the tile; lo = 1: the bf16 residual
  // terms of P (columns 64..127 of S) instead of the rounded weights
  auto pv = [&](int i, uint32_t slot, int half, uint32_t acc, int lo = 0) {
    const uint32_t dO = tmem + 256u + (uint32_t)i * 128u;
    const uint32_t aP = tmem + (uint32_t)i * 128u + 64u * (uint32_t)lo + 32u * (uint32_t)half;
    const uint32_t vd = dv + slot * (kTileBytes >> 4) + 512u * (uint32_t)half;  // 64 rows x 128 B
    ptx::mma_f16_ts_lo(dO, aP, vd, ID_PV, acc);
#pragma unroll
    for (int k = 1; k < 4; ++k)  // 16 keys per step: 8 TMEM columns of P, 16 rows of V (2 KB)
      ptx::mma_f16_ts_lo(dO, aP + 8u * k, vd + 128u * k, ID_PV, 1);
  };
  // the first two map entries are read before any wait, so their latency hides behind Q's
  const int ent0 = p.entries[e0];
  int e_next = n > 1 ? p.entries[e0 + 1] : 0;  // map entries are read one tile ahead
  // raw queries: wait for the softmax warps' prologue (which itself waited for Q)
  bool ok = wait1(ctl, bar(p.q_rope ? BAR_QN + 0 : BAR_Q + 0), 0);
  bool q8_ready = false;  // the INT8 query codes are awaited before the first INT8 tile
  auto need_q8 = [&](int kind) {
    if (!(kind & KREA_KIND_INT8) || q8_ready) return true;
    if (!wait1(ctl, bar(BAR_Q8), 0)) return false;
    ptx::tc_fence_after();
    q8_ready = true;
    return true;
  };
  uint32_t it = 0;
  if (ok) {
    ptx::tc_fence_after();
    ok = wait1(ctl, bar(BAR_FULL + 0), 0);
  }
  if (ok) ok = need_q8(ent0 & 3);
  if (ok) {
    ptx::tc_fence_after();
    const int kind0 = ent0 & 3;
    for (int i = 0; i < nh && ok; ++i) {
      if (i > 0) {  // head i's Q (rotated after head 0's, with q_rope)
        ok = wait1(ctl, bar(p.q_rope ? BAR_QN + i : BAR_Q + i), 0);
        if (!ok) break;
        ptx::tc_fence_after();
      }
      qk(i, kind0, 0);
      ptx::tc_commit(bar(BAR_S + i));
    }
    ptx::tc_commit(bar(BAR_EMPTY + 0));
    if (n == 1) ptx::tc_commit(bar(BAR_QFREE));
    it = 1;
    for (int t = 0; t < n && ok; ++t) {
      const uint32_t slot_v = it % kSlots;
      ok = wait1(ctl, bar(BAR_FULL + slot_v), (it / kSlots) & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      ++it;
      const bool has_next = t + 1 < n;
      const uint32_t slot_k = it % kSlots;
      const int kind_next = e_next & 3;
      if (t + 2 < n) e_next = p.entries[e0 + t + 2];
      for (int i = 0; i < nh && ok; ++i) {
        ok = wait1(ctl, bar(BAR_PH + i), t & 1);  // keys 0..63 of P_i(t)
        if (!ok) break;
        ptx::tc_fence_after();
        pv(i, slot_v, 0, t > 0 ? 1u : 0u);
        ok = wait1(ctl, bar(BAR_P + i), t & 1);   // all of P_i(t)
        if (!ok) break;
        ptx::tc_fence_after();
        pv(i, slot_v, 1, 1u);
        if (split) {
          pv(i, slot_v, 0, 1u, 1);
          pv(i, slot_v, 1, 1u, 1);
        }
        if (!has_next) ptx::tc_commit(bar(BAR_O + i));  // O_i is final: its epilogue may start
        if (has_next) {
          if (i == 0) {
            ok = wait1(ctl, bar(BAR_FULL + slot_k), (it / kSlots) & 1) && need_q8(kind_next);
            if (!ok) break;
            ptx::tc_fence_after();
          }
          qk(i, kind_next, slot_k);
          ptx::tc_commit(bar(BAR_S + i));
        }
      }
      if (!ok) break;
      if (t + 2 == n) ptx::tc_commit(bar(BAR_QFREE));  // the last QK^T has been issued
      ptx::tc_commit(bar(BAR_EMPTY + slot_v));
      if (has_next) {
        ptx::tc_commit(bar(BAR_EMPTY + slot_k));
        ++it;
      }
    }
  }
  // every MMA this thread issued finishes before TMEM is freed, also when a
  // softmax warp gave up waiting on O
  ptx::tc_commit(bar(BAR_DRAIN));
  wait_drain(bar(BAR_DRAIN), 0);
}

// ---------------------------------------------------------------------------
template <bool BF16, bool ALL_POLY>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnMaps tm, const __grid_constant__ AttnDevParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sb = smem_raw + (base - raw);

  const Item item = decode_item((int)blockIdx.x, p);
  const int qt = item.qt, pair = item.pair, g = item.g, b = item.b;
  const int h0 = g * p.rep + pair * p.nh;
  // Every CTA lets the next kernel on the stream launch at once: when that kernel
  // is a programmatic dependent (the caller's overlap_previous), its CTAs take the
  // SMs this grid's last wave leaves idle. A grid launched that way waits for its
  // predecessor before any CTA exits, so it never completes first.
  if (threadIdx.x == 0) ptx::launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return base + SM_BAR + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + SM_ABORT);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sb + SM_TMEM_PTR);
  const Ctl ctl{abort_flag, p.status, p.wait_limit};
  // the map row and the status word are read while thread 0 sets up the barriers
  // and starts the Q copy, which needs neither
  const int e0 = p.row_ptr[qt];
  const int e1 = p.row_ptr[qt + 1];
  const int status0 = p.status ? *reinterpret_cast<volatile int32_t*>(p.status) : 0;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(BAR_Q + 0), 1);
    ptx::mbar_init(bar(BAR_Q + 1), 1);
    for (int i = 0; i < kSlots; ++i) {
      ptx::mbar_init(bar(BAR_FULL + i), 1);
      ptx::mbar_init(bar(BAR_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(BAR_S + i), 1);
      ptx::mbar_init(bar(BAR_P + i), 4);  // one arrival per softmax warp
      ptx::mbar_init(bar(BAR_O + i), 1);
    }
    ptx::mbar_init(bar(BAR_DRAIN), 1);
    ptx::mbar_init(bar(BAR_NEVER), 1);
    ptx::mbar_init(bar(BAR_QFREE), 1);
    ptx::mbar_init(bar(BAR_GATE), 1);
    ptx::mbar_init(bar(BAR_Q8), 1);
    ptx::mbar_init(bar(BAR_PH + 0), 4);  // one arrival per softmax warp
    ptx::mbar_init(bar(BAR_PH + 1), 4);
    for (int i = 0; i < 8; ++i) ptx::mbar_init(bar(BAR_EPI + i), 128);
    ptx::mbar_init(bar(BAR_QN + 0), 256);  // one arrival per softmax thread
    ptx::mbar_init(bar(BAR_QN + 1), 256);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
    // Q goes out first, before TMEM allocation and the CTA barrier: its latency
    // is the longest wait of a CTA's start. One barrier per head, so that head 0's
    // QK^T may start before head 1's Q has landed.
    const int nbox = p.d / 64, qr0 = tile_row0(qt, p);
    for (int i = 0; i < p.nh; ++i) {
      ptx::mbar_arrive_expect_tx(bar(BAR_Q + i), nbox * kBox);
      for (int x = 0; x < nbox; ++x)
        ptx::tma_load_4d(base + SM_Q + i * kTileBytes + x * kBox, &tm.q, bar(BAR_Q + i), x * 64, h0 + i, qr0, b);
    }
  }
  const int n = e1 - e0;
  if (n <= 0 ||  // a tile of padding slots only
      // fail fast: once any CTA of this launch (or an earlier one) has given up, do no work
      status0 != 0) {
    if (threadIdx.x == 0)  // the Q copies land before the CTA exits
      for (int i = 0; i < p.nh; ++i) wait_drain(bar(BAR_Q + i), 0);
    if (p.overlap_previous) ptx::wait_prerequisites();
    return;
  }
  if (threadIdx.x == 0) {
    // the first K and V tiles follow Q at once (slots 0 and 1); the producer warp
    // starts with the second map entry
    const int ent0 = p.entries[e0];
    const int nbox = p.d / 64, krow0 = tile_row0(ent0 >> 2, p);
    const uint32_t dk0 = base + SM_SLOT, dv0 = base + SM_SLOT + kTileBytes;
    if (ent0 & KREA_KIND_INT8) {
      ptx::mbar_arrive_expect_tx(bar(BAR_FULL + 0), kBox);
      ptx::tma_load_4d(dk0, &tm.k8, bar(BAR_FULL + 0), 0, g, krow0, b);
    } else {
      ptx::mbar_arrive_expect_tx(bar(BAR_FULL + 0), nbox * kBox);
      for (int x = 0; x < nbox; ++x) ptx::tma_load_4d(dk0 + x * kBox, &tm.k, bar(BAR_FULL + 0), x * 64, g, krow0, b);
    }
    ptx::mbar_arrive_expect_tx(bar(BAR_FULL + 1), nbox * kBox);
    for (int x = 0; x < nbox; ++x) ptx::tma_load_4d(dv0 + x * kBox, &tm.v, bar(BAR_FULL + 1), x * 64, g, krow0, b);
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_ptr), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int nh = p.nh;
  const int d = p.d;
  // Staged epilogue (gate prefetched by TMA, output written by TMA stores) when the
  // tile's physical rows are exactly its query rows and all lie in the slice:
  // no text padding inside the tile; rows past L are clipped by the TMA unit.
  const int qrow0 = tile_row0(qt, p);
  const int s0q = qt * kTile;
  // bf16 rows with at most kSplitMaxTiles key tiles: P to 16 bits (two PV terms)
  const bool split = BF16 && n <= kSplitMaxTiles;
  const bool staged = p.tma_out && ((s0q + kTile <= p.T) || (s0q >= p.Pt) || (p.T == p.Pt)) &&
                      qrow0 >= p.q_lo && min(qrow0 + kTile, p.L) <= p.q_hi;

  if (warp >= 8) {
  ptx::regs_dec<kOtherRegs>();  // the whole third warpgroup
  if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm.k);
      ptx::prefetch_tmap(&tm.v);
      const int nbox = d / 64;
      if (staged && p.has_gate)  // warm L2 with the gate tiles the epilogue will need
        for (int i = 0; i < nh; ++i)
          for (int x = 0; x < nbox; ++x) ptx::tma_prefetch_l2_4d(&tm.gate, x * 64, h0 + i, qrow0, b);
      uint32_t it = 2;  // K and V of the first entry: issued by thread 0
      for (int t = 1; t < n; ++t) {
        const int e = p.entries[e0 + t];
        const int krow0 = tile_row0(e >> 2, p);
        // K tile (INT8 codes for INT8 tiles)
        uint32_t slot = it % kSlots;
        if (!wait1(ctl, bar(BAR_EMPTY + slot), ((it / kSlots) & 1) ^ 1)) break;
        uint32_t dst = base + SM_SLOT + slot * kTileBytes;
        if (e & KREA_KIND_INT8) {
          ptx::mbar_arrive_expect_tx(bar(BAR_FULL + slot), kBox);
          ptx::tma_load_4d(dst, &tm.k8, bar(BAR_FULL + slot), 0, g, krow0, b);
        } else {
          ptx::mbar_arrive_expect_tx(bar(BAR_FULL + slot), nbox * kBox);
          for (int x = 0; x < nbox; ++x)
            ptx::tma_load_4d(dst + x * kBox, &tm.k, bar(BAR_FULL + slot), x * 64, g, krow0, b);
        }
        ++it;
        // V tile
        slot = it % kSlots;
        if (!wait1(ctl, bar(BAR_EMPTY + slot), ((it / kSlots) & 1) ^ 1)) break;
        dst = base + SM_SLOT + slot * kTileBytes;
        ptx::mbar_arrive_expect_tx(bar(BAR_FULL + slot), nbox * kBox);
        for (int x = 0; x < nbox; ++x)
          ptx::tma_load_4d(dst + x * kBox, &tm.v, bar(BAR_FULL + slot), x * 64, g, krow0, b);
        ++it;
      }
      // gate tiles of the staged epilogue go into the Q area once the last QK^T is done
      bool gate_issued = false;
      if (staged && p.has_gate && it == 2u * (uint32_t)n && wait1(ctl, bar(BAR_QFREE), 0)) {
        ptx::mbar_arrive_expect_tx(bar(BAR_GATE), nh * nbox * kBox);
        for (int i = 0; i < nh; ++i)
          for (int x = 0; x < nbox; ++x)
            ptx::tma_load_4d(base + SM_Q + i * kTileBytes + x * kBox, &tm.gate, bar(BAR_GATE), x * 64, h0 + i,
                             qrow0, b);
        gate_issued = true;
      }
      // Every copy this thread started lands before the CTA may exit (already
      // true on the normal path, where the MMA thread consumed them all).
      for (int i = 0; i < nh; ++i) wait_drain(bar(BAR_Q + i), 0);  // thread 0 issued them
      if (gate_issued) wait_drain(bar(BAR_GATE), 0);
      for (uint32_t j = (it > kSlots ? it - kSlots : 0); j < it; ++j)
        wait_drain(bar(BAR_FULL + j % kSlots), (j / kSlots) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      if (d == 128) mma_thread<BF16, 128>(p, base, tmem, e0, n, nh, ctl, split);
      else mma_thread<BF16, 64>(p, base, tmem, e0, n, nh, ctl, split);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------- INT8 query codes
    // Off the producer's path: scanning the row's map entries would delay Q and K_0.
    if (lane == 0) {
      bool has_int8 = false;
      for (int t = 0; t < n; ++t) has_int8 |= (p.entries[e0 + t] & KREA_KIND_INT8) != 0;
      if (has_int8) {
        ptx::prefetch_tmap(&tm.q8);
        ptx::mbar_arrive_expect_tx(bar(BAR_Q8), nh * kBox);
        for (int i = 0; i < nh; ++i)
          ptx::tma_load_4d(base + SM_Q8 + i * kBox, &tm.q8, bar(BAR_Q8), 0, h0 + i, qrow0, b);
        wait_drain(bar(BAR_Q8), 0);  // the copy lands before the CTA may exit
      }
    }
  }
  } else {
    // ------------------------------------------------------------- softmax
    ptx::regs_inc<kSoftmaxRegs>();
    const int wg = warp >> 2, wq = warp & 3;
    bool q_ok = true;
    if (p.q_rope) {  // the QK prologue on the raw Q tiles, head by head, all 256 threads
      auto run = [&](auto& rq) {
        rq.load_table(qrow0, (int)threadIdx.x, p);
        for (int i = 0; i < nh; ++i) {
          if (q_ok) q_ok = wait_warp(ctl, bar(BAR_Q + i), 0);
          if (q_ok) rq.apply(base + SM_Q + (uint32_t)i * kTileBytes, qrow0, p);
          ptx::fence_proxy_async_smem();  // the rows are read by the tensor core next
          ptx::mbar_arrive(bar(BAR_QN + i));
        }
      };
      if (d == 128) {
        RopeQ<BF16, 128> rq;
        run(rq);
      } else {
        RopeQ<BF16, 64> rq;
        run(rq);
      }
    }
    if (wg < nh) {
      const int h = h0 + wg;
      const int row = wq * 32 + lane;
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      const uint32_t tS = tmem + lane_base + (uint32_t)wg * 128u;
      const uint32_t tO = tmem + lane_base + 256u + (uint32_t)wg * 128u;
      const int qs = qt * kTile + row;  // logical slot of this query row
      const int phys_q = qs < p.T ? qs : (qs < p.Pt ? -1 : (qs < p.Pt + p.N ? qs - p.Pt + p.T : -1));
      const bool q_valid = phys_q >= 0 && phys_q >= p.q_lo && phys_q < p.q_hi;
      // key slots this row admits beyond the text: [klo, khi)
      int klo = p.Pt, khi = p.Pt + p.N;
      if (!p.tile_aligned && phys_q >= p.T) {
        const int r = (qs - p.Pt) / p.W;
        klo = p.Pt + max(0, r - p.window_half) * p.W;
        khi = p.Pt + min(p.H, r + p.window_half + 1) * p.W;
      }
      const float sq_row = p.sq ? p.sq[((long long)b * p.Hq + h) * p.nt_scale + qt] : 0.f;
      const float* sk_row = p.sk ? p.sk + ((long long)b * p.Hkv + g) * p.nt_scale : nullptr;
      bool ok = q_ok;
      float m = kNegInf, l = 0.f;
      if ((p.debug_flags & 1) && wg == 0 && wq == 0) ok = wait_warp(ctl, bar(BAR_NEVER), 0);
      // map entries are read two tiles ahead and an INT8 tile's key-block scale one
      // tile ahead, so that neither load waits behind the S barrier
      auto sk_of = [&](int e) { return (sk_row && (e & KREA_KIND_INT8)) ? sk_row[e >> 2] : 0.f; };
      int e_cur = p.entries[e0];
      int e_nxt = n > 1 ? p.entries[e0 + 1] : 0;
      float sk_cur = sk_of(e_cur);
      for (int t = 0; t < n && ok; ++t) {
        const int e = e_cur;
        const float sk_e = sk_cur;
        if (t + 1 < n) {
          sk_cur = sk_of(e_nxt);
          e_cur = e_nxt;
        }
        if (t + 2 < n) e_nxt = p.entries[e0 + t + 2];
        const int kb = e >> 2;
        ok = wait_warp(ctl, bar(BAR_S + wg), t & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        uint32_t v[128];
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 2; ++j) ptx::tmem_ld64(tS + 64u * j, *reinterpret_cast<uint32_t(*)[64]>(&v[64 * j]));
        ptx::tmem_wait_ld();
        const int kind = e & 3;
        // log2-unit score scale; INT8 tiles also carry both block scales (a zero
        // scale means an all-zero block: any positive multiplier gives score 0)
        const float mult = (kind & KREA_KIND_INT8) ? fmaxf(p.scale_log2 * sq_row * sk_e, 1e-30f) : p.scale_log2;
        // admitted key columns of this tile: [0, a1) text, [a2, a3) image window
        const int s0 = kb * kTile;
        const int a1 = p.T - s0, a2 = klo - s0, a3 = khi - s0;
        const bool first = t == 0;
        const uint32_t hb = bar(BAR_PH + wg);
        if (BF16 && split) {
          if (kind == 0) softmax_tile<BF16, false, false, ALL_POLY, BF16>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else if (kind == 1) softmax_tile<BF16, false, true, ALL_POLY, BF16>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else if (kind == 2) softmax_tile<BF16, true, false, ALL_POLY, BF16>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else softmax_tile<BF16, true, true, ALL_POLY, BF16>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
        } else {
          if (kind == 0) softmax_tile<BF16, false, false, ALL_POLY, false>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else if (kind == 1) softmax_tile<BF16, false, true, ALL_POLY, false>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else if (kind == 2) softmax_tile<BF16, true, false, ALL_POLY, false>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
          else softmax_tile<BF16, true, true, ALL_POLY, false>(v, mult, a1, a2, a3, m, l, first, tS, tO, d, hb);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(BAR_P + wg));
      }
      if (ok) ok = wait_warp(ctl, bar(BAR_O + wg), 0);
      if (ok && staged && p.has_gate) ok = wait_warp(ctl, bar(BAR_GATE), 0);
      if (ok && p.lse && q_valid)  // the softmax normaliser, natural log: (m + log2 l) ln 2
        p.lse[((long long)b * p.Hq + h) * p.L + phys_q] = (m + log2f(l)) * 0.69314718055994531f;
      if (ok && staged) {
        // Staged epilogue: the gate row comes from the Q area (TMA-loaded, 64 values per
        // 128-byte swizzled row), out = O / l * sigmoid(gate) goes to free K/V slots in
        // the 128-byte swizzled layout of the out map, then one thread stores by TMA.
        // Head 0 may start while head 1's last PV still reads V, which sits in an odd
        // slot (the producer fills K, V, K, V, ...): head 0 stages only in even slots.
        // Output box x (32 fp32 or 64 16-bit columns, 16 KB) of head wg sits in slot
        // 2 (x / 2) + wg, at offset (x % 2) * 16 KB.
        ptx::tc_fence_after();
        const float inv_l = 1.0f / l;
        const uint32_t gbase = SM_Q + (uint32_t)wg * kTileBytes;
        auto stage = [&](int x) {
          return SM_SLOT + (uint32_t)(2 * (x >> 1) + wg) * kTileBytes + (uint32_t)(x & 1) * kBox;
        };
        const uint32_t rsw = (uint32_t)(row & 7), rofs = (uint32_t)row * 128u;
        for (int j = 0; j < d / 32; ++j) {
          uint32_t o[32];
          __syncwarp();
          ptx::tmem_ld32(tO + 32u * j, o);
          ptx::tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) y[c] = __uint_as_float(o[c]) * inv_l;
          if (p.has_gate) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {  // columns 32j + 8v ..: box j/2, 16-byte piece (j%2)*4 + v
              const uint32_t q = (uint32_t)((j & 1) * 4 + v);
              const uint4 u = *reinterpret_cast<const uint4*>(sb + gbase + (uint32_t)(j >> 1) * kBox + rofs +
                                                               ((q ^ rsw) << 4));
              const uint16_t* ge = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
              for (int c = 0; c < 8; ++c) y[8 * v + c] *= sigmoidf_(h2f<BF16>(ge[c]));
            }
          }
          if (p.out_f32) {
#pragma unroll
            for (int v = 0; v < 8; ++v)  // box j holds columns 32j .. 32j+31
              *reinterpret_cast<float4*>(sb + stage(j) + rofs + (((uint32_t)v ^ rsw) << 4)) =
                  make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v) {  // box j/2 holds columns 64(j/2) ..; piece (j%2)*4 + v
              const uint32_t q = (uint32_t)((j & 1) * 4 + v);
              *reinterpret_cast<uint4*>(sb + stage(j >> 1) + rofs + ((q ^ rsw) << 4)) =
                  make_uint4(pack2<BF16>(y[8 * v], y[8 * v + 1]), pack2<BF16>(y[8 * v + 2], y[8 * v + 3]),
                             pack2<BF16>(y[8 * v + 4], y[8 * v + 5]), pack2<BF16>(y[8 * v + 6], y[8 * v + 7]));
            }
          }
          // Box x (32 fp32 or 64 16-bit columns) is stored as soon as its 128 rows are
          // staged, so the stores overlap the remaining columns' work.
          if (p.out_f32 || (j & 1)) {
            const int x = p.out_f32 ? j : (j >> 1);
            ptx::fence_proxy_async_smem();  // make the rows visible to the TMA unit
            ptx::mbar_arrive(bar(BAR_EPI + 4 * wg + x));
            if (wq == 0 && lane == 0 && wait1(ctl, bar(BAR_EPI + 4 * wg + x), 0)) {
              ptx::tma_store_4d(&tm.out, base + stage(x), x * (p.out_f32 ? 32 : 64), h, qrow0, b);
              ptx::bulk_commit();
            }
          }
        }
        if (wq == 0 && lane == 0) ptx::bulk_wait_read0();  // shared memory must outlive the stores' reads
      } else if (ok) {
        ptx::tc_fence_after();
        const float inv_l = 1.0f / l;
        const long long tok = q_valid ? phys_q : 0;
        const uint16_t* grow =
            p.has_gate ? static_cast<const uint16_t*>(p.gate) + b * p.gate_stride[0] + tok * p.gate_stride[1] +
                             (long long)h * p.gate_stride[2]
                       : nullptr;
        for (int j = 0; j < d / 32; ++j) {
          uint32_t o[32];
          __syncwarp();
          ptx::tmem_ld32(tO + 32u * j, o);
          ptx::tmem_wait_ld();
          if (!q_valid) continue;
          float y[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) y[c] = __uint_as_float(o[c]) * inv_l;
          if (grow) {
            const uint4* gp = reinterpret_cast<const uint4*>(grow + 32 * j);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 u = gp[v];
              const uint16_t* ge = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
              for (int c = 0; c < 8; ++c) y[8 * v + c] *= sigmoidf_(h2f<BF16>(ge[c]));
            }
          }
          if (p.out_f32) {
            float4* op = reinterpret_cast<float4*>(static_cast<float*>(p.out) + b * p.out_stride[0] +
                                                   tok * p.out_stride[1] + (long long)h * p.out_stride[2] + 32 * j);
#pragma unroll
            for (int v = 0; v < 8; ++v) op[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
          } else {
            uint4* op = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + b * p.out_stride[0] +
                                                 tok * p.out_stride[1] + (long long)h * p.out_stride[2] + 32 * j);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              op[v] = make_uint4(pack2<BF16>(y[8 * v], y[8 * v + 1]), pack2<BF16>(y[8 * v + 2], y[8 * v + 3]),
                                 pack2<BF16>(y[8 * v + 4], y[8 * v + 5]), pack2<BF16>(y[8 * v + 6], y[8 * v + 7]));
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, 512);
  if (p.overlap_previous && threadIdx.x == 0) ptx::wait_prerequisites();
}

// ALL_POLY = true sends every exponential through exp2_poly2 (tests of its accuracy).
template <bool BF16, bool ALL_POLY>
int launch(const AttnDevParams& p, const AttnMaps& maps, cudaStream_t s) {
  static int checked = 0;  // 1 = the kernel has the register count the setmaxnreg split needs
  if (!checked) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_fwd_kernel<BF16, ALL_POLY>) != cudaSuccess) return KREA_ERR_CUDA;
    checked = (fa.numRegs == kLaunchRegs) ? 1 : -1;
  }
  if (checked != 1) return KREA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(attn_fwd_kernel<BF16, ALL_POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_ALLOC) != cudaSuccess)
    return KREA_ERR_CUDA;
  const long long grid = (long long)p.B * p.Hkv * p.npairs * p.n_slice_tiles;
  if (grid <= 0 || grid > 0x7fffffffLL) return KREA_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.overlap_previous ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, attn_fwd_kernel<BF16, ALL_POLY>, maps, p) != cudaSuccess) return KREA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace

int launch_attention(const AttnDevParams& p, const AttnMaps& maps, bool bf16, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.debug_flags & 2) return bf16 ? launch<true, true>(p, maps, s) : launch<false, true>(p, maps, s);
  return bf16 ? launch<true, false>(p, maps, s) : launch<false, false>(p, maps, s);
}

}  // namespace krea
