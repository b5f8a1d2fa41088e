// Backward of the Krea 2 attention core (dense and scanline; FP16/BF16 tiles).
//
// With P the softmax weights over the admitted keys (recomputed from the
// forward's log-sum-exp), O = P V before the gate and out = sigmoid(g) O:
//   dO = dout sigmoid(g),  D_i = sum_c dout_ic out_ic = dO_i . O_i,
//   dgate = dout out (1 - sigmoid(g)),
//   dP = dO V^T,  dS = P (dP - D),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K,
// dK and dV summed over the query heads that share a kv head.
//
// bwd_prep_kernel: dO (input dtype), D and dgate, one pass over out / dout.
// bwd_kernel: one CTA per (batch, kv head, key tile j), 320 threads:
//   warps 0-7  warp w: TMEM lanes 32 (w % 4) .. (query rows of the current query
//              tile, key rows of tile j at the end) and key / head-dim columns
//              [64 (w / 4), + 64): P and dS need no row-wide reduction (the
//              forward's lse and D are per-row constants), so the two warps of a
//              row work independently
//   warp  8    TMA producer: K_j and V_j once, then Q_i, dO_i per step (as soon
//              as dV and dK of the previous step have read them)
//   warp  9    TMEM allocator and the thread issuing every tcgen05.mma
// A step is one (query head, query tile i) of the key tile's map row (the
// scanline rule is symmetric, so row j lists the query tiles that see tile j):
//   S = Q_i K_j^T, dP = dO_i V_j^T                 (TMEM columns 0..127, 128..255)
//   softmax warps: P = exp2(S scale log2e - lse log2e) on admitted pairs, dS;
//                  both stored row-major over keys in 128-byte-swizzled shared
//                  tiles (the layout TMA gives a [rows][64-element] box)
//   dV += P^T dO_i, dK += dS^T Q_i                  (TMEM 256..383, 384..511: the P
//                  and dS tiles read as MN-major A operands, Q and dO as MN-major B)
//   dQ_i part = dS K_j                              (TMEM 128..255, dS as K-major A),
//                  followed at once by the next step's S: only its dP waits for
//                  the softmax warps to read the dQ part out
//   P is stored and released before dS, so that dV runs while dS still waits for
//   the TMA unit to finish reading the previous step's staged dQ in its area
//   softmax warps stage scale * dQ part in shared memory (where P and dS were) and
//   one thread adds it into the fp32 dq buffer with TMA reduce-adds, so the
//   additions leave the softmax warps' path.
// Every barrier wait is bounded as in the forward kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "krea_internal.h"
#include "ptx_sm100.cuh"

namespace krea {
namespace {

constexpr int kBThreads = 320;
constexpr uint32_t kBBox = 16384;        // 128 rows x 128 bytes
// Q in two buffers (step s uses Q buffer s % 2, so the next step's Q loads while
// this step's dK still reads its own)
constexpr uint32_t BS_K = 0, BS_V = 32768, BS_Q = 65536, BS_DO = 131072, BS_P = 163840, BS_DS = 196608;
// the dQ part of a step is staged for its TMA reduce-add where P and dS were (their
// MMAs are done by then): fp32 box c (32 columns x 128 rows, 16 KB) at BS_P + c * 16 KB
constexpr uint32_t BS_DQ = BS_P;
constexpr uint32_t BS_BAR = BS_DS + 32768;
enum {
  BB_KV = 0,
  BB_QF,           // 2: Q of a step landed in buffer s % 2
  BB_DOF = BB_QF + 2,  // dO of a step landed
  BB_SDP,
  BB_PRDY,         // P of a step is in shared memory (dV may start)
  BB_DSRDY,        // dS of a step is in shared memory (dK, dQ may start)
  BB_GRAD,
  BB_SFREE,        // the dQ part of a step has been read out of TMEM
  BB_DRAIN,
  BB_QFREE,        // 2: dK of a step has read Q buffer s % 2
  BB_DOFREE = BB_QFREE + 2,  // dV of a step has read dO
  BB_DQ,
  BB_STAGEDP,      // the TMA unit has read the staged dQ boxes in the P area
  BB_STAGEDDS,     // ... and those in the dS area
  BB_N
};
constexpr uint32_t BS_TMEM = BS_BAR + 8 * BB_N;
constexpr uint32_t BS_ABORT = BS_TMEM + 4;
constexpr uint32_t B_SMEM_ALLOC = BS_BAR + 256 + 1024;  // + slack to align the base to 1024
static_assert(BS_ABORT + 4 <= BS_BAR + 256, "barrier block");
static_assert(B_SMEM_ALLOC <= 232448, "shared memory budget");
constexpr long long kBDrain = 4000000000LL;

struct BCtl {
  volatile int* abort;
  int32_t* status;
  long long limit;
};

__device__ __forceinline__ void b_timeout(const BCtl& c) {
  *c.abort = 1;
  if (c.status) atomicCAS(c.status, 0, KREA_ERR_DEVICE_TIMEOUT);
}

__device__ __forceinline__ bool b_wait1(const BCtl& c, uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (*c.abort) return false;
    if (clock64() - t0 > c.limit) {
      b_timeout(c);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool b_wait_warp(const BCtl& c, uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    const bool done = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    const bool stop = *c.abort || (clock64() - t0 > c.limit);
    if (__any_sync(0xffffffffu, stop)) {
      if ((threadIdx.x & 31) == 0 && !*c.abort) b_timeout(c);
      return false;
    }
  }
}

__device__ __forceinline__ void b_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kBDrain) return;
}

// Physical token of logical slot s (-1: padding).
__device__ __forceinline__ int b_phys(int s, const BwdDevParams& p) {
  if (s < p.T) return s;
  if (s < p.Pt) return -1;
  if (s < p.Pt + p.N) return s - p.Pt + p.T;
  return -1;
}

// First physical row of logical tile `tile` (text slots map to themselves, image
// slots start at Pt).
__device__ __forceinline__ int b_row0(int tile, const BwdDevParams& p) {
  const int s0 = tile * kTile;
  return s0 < p.Pt ? s0 : s0 - p.Pt + p.T;
}

template <bool BF16>
__device__ __forceinline__ uint32_t b_pack(float lo, float hi) {
  if constexpr (BF16) return ptx::pack_bf16(lo, hi);
  else return ptx::pack_f16(lo, hi);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

template <bool BF16>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_kernel(const __grid_constant__ BwdMaps tm, const __grid_constant__ BwdDevParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sb = smem_raw + (base - raw);
  const int j = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int e0 = p.row_ptr[j];
  const int n = p.row_ptr[j + 1] - e0;
  if (n <= 0) return;
  if (p.status && *reinterpret_cast<volatile int32_t*>(p.status) != 0) return;
  const int nsteps = n * p.rep;  // step s: query head g * rep + s / n, map entry s % n

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return base + BS_BAR + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + BS_ABORT);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sb + BS_TMEM);
  const BCtl ctl{abort_flag, p.status, p.wait_limit};
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(BB_KV), 1);
    ptx::mbar_init(bar(BB_QF + 0), 1);
    ptx::mbar_init(bar(BB_QF + 1), 1);
    ptx::mbar_init(bar(BB_DOF), 1);
    ptx::mbar_init(bar(BB_SDP), 1);
    ptx::mbar_init(bar(BB_PRDY), 8);
    ptx::mbar_init(bar(BB_DSRDY), 8);
    ptx::mbar_init(bar(BB_GRAD), 1);
    ptx::mbar_init(bar(BB_SFREE), 8);
    ptx::mbar_init(bar(BB_DRAIN), 1);
    ptx::mbar_init(bar(BB_QFREE + 0), 1);
    ptx::mbar_init(bar(BB_QFREE + 1), 1);
    ptx::mbar_init(bar(BB_DOFREE), 1);
    ptx::mbar_init(bar(BB_DQ), 8);       // every softmax warp staged its dQ rows
    ptx::mbar_init(bar(BB_STAGEDP), 1);  // the staged dQ has been read by the TMA unit:
    ptx::mbar_init(bar(BB_STAGEDDS), 1); // the P area's boxes, then the dS area's
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_ptr), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int d = p.d;
  const int nbox = d / 64;

  if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      const int krow0 = b_row0(j, p);
      ptx::mbar_arrive_expect_tx(bar(BB_KV), 2 * nbox * kBBox);
      for (int x = 0; x < nbox; ++x) {
        ptx::tma_load_4d(base + BS_K + x * kBBox, &tm.k, bar(BB_KV), x * 64, g, krow0, b);
        ptx::tma_load_4d(base + BS_V + x * kBBox, &tm.v, bar(BB_KV), x * 64, g, krow0, b);
      }
      int nq = 0, nd = 0;  // Q and dO copies issued
      for (int s = 0; s < nsteps; ++s) {
        const uint32_t qb = (uint32_t)s & 1u;
        // Q of step s into buffer s % 2, once dK of step s - 2 has read it
        if (s >= 2 && !b_wait1(ctl, bar(BB_QFREE + qb), ((s >> 1) - 1) & 1)) break;
        const int h = g * p.rep + s / n;
        const int qrow0 = b_row0(p.entries[e0 + s % n] >> 2, p);
        ptx::mbar_arrive_expect_tx(bar(BB_QF + qb), nbox * kBBox);
        for (int x = 0; x < nbox; ++x)
          ptx::tma_load_4d(base + BS_Q + qb * 32768u + x * kBBox, &tm.q, bar(BB_QF + qb), x * 64, h, qrow0, b);
        ++nq;
        // dO of step s, once dV of step s - 1 has read dO
        if (s >= 1 && !b_wait1(ctl, bar(BB_DOFREE), (s - 1) & 1)) break;
        ptx::mbar_arrive_expect_tx(bar(BB_DOF), nbox * kBBox);
        for (int x = 0; x < nbox; ++x)
          ptx::tma_load_4d(base + BS_DO + x * kBBox, &tm.dout, bar(BB_DOF), x * 64, h, qrow0, b);
        ++nd;
      }
      // every copy this thread started lands before the CTA may exit
      b_drain(bar(BB_KV), 0);
      for (int t = (nq > 2 ? nq - 2 : 0); t < nq; ++t) b_drain(bar(BB_QF + (t & 1)), (t >> 1) & 1);
      if (nd > 0) b_drain(bar(BB_DOF), (nd - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ab = BF16 ? 1u : 0u;
      const uint32_t ID_KK = ptx::idesc(1, ab, 0, 0, 128, 128);   // S, dP: A, B K-major
      const uint32_t ID_MM = ptx::idesc(1, ab, 1, 1, (uint32_t)d, 128);  // dV, dK: A, B MN-major
      const uint32_t ID_KM = ptx::idesc(1, ab, 0, 1, (uint32_t)d, 128);  // dQ: A K-major, B MN-major
      constexpr uint32_t kb4 = kBBox >> 4;
      const uint32_t dK_ = ptx::sdesc_lo(base + BS_K, 16), dV_ = ptx::sdesc_lo(base + BS_V, 16);
      const uint32_t dQ_ = ptx::sdesc_lo(base + BS_Q, 16), dO_ = ptx::sdesc_lo(base + BS_DO, 16);
      const uint32_t dS_k = ptx::sdesc_lo(base + BS_DS, 16);
      const uint32_t mP = ptx::sdesc_lo(base + BS_P, kBBox), mDS = ptx::sdesc_lo(base + BS_DS, kBBox);
      const uint32_t mDO = ptx::sdesc_lo(base + BS_DO, kBBox), mQ = ptx::sdesc_lo(base + BS_Q, kBBox);
      const uint32_t mK = ptx::sdesc_lo(base + BS_K, kBBox);
      auto qk = [&](int s) {  // S = Q K^T of step s into columns 0..127, K = head dim
        const uint32_t qoff = ((uint32_t)s & 1u) * (32768u >> 4);
        for (int k = 0; k < d / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * kb4 + (uint32_t)(k & 3) * 2u;
          ptx::mma_f16_ss_lo(tmem, dQ_ + qoff + off, dK_ + off, ID_KK, k > 0);
        }
      };
      bool ok = b_wait1(ctl, bar(BB_KV), 0) && b_wait1(ctl, bar(BB_QF + 0), 0);
      if (ok) {
        ptx::tc_fence_after();
        qk(0);
      }
      for (int s = 0; s < nsteps && ok; ++s) {
        const uint32_t qb = (uint32_t)s & 1u, qoff = qb * (32768u >> 4);  // Q buffer of this step
        // dP goes where the previous step's dQ part was: once the softmax warps read it
        if (s > 0) ok = b_wait1(ctl, bar(BB_SFREE), (s - 1) & 1);
        if (ok) ok = b_wait1(ctl, bar(BB_DOF), s & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int k = 0; k < d / 16; ++k) {  // dP = dO V^T
          const uint32_t off = (uint32_t)(k >> 2) * kb4 + (uint32_t)(k & 3) * 2u;
          ptx::mma_f16_ss_lo(tmem + 128u, dO_ + off, dV_ + off, ID_KK, k > 0);
        }
        ptx::tc_commit(bar(BB_SDP));
        ok = b_wait1(ctl, bar(BB_PRDY), s & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int k = 0; k < 8; ++k) {  // K = 128 query rows, 16 (2 KB of a tile) per step
          const uint32_t acc = (s > 0 || k > 0) ? 1u : 0u;
          ptx::mma_f16_ss_lo(tmem + 256u, mP + 128u * k, mDO + 128u * k, ID_MM, acc);   // dV += P^T dO
        }
        ptx::tc_commit(bar(BB_DOFREE));  // the next step's dO may load
        ok = b_wait1(ctl, bar(BB_DSRDY), s & 1);  // dS lands while dV runs
        if (!ok) break;
        ptx::tc_fence_after();
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (s > 0 || k > 0) ? 1u : 0u;
          ptx::mma_f16_ss_lo(tmem + 384u, mDS + 128u * k, mQ + qoff + 128u * k, ID_MM, acc);  // dK += dS^T Q
        }
        ptx::tc_commit(bar(BB_QFREE + qb));  // this Q buffer may take step s + 2's Q
        for (int k = 0; k < 8; ++k) {  // dQ part = dS K_j into columns 128..255, K = 128 keys
          const uint32_t off = (uint32_t)(k >> 2) * kb4 + (uint32_t)(k & 3) * 2u;
          ptx::mma_f16_ss_lo(tmem + 128u, dS_k + off, mK + 128u * k, ID_KM, k > 0);
        }
        ptx::tc_commit(bar(BB_GRAD));
        // the next step's S right behind it: S and dP of this step were consumed before
        // its P and dS were released, and the softmax warps read the dQ part meanwhile
        if (s + 1 < nsteps) {
          ok = b_wait1(ctl, bar(BB_QF + (qb ^ 1u)), ((s + 1) >> 1) & 1);
          if (!ok) break;
          ptx::tc_fence_after();
          qk(s + 1);
        }
      }
      ptx::tc_commit(bar(BB_DRAIN));
      b_drain(bar(BB_DRAIN), 0);
    }
  } else {
    // ------------------------------------------------------------- softmax warps
    const int wq = warp & 3, hf = warp >> 2, row = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base, tP = tS + 128u, tdV = tS + 256u, tdK = tS + 384u;
    const uint32_t rsw = (uint32_t)(row & 7), rofs = (uint32_t)row * 128u;
    const int hd0 = hf * (d / 2);  // this warp's head-dim columns of dQ, dK, dV: [hd0, hd0 + d/2)
    const bool issuer = warp == 0 && lane == 0;  // issues the dQ reduce-adds
    // Every key slot of tile j is a valid token and, with the tile-aligned rule, every
    // valid query row of a listed query tile admits all of them: P needs no per-key
    // predicate (padding query rows have lse = +inf, so their P is 0 anyway).
    const int kj0 = j * kTile;
    const bool kfull = p.tile_aligned && ((kj0 + kTile <= p.T) || (kj0 >= p.Pt && kj0 + kTile <= p.Pt + p.N));
    bool ok = true;
    for (int s = 0; s < nsteps && ok; ++s) {
      const int hh = s / n, h = g * p.rep + hh;
      const int i = p.entries[e0 + s % n] >> 2;
      const int qs = i * kTile + row;
      const int phys_q = b_phys(qs, p);
      const bool q_valid = phys_q >= 0;
      int klo = p.Pt, khi = p.Pt + p.N;  // image keys this row admits
      if (!p.tile_aligned && phys_q >= p.T) {
        const int r = (qs - p.Pt) / p.W;
        klo = p.Pt + max(0, r - p.window_half) * p.W;
        khi = p.Pt + min(p.H, r + p.window_half + 1) * p.W;
      }
      const long long rix = ((long long)b * p.Hq + h) * p.L + (q_valid ? phys_q : 0);
      const float lse2 = q_valid ? p.lse[rix] * 1.4426950408889634f : INFINITY;
      const float Dr = q_valid ? p.D[rix] : 0.f;
      ok = b_wait_warp(ctl, bar(BB_SDP), s & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      // P and dS go where the previous step's dQ was staged, each once the TMA unit
      // has read the boxes in its area: the P area's boxes form the older bulk group
      auto staged = [&](bool ds_area) {
        if (s == 0) return true;
        if (issuer) {
          if (ds_area || d == 64) ptx::bulk_wait_read0();
          else ptx::bulk_wait_read1();
          ptx::mbar_arrive(bar(ds_area ? BB_STAGEDDS : BB_STAGEDP));
        }
        return b_wait_warp(ctl, bar(ds_area ? BB_STAGEDDS : BB_STAGEDP), (s - 1) & 1);
      };
      // P first, so that dV starts while dS waits for its area
      auto ready = [&](int bb) {
        ptx::fence_proxy_async_smem();  // the tensor core reads the tile next
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bb));
      };
      if (kfull) {  // keys 64 hf .. + 63 of S and dP -> P and dS, packed pairs, no predicate
        uint32_t sv[64], dp[64];
        __syncwarp();
#pragma unroll
        for (int ck = 0; ck < 2; ++ck) {
          ptx::tmem_ld32(tS + 64u * hf + 32u * ck, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * ck]));
          ptx::tmem_ld32(tP + 64u * hf + 32u * ck, *reinterpret_cast<uint32_t(*)[32]>(&dp[32 * ck]));
        }
        ptx::tmem_wait_ld();
        const uint64_t sc2 = ptx::f2(p.scale_log2, p.scale_log2), nl2 = ptx::f2(-lse2, -lse2);
        const uint64_t nd2 = ptx::f2(-Dr, -Dr);
        uint32_t pw[8][4], dw[8][4];  // all of the warp's P and dS first: the exponentials
                                      // overlap the TMA unit's read of the staged dQ
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {  // 8 keys = 16 bytes of P and of dS
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = 8 * pc + 2 * u;
            float x0, x1;
            ptx::unf2(ptx::fma2(ptx::f2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc2, nl2), x0, x1);
            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
            const uint64_t pp = ptx::f2(p0, p1);
            const uint64_t dd =
                ptx::mul2(pp, ptx::add2(ptx::f2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nd2));
            float d0, d1;
            ptx::unf2(dd, d0, d1);
            pw[pc][u] = b_pack<BF16>(p0, p1);
            dw[pc][u] = b_pack<BF16>(d0, d1);
          }
        }
        ok = staged(false);
        if (!ok) break;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          const uint32_t at = (uint32_t)hf * kBBox + rofs + (((uint32_t)pc ^ rsw) << 4);
          ptx::sts128(base + BS_P + at, make_uint4(pw[pc][0], pw[pc][1], pw[pc][2], pw[pc][3]));
        }
        ready(BB_PRDY);
        ok = staged(true);
        if (!ok) break;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          const uint32_t at = (uint32_t)hf * kBBox + rofs + (((uint32_t)pc ^ rsw) << 4);
          ptx::sts128(base + BS_DS + at, make_uint4(dw[pc][0], dw[pc][1], dw[pc][2], dw[pc][3]));
        }
        ready(BB_DSRDY);
      } else {
      ok = staged(false) && staged(true);
      if (!ok) break;
      for (int ck = 0; ck < 2; ++ck) {  // keys 64 hf + 32 ck .. + 31 of S and dP -> P and dS
        uint32_t sv[32], dp[32];
        __syncwarp();
        ptx::tmem_ld32(tS + 64u * hf + 32u * ck, sv);
        ptx::tmem_ld32(tP + 64u * hf + 32u * ck, dp);
        ptx::tmem_wait_ld();
        const int ks0 = j * kTile + 64 * hf + 32 * ck;  // logical slot of the chunk's first key
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {  // 8 keys = 16 bytes of P and of dS
          uint32_t pw[4], dw[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float pr[2], dr[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = pc * 8 + 2 * u + e;
              const int ks = ks0 + c;
              const bool adm = q_valid && (ks < p.T || (ks >= klo && ks < khi));
              const float pv = adm ? ptx::ex2(__uint_as_float(sv[c]) * p.scale_log2 - lse2) : 0.f;
              pr[e] = pv;
              dr[e] = pv * (__uint_as_float(dp[c]) - Dr);
            }
            pw[u] = b_pack<BF16>(pr[0], pr[1]);
            dw[u] = b_pack<BF16>(dr[0], dr[1]);
          }
          const uint32_t piece = (uint32_t)(4 * ck + pc);  // 16-byte piece of the 128-byte row
          const uint32_t at = (uint32_t)hf * kBBox + rofs + ((piece ^ rsw) << 4);
          *reinterpret_cast<uint4*>(sb + BS_P + at) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4*>(sb + BS_DS + at) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
        }
      }
      ready(BB_PRDY);
      ready(BB_DSRDY);
      }
      ok = b_wait_warp(ctl, bar(BB_GRAD), s & 1);
      if (!ok) break;
      ptx::tc_fence_after();
      // this warp's half of the dQ row into registers, free the TMEM columns, stage
      // it (scaled) in the 128-byte-swizzled layout of the dq map's 32-column boxes,
      // then one thread adds the whole tile into dq by TMA. Rows of padding slots
      // are exact zeros (their P is 0), so adding them to whatever token the box
      // covers there changes nothing.
      uint32_t dqv[64];
      __syncwarp();
      ptx::tmem_ld32(tP + (uint32_t)hd0, *reinterpret_cast<uint32_t(*)[32]>(&dqv[0]));
      if (d == 128) ptx::tmem_ld32(tP + (uint32_t)hd0 + 32u, *reinterpret_cast<uint32_t(*)[32]>(&dqv[32]));
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(BB_SFREE));
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {  // boxes hd0 / 32 + c2
        if (c2 >= d / 64) break;
        const uint32_t box = base + BS_DQ + (uint32_t)(hd0 / 32 + c2) * kBBox;
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          ptx::sts128(box + rofs + (((uint32_t)v4 ^ rsw) << 4),
                      make_uint4(__float_as_uint(__uint_as_float(dqv[32 * c2 + 4 * v4]) * p.scale),
                                 __float_as_uint(__uint_as_float(dqv[32 * c2 + 4 * v4 + 1]) * p.scale),
                                 __float_as_uint(__uint_as_float(dqv[32 * c2 + 4 * v4 + 2]) * p.scale),
                                 __float_as_uint(__uint_as_float(dqv[32 * c2 + 4 * v4 + 3]) * p.scale)));
      }
      ptx::fence_proxy_async_smem();  // the TMA unit reads the staged rows next
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(BB_DQ));
      if (warp == 0) {  // the issuing lane's wait decides for its whole warp
        if (issuer) {
          ok = b_wait1(ctl, bar(BB_DQ), s & 1);
          if (ok) {
            const int qrow0 = b_row0(i, p);
            for (int c = 0; c < d / 32; ++c) {  // boxes 0, 1 in the P area: one bulk group
              ptx::tma_reduce_add_4d(&tm.dq, base + BS_DQ + (uint32_t)c * kBBox, 32 * c, h, qrow0, b);
              if (c == 1) ptx::bulk_commit();
            }
            if (d / 32 > 2) ptx::bulk_commit();  // boxes 2, 3 in the dS area: a second one
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (ok) {
      // dK and dV of key tile j, row = key row, this warp's half of the head dim:
      // the last GRAD commit covers every MMA
      const int phys_k = b_phys(j * kTile + row, p);
      for (int c32 = hd0 / 32; c32 < (hd0 + d / 2) / 32; ++c32) {
        uint32_t kv[32], vv[32];
        __syncwarp();
        ptx::tmem_ld32(tdK + 32u * c32, kv);
        ptx::tmem_ld32(tdV + 32u * c32, vv);
        ptx::tmem_wait_ld();
        if (phys_k >= 0) {
          const long long o = (((long long)b * p.L + phys_k) * p.Hkv + g) * d + 32 * c32;
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            *reinterpret_cast<float4*>(p.dk + o + 4 * v4) =
                make_float4(__uint_as_float(kv[4 * v4]) * p.scale, __uint_as_float(kv[4 * v4 + 1]) * p.scale,
                            __uint_as_float(kv[4 * v4 + 2]) * p.scale, __uint_as_float(kv[4 * v4 + 3]) * p.scale);
            *reinterpret_cast<float4*>(p.dv + o + 4 * v4) =
                make_float4(__uint_as_float(vv[4 * v4]), __uint_as_float(vv[4 * v4 + 1]),
                            __uint_as_float(vv[4 * v4 + 2]), __uint_as_float(vv[4 * v4 + 3]));
          }
        }
      }
    }
  }

  // every reduce-add this CTA started has finished before it exits
  if (warp == 0 && lane == 0) ptx::bulk_wait0();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, 512);
}

// dO = dout sigmoid(g) (input dtype), D = sum_c dout out, dgate = dout out (1 - sigmoid(g)).
// One warp per two rows: 16 lanes x 8 channels (d = 128) or 8 lanes (d = 64).
template <bool BF16, bool OUT32>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdPrepParams p) {
  const int lpr = p.d / 8, rpw = 32 / lpr;
  const int lane = threadIdx.x & 31, sub = lane / lpr, li = lane % lpr;
  const long long warp_id = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nrows = (long long)p.B * p.L * p.H;
  const long long row = warp_id * rpw + sub;
  const bool live = row < nrows;
  const long long rr = live ? row : 0;
  const int h = (int)(rr % p.H);
  const long long bt = rr / p.H;
  const int t = (int)(bt % p.L), b = (int)(bt / p.L);
  const int c0 = 8 * li;
  float o[8], g8[8], dout[8];
  if (live) {
    const long long oi = rr * p.d + c0;
    if constexpr (OUT32) {
      const float4* a = reinterpret_cast<const float4*>(static_cast<const float*>(p.out) + oi);
      const float4* c = reinterpret_cast<const float4*>(static_cast<const float*>(p.dout) + oi);
      const float4 a0 = a[0], a1 = a[1], c0v = c[0], c1v = c[1];
      o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w; o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
      dout[0] = c0v.x; dout[1] = c0v.y; dout[2] = c0v.z; dout[3] = c0v.w;
      dout[4] = c1v.x; dout[5] = c1v.y; dout[6] = c1v.z; dout[7] = c1v.w;
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.out) + oi);
      const uint4 c = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dout) + oi);
      const uint16_t* ae = reinterpret_cast<const uint16_t*>(&a);
      const uint16_t* ce = reinterpret_cast<const uint16_t*>(&c);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        o[e] = BF16 ? __bfloat162float(__ushort_as_bfloat16(ae[e])) : __half2float(__ushort_as_half(ae[e]));
        dout[e] = BF16 ? __bfloat162float(__ushort_as_bfloat16(ce[e])) : __half2float(__ushort_as_half(ce[e]));
      }
    }
    if (p.gate) {
      const uint4 gv = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.gate) + b * p.g_stride[0] +
                                                       (long long)t * p.g_stride[1] + h * p.g_stride[2] + c0);
      const uint16_t* ge = reinterpret_cast<const uint16_t*>(&gv);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = BF16 ? __bfloat162float(__ushort_as_bfloat16(ge[e])) : __half2float(__ushort_as_half(ge[e]));
        g8[e] = 1.0f / (1.0f + expf(-x));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) g8[e] = 1.0f;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = dout[e] = 0.f, g8[e] = 1.f;
  }
  float dsum = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) dsum = fmaf(dout[e], o[e], dsum);
  for (int off = lpr / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
  if (!live) return;
  if (p.dq) {  // dq starts from zero: the gradient kernel adds every key tile's part into it
    float4* z = reinterpret_cast<float4*>(p.dq + rr * p.d + c0);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  uint4 w;
  uint32_t* we = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int u = 0; u < 4; ++u) we[u] = b_pack<BF16>(dout[2 * u] * g8[2 * u], dout[2 * u + 1] * g8[2 * u + 1]);
  *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dO) + rr * p.d + c0) = w;
  if (li == 0) p.D[((long long)b * p.H + h) * p.L + t] = dsum;
  if (p.dgate) {
    float* dg = p.dgate + rr * p.d + c0;
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = dout[e] * o[e] * (1.0f - g8[e]);
    reinterpret_cast<float4*>(dg)[0] = make_float4(r[0], r[1], r[2], r[3]);
    reinterpret_cast<float4*>(dg)[1] = make_float4(r[4], r[5], r[6], r[7]);
  }
}

template <bool BF16>
int run_bwd(const BwdDevParams& p, const BwdMaps& m, cudaStream_t s) {
  static bool opted_in = false;
  if (!opted_in) {
    if (cudaFuncSetAttribute(bwd_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)B_SMEM_ALLOC) !=
        cudaSuccess)
      return KREA_ERR_CUDA;
    opted_in = true;
  }
  const dim3 grid((unsigned)p.n_tiles, (unsigned)p.Hkv, (unsigned)p.B);
  bwd_kernel<BF16><<<grid, kBThreads, B_SMEM_ALLOC, s>>>(m, p);
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

}  // namespace

int launch_bwd_prep(const BwdPrepParams& p, bool bf16, bool out32, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long rows = (long long)p.B * p.L * p.H;
  const long long warps = (rows * (p.d / 8) + 31) / 32;
  const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
  if (bf16) out32 ? bwd_prep_kernel<true, true><<<blocks, 256, 0, s>>>(p) : bwd_prep_kernel<true, false><<<blocks, 256, 0, s>>>(p);
  else out32 ? bwd_prep_kernel<false, true><<<blocks, 256, 0, s>>>(p) : bwd_prep_kernel<false, false><<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? KREA_OK : KREA_ERR_CUDA;
}

int launch_backward(const BwdDevParams& p, const BwdMaps& m, bool bf16, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return bf16 ? run_bwd<true>(p, m, s) : run_bwd<false>(p, m, s);
}

}  // namespace krea
