// lowrank_dyn.cu — per-prompt ("dynamic") low-rank factors of a weight and
// the residual that TTQ then quantizes.
//
// TTQ review, "Proposed method", bullet 5: when needed, W is written as
// W_q + B A with dynamic factors B and A and W_q is quantized on the fly;
// "Main results", bullet 4: TTQ quantizes the residual and adds the
// low-rank projection. The factors are found per prompt, once TTQ's scales
// s are known, by randomized subspace iteration (Halko, Martinsson and
// Tropp, "Finding structure with randomness", Algorithm 4.4) on the matrix
// TTQ quantizes, W_s = W diag(s), from r caller-drawn probe vectors Omega:
//   Q = orth(W_s Omega^T);  iters x { Z = orth(W_s^T Q); Q = orth(W_s Z) }
//   B = bf16(Q),  A = bf16(Q^T W)
// orth() keeps Gram-Schmidt's column order and drops a column whose part
// orthogonal to the kept columns is at most 2^-10 of the input's largest
// column norm (its output column is zero).
//
// Kernels:
//  skinny_kernel<TRANS>  out[j][m] = sum_c W[m][c] P[j][c] (TRANS: W[c][m]),
//      the r <= 64 columns of a product with the weight on tcgen05. W is
//      read once by TMA in 128 x 128 bf16 stages; eight converter warps move
//      a stage into TMEM as fp16 pairs (the A operand: a thread per output
//      row m = TMEM lane; TRANS reads a column of the stage per thread), and
//      one thread issues M=128, N=rpad, K=16 MMAs against the fp16 P tile.
//      The contraction is split over gridDim.y; each split writes its
//      partial sums, which the next kernel adds in split order.
//  gram_kernel           partial Gram matrices of y_m = sc_m sum_p parts
//      (fp32 entries, fp64 products and sums), one per CTA.
//  apply_kernel          every CTA adds the partials in CTA order and
//      factors the Gram matrix (Cholesky with the drop rule, fp64) into R,
//      then q_m = y_m R^-1 by forward substitution in fp64 (y as the Gram
//      kernel summed it): Q in fp32,
//      and the fp16 operand P = (post_m q_m) of the next product. One
//      gram/apply round orthonormalises a block of columns: the Gram
//      matrix is exact up to fp64 sums of exact products, so Q is
//      orthonormal to about cond(Y)^2 x 1e-16 (cond(Y) stays below about
//      4 x 2^10 because of the drop rule).
//  factors_out_kernel    B = bf16(Q_N)^T and A = bf16(sum_p parts).
//  residual_kernel       R = bf16(W - B A), fp32 accumulation in j order.
// Every mbarrier wait is bounded (TTQ_DEVERR_TIMEOUT, then the CTA winds
// down); nothing spins on another CTA.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ttq {
namespace {

constexpr int kBM = 128;                  // output rows per CTA (TMEM lanes)
constexpr int kSC = 128;                  // contraction per stage
constexpr uint32_t kWBox = kBM * 128u;    // one 128 x 64 bf16 box, bytes
constexpr uint32_t kWStage = 2u * kWBox;  // two boxes per stage
constexpr int kConvWarps = 8;
constexpr int kSkinnyThreads = 32 * (2 + kConvWarps);
constexpr int kTmemCols = 256;            // accumulator (64) + 3 stages
constexpr int kAccCols = 64;
constexpr float kDropTol = 0.0009765625f;  // 2^-10

struct SkinnyArgs {
  int M, C;          // output rows, contraction length
  int rpad, r;       // MMA N (16..64) and rows j of the output
  int c_stages;      // ceil(C / 128)
  int per;           // stages per split
  int S;             // shared-memory ring depth (2 or 3)
  float* out;        // [split][r][ldo]
  long long ldo;
  uint32_t* err;
};

__device__ __forceinline__ uint32_t bf16_pair_to_f16_pair(uint32_t v,
                                                          bool& range) {
  const float a = __uint_as_float(v << 16);
  const float b = __uint_as_float(v & 0xFFFF0000u);
  range |= !(fabsf(a) < 65504.f) || !(fabsf(b) < 65504.f);
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
  return v;
}

template <bool TRANS>
__global__ void __launch_bounds__(kSkinnyThreads, 2)
    skinny_kernel(const __grid_constant__ CUtensorMap tm_w,
                  const __grid_constant__ CUtensorMap tm_p,
                  const SkinnyArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  const int S = a.S;
  const uint32_t pbox = (uint32_t)a.rpad * 128u;  // one 64-column P box
  const uint32_t p_off = (uint32_t)S * kWStage;
  const uint32_t bar_off = p_off + (uint32_t)S * 2u * pbox;
  const uint32_t b_loaded = base + bar_off;
  const uint32_t b_ready = b_loaded + 8u * S;
  const uint32_t b_empty = b_ready + 8u * S;
  const uint32_t b_acc = b_empty + 8u * S;
  volatile uint32_t* tmem_slot =
      reinterpret_cast<volatile uint32_t*>(gbase + bar_off + 24u * S + 8u);
  volatile int* aborted =
      reinterpret_cast<volatile int*>(gbase + bar_off + 24u * S + 12u);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;
  const int split = blockIdx.y;
  const int s_begin = min(split * a.per, a.c_stages);
  const int n = min(s_begin + a.per, a.c_stages) - s_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(b_loaded + 8 * i, 1);
      mbar_init(b_ready + 8 * i, 32 * kConvWarps);
      mbar_init(b_empty + 8 * i, 1);
    }
    mbar_init(b_acc, 1);
    *aborted = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_p);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_enter();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_w = tmem + kAccCols;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < n; ++s) {
        const int slot = s % S;
        if (s >= S &&
            !mbar_wait(b_empty + 8 * slot, (uint32_t)(s / S - 1) & 1u, a.err)) {
          *aborted = 1;
          break;
        }
        if (*aborted) break;
        const int c0 = (s_begin + s) * kSC;
        const uint32_t bar = b_loaded + 8 * slot;
        const uint32_t wdst = base + (uint32_t)slot * kWStage;
        const uint32_t pdst = base + p_off + (uint32_t)slot * 2u * pbox;
        mbar_arrive_expect_tx(bar, kWStage + 2u * pbox);
        if constexpr (TRANS) {
          tma_load_2d(wdst, &tm_w, m0, c0, bar);
          tma_load_2d(wdst + kWBox, &tm_w, m0 + 64, c0, bar);
        } else {
          tma_load_2d(wdst, &tm_w, c0, m0, bar);
          tma_load_2d(wdst + kWBox, &tm_w, c0 + 64, m0, bar);
        }
        tma_load_2d(pdst, &tm_p, c0, 0, bar);
        tma_load_2d(pdst + pbox, &tm_p, c0 + 64, 0, bar);
        issued = s + 1;
      }
      // no bulk copy may still be writing shared memory at exit
      for (int i = 0; i < S && i < issued; ++i) {
        const int q = issued - 1 - i;
        mbar_wait(b_loaded + 8 * (q % S), (uint32_t)(q / S) & 1u, a.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kBM, a.rpad);
      for (int s = 0; s < n; ++s) {
        const int slot = s % S;
        if (!mbar_wait(b_ready + 8 * slot, (uint32_t)(s / S) & 1u, a.err)) {
          *aborted = 1;
          break;
        }
        tc_fence_after();
        const uint32_t ad = tmem_w + (uint32_t)slot * 64u;
        const uint32_t pd = base + p_off + (uint32_t)slot * 2u * pbox;
        const uint64_t bd0 = smem_desc_sw128(pd);
        const uint64_t bd1 = smem_desc_sw128(pd + pbox);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_f16_ts(tmem, ad + 8 * k, bd0 + 2 * k, idesc,
                        (s > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_f16_ts(tmem, ad + 32 + 8 * k, bd1 + 2 * k, idesc, 1u);
        tc_commit(b_empty + 8 * slot);
      }
      tc_commit(b_acc);
    }
  } else {
    // ---------------------------------------------- converter warps ---
    // thread = output row i of the tile = TMEM lane; the two warps of a
    // lane quarter take the two 64-wide halves of a stage's contraction
    const int q4 = warp & 3;
    const int h = (warp - 2) >> 2;
    const int i = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    bool range = false;
    for (int s = 0; s < n; ++s) {
      const int slot = s % S;
      // the load of stage s follows the MMA of stage s - S (the producer
      // waited for it), so this TMEM slot is free once `loaded` completes
      const bool ok =
          mbar_wait(b_loaded + 8 * slot, (uint32_t)(s / S) & 1u, a.err) &&
          !*aborted;
      if (!__all_sync(0xffffffffu, ok)) break;  // the TMEM store is per warp
      const uint32_t wst = base + (uint32_t)slot * kWStage;
      uint32_t o[32];
      if constexpr (!TRANS) {
        // row i of box h: 8 chunks of 16 bytes at chunk ^ (i % 8)
        const uint32_t row = wst + (uint32_t)h * kWBox + (uint32_t)i * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[4];
          asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                       : "r"(row + (((uint32_t)c ^ ((uint32_t)i & 7u)) << 4))
                       : "memory");
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[4 * c + e] = bf16_pair_to_f16_pair(v[e], range);
        }
      } else {
        // column i (box i / 64, column i % 64) of stage rows 64h .. 64h+63
        const uint32_t col = wst + (uint32_t)(i >> 6) * kWBox +
                             (uint32_t)(i & 7) * 2u;
        const uint32_t chunk = (uint32_t)((i & 63) >> 3);
#pragma unroll
        for (int pp = 0; pp < 32; ++pp) {
          const uint32_t c0 = (uint32_t)(64 * h + 2 * pp);
          const uint32_t lo = ld_shared_u16(col + c0 * 128u +
                                            ((chunk ^ (c0 & 7u)) << 4));
          const uint32_t hi = ld_shared_u16(col + (c0 + 1u) * 128u +
                                            ((chunk ^ ((c0 + 1u) & 7u)) << 4));
          o[pp] = bf16_pair_to_f16_pair(lo | (hi << 16), range);
        }
      }
      tmem_st32(tmem_w + (uint32_t)slot * 64u + lane_base + 32u * h, o);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_ready + 8 * slot);
    }
    if (range) flag_error(a.err, TTQ_DEVERR_FP16_RANGE);
    // epilogue: every issued MMA has completed once b_acc does (the MMA
    // thread commits it on every path)
    const bool done = mbar_wait(b_acc, 0, a.err);
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, done && !*aborted);
    if (go && h == 0) {
      const int m = m0 + i;
      float* out = a.out + (long long)split * a.r * a.ldo + m;
      for (int j0 = 0; j0 < a.rpad; j0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)j0, v);
        if (m < a.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j0 + j < a.r) out[(long long)(j0 + j) * a.ldo] = v[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------- orthonormalisation ---

constexpr int kGramThreads = 256;
constexpr int kGramRows = 128;
constexpr int kMaxGramCtas = 32;
constexpr int kMaxPairs = 64 * 65 / 2;

struct GramArgs {
  const float* parts;  // [nparts][r][ld], nparts <= kMaxParts
  int nparts;
  long long ld;
  int M, r;
  const float* sc;     // row scales (null: 1)
  float* ysum;         // if not null: the summed, scaled y, [r][ld]
  double* partials;    // [gridDim.x][npairs]
  uint32_t* err;
};

constexpr int kMaxParts = 16;  // partial products per y (the splits)
constexpr int kYBatch = 8;     // y entries a thread sums at once

// The (a, b) pairs a <= b of an r x r upper triangle in row order, into
// shared tables (entry s0(a) + b - a, s0(a) = a r - a (a - 1) / 2).
__device__ __forceinline__ void pair_tables(int r, uint16_t* pa, uint16_t* pb) {
  for (int e = threadIdx.x; e < r; e += blockDim.x) {
    const int s0 = e * r - e * (e - 1) / 2;
    for (int b = e; b < r; ++b) {
      pa[s0 + b - e] = (uint16_t)e;
      pb[s0 + b - e] = (uint16_t)b;
    }
  }
}

__global__ void __launch_bounds__(kGramThreads) gram_kernel(const GramArgs g) {
  // rows of y (fp32) during the partial sums; the Gram matrix (fp64) in
  // the tail
  __shared__ __align__(16) uint8_t buf[kGramRows * 65 * 4 > 64 * 65 * 8
                                           ? kGramRows * 65 * 4
                                           : 64 * 65 * 8];
  __shared__ uint16_t pa[kMaxPairs], pb[kMaxPairs];
  griddep_enter();
  const int r = g.r, npairs = r * (r + 1) / 2;
  pair_tables(r, pa, pb);
  float* ys = reinterpret_cast<float*>(buf);  // [kGramRows][65]
  constexpr int kPer = (kMaxPairs + kGramThreads - 1) / kGramThreads;
  double acc[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) acc[q] = 0.0;
  const int nblk = (g.M + kGramRows - 1) / kGramRows;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    __syncthreads();
    // y = sc_m sum_p parts[p], parts added in order. Loads are issued in
    // batches of four parts x kYBatch entries before any of them is added
    // (issue is in order: an add between two loads would serialise them);
    // entries past the block read a valid address and are discarded.
    for (int e0 = threadIdx.x; e0 < kGramRows * r;
         e0 += kYBatch * kGramThreads) {
      float v[kYBatch];
      long long off[kYBatch];
#pragma unroll
      for (int u = 0; u < kYBatch; ++u) {
        v[u] = 0.f;
        const int e = e0 + u * kGramThreads;
        const int m = blk * kGramRows + e % kGramRows;
        off[u] = (e < kGramRows * r && m < g.M)
                     ? (long long)(e / kGramRows) * g.ld + m
                     : 0;
      }
      for (int p0 = 0; p0 < g.nparts; p0 += 4) {
        float raw[4][kYBatch];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const long long pb =
              (long long)min(p0 + pp, g.nparts - 1) * r * g.ld;
#pragma unroll
          for (int u = 0; u < kYBatch; ++u)
            raw[pp][u] = __ldcg(g.parts + pb + off[u]);
        }
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
          if (p0 + pp < g.nparts)
#pragma unroll
            for (int u = 0; u < kYBatch; ++u) v[u] += raw[pp][u];
      }
#pragma unroll
      for (int u = 0; u < kYBatch; ++u) {
        const int e = e0 + u * kGramThreads;
        if (e < kGramRows * r) {
          const int row = e % kGramRows, j = e / kGramRows;
          const int m = blk * kGramRows + row;
          float y = 0.f;
          if (m < g.M) {
            y = g.sc ? v[u] * g.sc[m] : v[u];
            if (g.ysum) g.ysum[(long long)j * g.ld + m] = y;
          }
          ys[row * 65 + j] = y;
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = threadIdx.x + q * kGramThreads;
      if (e < npairs) {
        const int ea = pa[e], eb = pb[e];
        // fp64 products of fp32 entries are exact: the Gram matrix keeps
        // the resolution the drop rule needs (a column's remaining squared
        // norm is a difference of such sums)
        // four independent sums over rows 4i .. 4i+3 (the multiply-adds
        // of one sum would otherwise wait on each other), added in a fixed
        // order
        double d[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
        for (int row = 0; row < kGramRows; row += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            d[u] = fma((double)ys[(row + u) * 65 + ea],
                       (double)ys[(row + u) * 65 + eb], d[u]);
        }
        acc[q] += (d[0] + d[1]) + (d[2] + d[3]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int e = threadIdx.x + q * kGramThreads;
    if (e < npairs) g.partials[(long long)blockIdx.x * npairs + e] = acc[q];
  }
}

// R (upper, in G[a * ld + b], a <= b) of the Cholesky factorisation with the
// drop rule of the Gram matrix sum_c partials[c] (nc partials, added in
// order). Every thread of the CTA takes part; every CTA that runs it on
// the same partials gets the same R.
__device__ void factor_gram(const double* __restrict__ partials, int nc,
                            int r, const uint16_t* pa, const uint16_t* pb,
                            double* G, int ld, double* diag_max) {
  const int npairs = r * (r + 1) / 2;
  for (int e = threadIdx.x; e < npairs; e += blockDim.x) {
    // the CTAs' partials (at most kMaxGramCtas) in CTA order, their loads
    // issued together
    double raw[kMaxGramCtas];
#pragma unroll
    for (int u = 0; u < kMaxGramCtas; ++u)
      raw[u] = __ldcg(partials + (long long)min(u, nc - 1) * npairs + e);
    double v = 0.0;
#pragma unroll
    for (int u = 0; u < kMaxGramCtas; ++u)
      if (u < nc) v += raw[u];
    G[pa[e] * ld + pb[e]] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double mx = 0.0;
    for (int j = 0; j < r; ++j) mx = fmax(mx, G[j * ld + j]);
    *diag_max = mx;
  }
  __syncthreads();
  // right-looking Cholesky, upper factor in place; a column is dropped when
  // its remaining squared norm is at most (tol * largest column norm)^2
  const double dmax = *diag_max;
  const double thresh = (double)kDropTol * (double)kDropTol * dmax;
  for (int j = 0; j < r; ++j) {
    const double d = G[j * ld + j];
    const bool keep = dmax > 0.0 && d > thresh;
    // 1/sqrt(d): the fp32 estimate refined by two Newton steps in fp64
    // (each squares the relative error: 2^-22 -> 2^-44 -> below fp64's
    // precision), then sqrt(d) = d / sqrt(d); no fp64 divide or square
    // root on the factorisation's critical path
    double rinv = 0.0, rjj = 0.0;
    if (keep) {
      if (d > 1e-30 && d < 1e30) {  // inside fp32's range
        rinv = (double)rsqrtf((float)d);
        rinv = rinv * fma(-0.5 * d, rinv * rinv, 1.5);
        rinv = rinv * fma(-0.5 * d, rinv * rinv, 1.5);
      } else {
        rinv = 1.0 / sqrt(d);
      }
      rjj = d * rinv;
    }
    __syncthreads();
    for (int b = j + 1 + threadIdx.x; b < r; b += blockDim.x)
      G[j * ld + b] = keep ? G[j * ld + b] * rinv : 0.0;
    if (threadIdx.x == 0) G[j * ld + j] = rjj;
    __syncthreads();
    const int rest = r - j - 1;
    for (int e = threadIdx.x; e < rest * rest; e += blockDim.x) {
      const int ia = j + 1 + e / rest, ib = j + 1 + e % rest;
      if (ia <= ib) G[ia * ld + ib] -= G[j * ld + ia] * G[j * ld + ib];
    }
    __syncthreads();
  }
}

struct ApplyArgs {
  const float* y;      // [r][ldy]: the rows the Gram kernel factored
  long long ldy;
  int M, r;
  const double* partials;  // the Gram kernel's [nc][npairs] partial sums
  int nc;
  float* Q;            // [r][ldq] or null
  long long ldq;
  __half* P;           // [rpad][ldp] fp16 operand or null
  long long ldp;
  int rpad, Mp;        // P rows and the padded columns written
  const float* post;   // scales of P's columns (null: 1)
};

template <int RT>
__global__ void __launch_bounds__(256) apply_kernel(const ApplyArgs a) {
  // every CTA factors the Gram matrix itself (no CTA waits for another),
  // then substitutes its rows
  __shared__ double Rs[RT][RT + 1];
  __shared__ double Rinv[RT];  // 1 / R_jj (0 for a dropped column)
  __shared__ uint16_t pa[RT * (RT + 1) / 2], pb[RT * (RT + 1) / 2];
  __shared__ double diag_max;
  griddep_enter();
  const int r = a.r;
  pair_tables(r, pa, pb);
  for (int e = threadIdx.x; e < RT * (RT + 1); e += blockDim.x)
    (&Rs[0][0])[e] = 0.0;
  __syncthreads();
  factor_gram(a.partials, a.nc, r, pa, pb, &Rs[0][0], RT + 1, &diag_max);
  for (int j = threadIdx.x; j < RT; j += blockDim.x)
    Rinv[j] = Rs[j][j] > 0.0 ? 1.0 / Rs[j][j] : 0.0;
  __syncthreads();
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= a.Mp) return;
  if (m >= a.M) {
    if (a.P)
      for (int j = 0; j < a.rpad; ++j) a.P[(long long)j * a.ldp + m] =
          __float2half_rn(0.f);
    return;
  }
  // forward substitution in fp64: with R from an fp64 Gram matrix, one
  // Cholesky-QR round leaves Q orthonormal to about cond(Y)^2 x 1e-16,
  // far below the fp32 and bf16 roundings that follow
  float yv[RT];
  double q[RT];
#pragma unroll
  for (int j = 0; j < RT; ++j)
    yv[j] = j < r ? __ldcg(a.y + (long long)j * a.ldy + m) : 0.f;
#pragma unroll
  for (int j = 0; j < RT; ++j) {
    q[j] = 0.0;
    if (j < r && Rinv[j] > 0.0) {
      double v = (double)yv[j];
#pragma unroll
      for (int k = 0; k < j; ++k) v = fma(-Rs[k][j], q[k], v);
      q[j] = v * Rinv[j];
    }
  }
  const float post = a.post ? a.post[m] : 1.f;
#pragma unroll
  for (int j = 0; j < RT; ++j) {
    if (j < r) {
      const float qf = (float)q[j];
      if (a.Q) a.Q[(long long)j * a.ldq + m] = qf;
      if (a.P) a.P[(long long)j * a.ldp + m] = __float2half_rn(post * qf);
    } else if (a.P && j < a.rpad) {
      a.P[(long long)j * a.ldp + m] = __float2half_rn(0.f);
    }
  }
  if (a.P)
    for (int j = RT; j < a.rpad; ++j)
      a.P[(long long)j * a.ldp + m] = __float2half_rn(0.f);
}

// P[j][k] = fp16(s_k omega[j][k]); zeros past r rows and K columns
__global__ void probe_kernel(const float* __restrict__ omega,
                             const float* __restrict__ s, int r, int K,
                             int rpad, int Kp, __half* __restrict__ P) {
  griddep_enter();
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)rpad * Kp) return;
  const int j = (int)(e / Kp), k = (int)(e % Kp);
  const float v = (j < r && k < K) ? s[k] * omega[(long long)j * K + k] : 0.f;
  P[e] = __float2half_rn(v);
}

// B[n][j] = bf16(Q[j][n]) and A[j][k] = bf16(sum_p parts[p][j][k])
__global__ void factors_out_kernel(const float* __restrict__ Qn, int N,
                                   const float* __restrict__ parts, int nparts,
                                   int K, int r, __nv_bfloat16* __restrict__ B,
                                   __nv_bfloat16* __restrict__ A) {
  griddep_enter();
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nb = (long long)N * r;
  if (e < nb) {
    const int nn = (int)(e / r), j = (int)(e % r);
    B[e] = __float2bfloat16_rn(Qn[(long long)j * N + nn]);
  } else if (e < nb + (long long)r * K) {
    // the parts in order, their loads issued four at a time
    const long long f = e - nb;
    float v = 0.f;
    for (int p0 = 0; p0 < nparts; p0 += 4) {
      float raw[4];
#pragma unroll
      for (int pp = 0; pp < 4; ++pp)
        raw[pp] = __ldcg(parts + (long long)min(p0 + pp, nparts - 1) * r * K +
                         f);
#pragma unroll
      for (int pp = 0; pp < 4; ++pp)
        if (p0 + pp < nparts) v += raw[pp];
    }
    A[f] = __float2bfloat16_rn(v);
  }
}

// --------------------------------------------------------- residual ----

// R[n][k] = bf16(W[n][k] - sum_j B[n][j] A[j][k]), accumulated from W in j
// order with fused multiply-adds. A thread owns CPT consecutive channels
// of kResRows rows and holds their column of A in registers; it keeps the
// weights of 32 / CPT rows in flight (loads issued before any arithmetic),
// so that enough bytes are outstanding to stream W at HBM rate.
constexpr int kResThreads = 256;
constexpr int kResRows = 32;

template <int CPT>
__device__ __forceinline__ void store_r(__nv_bfloat16* __restrict__ p,
                                        int left, const float (&v)[CPT]) {
  if constexpr (CPT == 4) {
    if (left >= 4) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&lo);
      u.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p) = u;
      return;
    }
  } else if constexpr (CPT == 2) {
    if (left >= 2) {
      *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
      return;
    }
  }
#pragma unroll
  for (int c = 0; c < CPT; ++c)
    if (c < left) p[c] = __float2bfloat16_rn(v[c]);
}

template <int RT, int CPT>
__global__ void __launch_bounds__(kResThreads)
    residual_kernel(const __nv_bfloat16* __restrict__ W, int N, int K,
                    long long ldw, const __nv_bfloat16* __restrict__ B,
                    const __nv_bfloat16* __restrict__ A, int r,
                    __nv_bfloat16* __restrict__ R, long long ldr) {
  constexpr int RB = 32 / CPT;  // rows in flight per thread
  __shared__ __align__(16) float Bs[kResRows][RT];
  griddep_enter();
  const int n0 = blockIdx.y * kResRows;
  const int k0 = (blockIdx.x * kResThreads + threadIdx.x) * CPT;
  for (int e = threadIdx.x; e < kResRows * RT; e += kResThreads) {
    const int rr = e / RT, j = e % RT;
    const int nn = n0 + rr;
    Bs[rr][j] = (nn < N && j < r) ? __bfloat162float(B[(long long)nn * r + j])
                                  : 0.f;
  }
  __syncthreads();
  if (k0 >= K) return;
  const int left = K - k0;
  float av[RT][CPT];
#pragma unroll
  for (int j = 0; j < RT; ++j)
#pragma unroll
    for (int c = 0; c < CPT; ++c)
      av[j][c] = (j < r && c < left)
                     ? __bfloat162float(A[(long long)j * K + k0 + c])
                     : 0.f;
  const int rows = min(kResRows, N - n0);
  for (int rr0 = 0; rr0 < rows; rr0 += RB) {
    float w[RB][CPT];
    if (left >= CPT && CPT > 1) {
      // the RB rows' loads are issued before any of them is used (rows
      // past the end re-read the last row and are not stored): issue is in
      // order, so a use between two loads would serialise them
      using Raw = typename std::conditional<CPT == 4, uint2, uint32_t>::type;
      Raw raw[RB];
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int rr = min(rr0 + u, rows - 1);
        raw[u] = *reinterpret_cast<const Raw*>(
            W + (long long)(n0 + rr) * ldw + k0);
      }
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        if constexpr (CPT == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(&raw[u]);
          w[u][0] = __uint_as_float(v.x << 16);
          w[u][1] = __uint_as_float(v.x & 0xFFFF0000u);
          w[u][2] = __uint_as_float(v.y << 16);
          w[u][3] = __uint_as_float(v.y & 0xFFFF0000u);
        } else {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(&raw[u]);
          w[u][0] = __uint_as_float(v << 16);
          w[u][CPT - 1] = __uint_as_float(v & 0xFFFF0000u);
        }
      }
    } else {
      // one channel per thread, or the ragged end of a row: scalar loads,
      // again all issued before the arithmetic
      uint16_t raw[RB][CPT];
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int rr = min(rr0 + u, rows - 1);
        const unsigned short* src = reinterpret_cast<const unsigned short*>(
            W + (long long)(n0 + rr) * ldw + k0);
#pragma unroll
        for (int c = 0; c < CPT; ++c) raw[u][c] = src[c < left ? c : 0];
      }
#pragma unroll
      for (int u = 0; u < RB; ++u)
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          w[u][c] = c < left ? __uint_as_float((uint32_t)raw[u][c] << 16)
                             : 0.f;
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      if (rr0 + u < rows) {
        // B's row as float4s; entries past r are zero and so are A's, so
        // the padded steps add exact zeros and need no test
        float bj[RT];
#pragma unroll
        for (int q = 0; q < RT / 4; ++q) {
          const float4 t = *reinterpret_cast<const float4*>(&Bs[rr0 + u][4 * q]);
          bj[4 * q] = t.x;
          bj[4 * q + 1] = t.y;
          bj[4 * q + 2] = t.z;
          bj[4 * q + 3] = t.w;
        }
        if constexpr (CPT >= 2) {
          // two channels per instruction (two independent fp32 fused
          // multiply-adds, each rounded as fmaf would round it)
          float2 acc[CPT / 2];
#pragma unroll
          for (int c = 0; c < CPT / 2; ++c)
            acc[c] = make_float2(w[u][2 * c], w[u][2 * c + 1]);
#pragma unroll
          for (int j = 0; j < RT; ++j) {
            const float2 nb = make_float2(-bj[j], -bj[j]);
#pragma unroll
            for (int c = 0; c < CPT / 2; ++c)
              acc[c] = __ffma2_rn(
                  nb, make_float2(av[j][2 * c], av[j][2 * c + 1]), acc[c]);
          }
#pragma unroll
          for (int c = 0; c < CPT / 2; ++c) {
            w[u][2 * c] = acc[c].x;
            w[u][2 * c + 1] = acc[c].y;
          }
        } else {
#pragma unroll
          for (int j = 0; j < RT; ++j) w[u][0] = fmaf(-bj[j], av[j][0], w[u][0]);
        }
        store_r<CPT>(R + (long long)(n0 + rr0 + u) * ldr + k0, left, w[u]);
      }
    }
  }
}

// ------------------------------------------------------------ host ------

inline long long round_up(long long v, long long a) { return (v + a - 1) / a * a; }

struct Carve {
  float* parts;      // [max_splits][r][max(N, K)]
  float* qn;         // [r][N]
  float* qk;         // [r][K]
  float* ysum;       // [r][max(N, K)]  summed products
  __half* pn;        // [rpad][Np]
  __half* pk;        // [rpad][Kp]
  double* partials;  // [kMaxGramCtas][kMaxPairs]
  size_t total;
};

constexpr int kMaxSplits = kMaxParts;

Carve carve(void* ws, int64_t N, int64_t K, int r) {
  const long long rpad = round_up(r, 16), Np = round_up(N, 8),
                  Kp = round_up(K, 8), MX = std::max(N, K);
  Carve c{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (size_t)round_up((long long)(off + bytes), 256);
    return at;
  };
  const size_t o_parts = take((size_t)kMaxSplits * r * MX * 4);
  const size_t o_qn = take((size_t)r * N * 4);
  const size_t o_qk = take((size_t)r * K * 4);
  const size_t o_ys = take((size_t)r * MX * 4);
  const size_t o_pn = take((size_t)rpad * Np * 2);
  const size_t o_pk = take((size_t)rpad * Kp * 2);
  const size_t o_part = take((size_t)kMaxGramCtas * kMaxPairs * 8);
  c.total = off;
  if (ws) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    c.parts = reinterpret_cast<float*>(b + o_parts);
    c.qn = reinterpret_cast<float*>(b + o_qn);
    c.qk = reinterpret_cast<float*>(b + o_qk);
    c.ysum = reinterpret_cast<float*>(b + o_ys);
    c.pn = reinterpret_cast<__half*>(b + o_pn);
    c.pk = reinterpret_cast<__half*>(b + o_pk);
    c.partials = reinterpret_cast<double*>(b + o_part);
  }
  return c;
}

size_t skinny_smem(int rpad, int S) {
  return 1024 + (size_t)S * (kWStage + 2u * (uint32_t)rpad * 128u) +
         24u * S + 16;
}

// out[split][j][m] partial products of W (bf16 [N][K], pitch ldw) with the
// fp16 operand P [rpad][Cp]; returns the number of splits written.
ttq_status run_skinny(bool trans, const void* W, int64_t N, int64_t K,
                      int64_t ldw, const __half* P, int r, float* out,
                      int* splits_out, cudaStream_t st) {
  const int rpad = (int)round_up(r, 16);
  const int64_t M = trans ? K : N, C = trans ? N : K;
  const int64_t Cp = round_up(C, 8);
  const int mtiles = (int)((M + kBM - 1) / kBM);
  const int cst = (int)((C + kSC - 1) / kSC);
  const int want = std::max(1, 2 * sm_count() / mtiles);
  int splits = std::min({want, cst, kMaxSplits});
  const int per = (cst + splits - 1) / splits;
  splits = (cst + per - 1) / per;
  const int S = rpad <= 16 ? 3 : 2;
  CUtensorMap tw, tp;
  if (!make_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W,
                          (uint64_t)K, (uint64_t)N, (uint64_t)ldw * 2, 64, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&tp, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, P,
                          (uint64_t)Cp, (uint64_t)rpad, (uint64_t)Cp * 2, 64,
                          (uint32_t)rpad, CU_TENSOR_MAP_SWIZZLE_128B))
    return TTQ_ERR_CUDA;
  SkinnyArgs a;
  a.M = (int)M;
  a.C = (int)C;
  a.rpad = rpad;
  a.r = r;
  a.c_stages = cst;
  a.per = per;
  a.S = S;
  a.out = out;
  a.ldo = M;
  a.err = device_error_word();
  const size_t smem = skinny_smem(rpad, S);
  auto kern = trans ? skinny_kernel<true> : skinny_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return TTQ_ERR_CUDA;
  LaunchShape ls;
  ls.grid = dim3((unsigned)mtiles, (unsigned)splits, 1);
  ls.block = dim3(kSkinnyThreads);
  ls.smem = smem;
  *splits_out = splits;
  return launch(ls, st, kern, tw, tp, a);
}

template <int RT>
ttq_status launch_apply(const ApplyArgs& a, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3((unsigned)((a.Mp + 255) / 256));
  ls.block = dim3(256);
  return launch(ls, st, apply_kernel<RT>, a);
}

// Orthonormal columns of y (the summed, row-scaled parts) by one
// Gram/Cholesky/apply round (Cholesky-QR with an fp64 Gram matrix and an
// fp64 forward substitution): Q fp32 [r][M] and the fp16 operand P
// [rpad][Mp] = post * Q.
ttq_status run_qr(const Carve& c, const float* parts, int nparts, int64_t M,
                  int r, const float* sc, float* Q, __half* P,
                  const float* post, cudaStream_t st) {
  const int rpad = (int)round_up(r, 16);
  const int64_t Mp = round_up(M, 8);
  const int ctas = (int)std::min<int64_t>(kMaxGramCtas, (M + kGramRows - 1) /
                                                            kGramRows);
  GramArgs g;
  g.parts = parts;
  g.nparts = nparts;
  g.ld = M;
  g.M = (int)M;
  g.r = r;
  g.sc = sc;
  g.ysum = c.ysum;
  g.partials = c.partials;
  g.err = device_error_word();
  LaunchShape ls;
  ls.grid = dim3((unsigned)ctas);
  ls.block = dim3(kGramThreads);
  ttq_status e = launch(ls, st, gram_kernel, g);
  if (e != TTQ_OK) return e;
  ApplyArgs a;
  a.y = c.ysum;
  a.ldy = M;
  a.M = (int)M;
  a.r = r;
  a.partials = c.partials;
  a.nc = ctas;
  a.Q = Q;
  a.ldq = M;
  a.P = P;
  a.ldp = Mp;
  a.rpad = rpad;
  a.Mp = (int)Mp;
  a.post = post;
  return r <= 16 ? launch_apply<16>(a, st)
         : r <= 32 ? launch_apply<32>(a, st) : launch_apply<64>(a, st);
}

template <int RT, int CPT>
ttq_status launch_residual_t(const void* W, int64_t N, int64_t K,
                             int64_t ldw, const void* B, const void* A, int r,
                             void* R, int64_t ldr, cudaStream_t st) {
  LaunchShape ls;
  const int64_t cols = (K + CPT - 1) / CPT;
  ls.grid = dim3((unsigned)((cols + kResThreads - 1) / kResThreads),
                 (unsigned)((N + kResRows - 1) / kResRows));
  ls.block = dim3(kResThreads);
  return launch(ls, st, residual_kernel<RT, CPT>,
                static_cast<const __nv_bfloat16*>(W), (int)N, (int)K,
                (long long)ldw, static_cast<const __nv_bfloat16*>(B),
                static_cast<const __nv_bfloat16*>(A), r,
                static_cast<__nv_bfloat16*>(R), (long long)ldr);
}

}  // namespace

size_t lowrank_factors_workspace_bytes(int64_t N, int64_t K, int r) {
  return carve(nullptr, N, K, r).total;
}

ttq_status launch_lowrank_factors(const void* W, int64_t N, int64_t K,
                                  int64_t ldw, const float* s,
                                  const float* omega, int r, int iters,
                                  void* B, void* A, void* workspace,
                                  cudaStream_t st) {
  const Carve c = carve(workspace, N, K, r);
  const int rpad = (int)round_up(r, 16);
  const int64_t Kp = round_up(K, 8);
  {
    LaunchShape ls;
    const long long total = (long long)rpad * Kp;
    ls.grid = dim3((unsigned)((total + 255) / 256));
    ls.block = dim3(256);
    ttq_status e = launch(ls, st, probe_kernel, omega, s, r, (int)K, rpad,
                          (int)Kp, c.pk);
    if (e != TTQ_OK) return e;
  }
  int splits = 0;
  ttq_status e = run_skinny(false, W, N, K, ldw, c.pk, r, c.parts, &splits, st);
  if (e != TTQ_OK) return e;
  e = run_qr(c, c.parts, splits, N, r, nullptr, c.qn, c.pn, nullptr, st);
  if (e != TTQ_OK) return e;
  for (int it = 0; it < iters; ++it) {
    e = run_skinny(true, W, N, K, ldw, c.pn, r, c.parts, &splits, st);
    if (e != TTQ_OK) return e;
    e = run_qr(c, c.parts, splits, K, r, s, c.qk, c.pk, s, st);
    if (e != TTQ_OK) return e;
    e = run_skinny(false, W, N, K, ldw, c.pk, r, c.parts, &splits, st);
    if (e != TTQ_OK) return e;
    e = run_qr(c, c.parts, splits, N, r, nullptr, c.qn, c.pn, nullptr, st);
    if (e != TTQ_OK) return e;
  }
  e = run_skinny(true, W, N, K, ldw, c.pn, r, c.parts, &splits, st);
  if (e != TTQ_OK) return e;
  LaunchShape ls;
  const long long total = (long long)N * r + (long long)r * K;
  ls.grid = dim3((unsigned)((total + 255) / 256));
  ls.block = dim3(256);
  return launch(ls, st, factors_out_kernel, (const float*)c.qn, (int)N,
                (const float*)c.parts, splits, (int)K, r,
                static_cast<__nv_bfloat16*>(B), static_cast<__nv_bfloat16*>(A));
}

ttq_status launch_lowrank_residual(const void* W, int64_t N, int64_t K,
                                   int64_t ldw, const void* B, const void* A,
                                   int r, void* R, int64_t ldr,
                                   cudaStream_t st) {
  if (r <= 16)
    return launch_residual_t<16, 4>(W, N, K, ldw, B, A, r, R, ldr, st);
  if (r <= 32)
    return launch_residual_t<32, 2>(W, N, K, ldw, B, A, r, R, ldr, st);
  return launch_residual_t<64, 1>(W, N, K, ldw, B, A, r, R, ldr, st);
}

}  // namespace ttq
