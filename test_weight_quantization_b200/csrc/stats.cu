// stats.cu — step 1 of TTQ: per-input-channel activation statistics.
//
// TTQ review, "Proposed method", bullets 2-3: the per-prompt activation
// statistic is the diagonal of the input covariance; here the kernel emits
// sum_t |x_tj|^p (p = 2: the diagonal of X^T X) and the scales kernel
// divides by the token count.
//
// Design (HBM-bound column reduction):
//   - a thread owns 8 consecutive channels and loads them as one 16-byte
//     vector (two for fp32); CW/8 threads cover a row segment of CW channels
//     and the 256-thread CTA covers 256/(CW/8) rows per pass;
//   - each CTA walks a contiguous range of rows with 16 independent loads
//     in flight per thread (8 for fp32), the last partial group predicated,
//     accumulating in fp32 registers;
//   - rows split across a thread-block cluster of up to 8 CTAs; partial sums
//     are reduced through distributed shared memory by cluster rank 0 in a
//     fixed order, so the result is deterministic and no global scratch is
//     needed;
//   - optionally (ttq_act_stats_scales) step 2 runs in the same launch: the
//     cluster that finishes its column tile last, told by a counter in
//     global memory, computes the scales of all K channels. Nothing waits on
//     another CTA, so the fused form adds no spin and no co-residency need.
#include <cooperative_groups.h>

#include <algorithm>

#include "awq_scale.cuh"
#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace ttq {
namespace {

constexpr int kThreads = 256;

// 8 elements from the raw 16-byte vector(s) loaded for them.
template <typename TX>
__device__ __forceinline__ void unpack8(const uint4 (&r)[sizeof(TX) == 4 ? 2 : 1],
                                        float (&x)[8]);
template <>
__device__ __forceinline__ void unpack8<float>(const uint4 (&r)[2],
                                               float (&x)[8]) {
  x[0] = __uint_as_float(r[0].x); x[1] = __uint_as_float(r[0].y);
  x[2] = __uint_as_float(r[0].z); x[3] = __uint_as_float(r[0].w);
  x[4] = __uint_as_float(r[1].x); x[5] = __uint_as_float(r[1].y);
  x[6] = __uint_as_float(r[1].z); x[7] = __uint_as_float(r[1].w);
}
template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const uint4 (&r)[1],
                                                       float (&x)[8]) {
  bf16x2_to_f32(r[0].x, x[0], x[1]);
  bf16x2_to_f32(r[0].y, x[2], x[3]);
  bf16x2_to_f32(r[0].z, x[4], x[5]);
  bf16x2_to_f32(r[0].w, x[6], x[7]);
}
template <>
__device__ __forceinline__ void unpack8<__half>(const uint4 (&r)[1],
                                                float (&x)[8]) {
  f16x2_to_f32(r[0].x, x[0], x[1]);
  f16x2_to_f32(r[0].y, x[2], x[3]);
  f16x2_to_f32(r[0].z, x[4], x[5]);
  f16x2_to_f32(r[0].w, x[6], x[7]);
}

template <int PK>
__device__ __forceinline__ float moment(float x, float p) {
  if (PK == 2) return x * x;
  if (PK == 1) return fabsf(x);
  return powf(fabsf(x), p);
}

// Step 2 fused behind the statistics; s == nullptr leaves it out.
struct ScalesTail {
  float* s;
  float* inv_s;
  unsigned int* counter;  // zero on entry; the last cluster resets it
  int64_t T_total;
  double alpha, lambda, p;
};

// grid = (column tiles, cluster size); cluster = (1, C, 1).
template <typename TX, int PK>
__global__ void __launch_bounds__(kThreads)
    act_stats_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                     int64_t ldx, float p, int accumulate, int cw,
                     float* __restrict__ sum_out, ScalesTail tail) {
  // [rows_per_pass][cw] then part[cw]
  extern __shared__ __align__(16) float smem[];
  __shared__ int last_flag;
  __shared__ double tile_part[kThreads / 32];
  griddep_enter();
  cg::cluster_group cluster = cg::this_cluster();
  const int tpr = cw / 8;                 // threads per row segment
  const int rows_per_pass = kThreads / tpr;
  const int tid = threadIdx.x;
  const int lane_col = tid % tpr;
  const int row_in_pass = tid / tpr;
  const int64_t col0 = (int64_t)blockIdx.x * cw + lane_col * 8;
  const bool col_ok = col0 < K;

  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int64_t rows_per_cta = (T + C - 1) / C;
  const int64_t r_begin = rank * rows_per_cta;
  const int64_t r_end = min(T, r_begin + rows_per_cta);

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  if (col_ok) {
    // keep kUnroll raw 16-byte vectors in flight per thread (two per row
    // for fp32), converting only after all of them were issued
    constexpr int V = sizeof(TX) == 4 ? 2 : 1;  // 16-byte vectors per row
    constexpr int U = sizeof(TX) == 4 ? 8 : 16;  // rows in flight
    int64_t r = r_begin + row_in_pass;
    for (; r + (int64_t)(U - 1) * rows_per_pass < r_end;
         r += (int64_t)U * rows_per_pass) {
      uint4 raw[U][V];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int v = 0; v < V; ++v)
          raw[u][v] = ld_stream_v4(X + (r + (int64_t)u * rows_per_pass) * ldx +
                                   col0 + v * (8 / V));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float x[8];
        unpack8<TX>(raw[u], x);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += moment<PK>(x[i], p);
      }
    }
    // fewer than U passes remain: one predicated block keeps them all in
    // flight (a row past the end reads as zero and adds exactly 0)
    if (r < r_end) {
      uint4 raw[U][V];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t rr = r + (int64_t)u * rows_per_pass;
#pragma unroll
        for (int v = 0; v < V; ++v)
          raw[u][v] = rr < r_end ? ld_stream_v4(X + rr * ldx + col0 + v * (8 / V))
                                 : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float x[8];
        unpack8<TX>(raw[u], x);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += moment<PK>(x[i], p);
      }
    }
  }

  // CTA reduction over the rows of a pass, fixed order.
  float* red = smem;
  float* part = smem + rows_per_pass * cw;
#pragma unroll
  for (int i = 0; i < 8; ++i) red[row_in_pass * cw + lane_col * 8 + i] = acc[i];
  __syncthreads();
  for (int c = tid; c < cw; c += kThreads) {
    float s = 0.f;
    for (int rr = 0; rr < rows_per_pass; ++rr) s += red[rr * cw + c];
    part[c] = s;
  }
  cluster.sync();

  // Cluster reduction by rank 0, ranks in order.
  double tile = 0.0;  // this thread's column (cw <= kThreads)
  if (rank == 0) {
    for (int c = tid; c < cw; c += kThreads) {
      const int64_t col = (int64_t)blockIdx.x * cw + c;
      if (col >= K) continue;
      float s = 0.f;
      for (int q = 0; q < C; ++q) s += cluster.map_shared_rank(part, q)[c];
      s = accumulate ? sum_out[col] + s : s;
      sum_out[col] = s;
      tile += (double)s;
    }
  }
  if (tail.s == nullptr) {
    cluster.sync();  // keep every CTA's shared memory alive until read
    return;
  }

  // Fused step 2. Rank 0 adds its tile's sums (fixed tree) and leaves the
  // fp64 total in words 2b, 2b+1 of s (b = column tile; s is written only
  // after every tile total was read), then publishes with one
  // acquire-release arrival per cluster; the arrival that completes the
  // count marks its cluster last and tells every CTA of the cluster through
  // its shared memory.
  if (rank == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      tile += __shfl_xor_sync(0xffffffffu, tile, o);
    if ((tid & 31) == 0) tile_part[tid >> 5] = tile;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) t += tile_part[w];
      const unsigned long long bits = (unsigned long long)__double_as_longlong(t);
      tail.s[2 * blockIdx.x] = __uint_as_float((uint32_t)bits);
      tail.s[2 * blockIdx.x + 1] = __uint_as_float((uint32_t)(bits >> 32));
      // acquire-release at GPU scope: the CTA's writes (ordered before this
      // thread by the barrier above) are released with the arrival, and the
      // last arrival acquires every other cluster's
      unsigned prev;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                   : "=r"(prev)
                   : "l"(tail.counter)
                   : "memory");
      const int last = prev == gridDim.x - 1;
      if (last) *tail.counter = 0u;  // every arrival of this launch is in
      for (int q = 0; q < C; ++q) *cluster.map_shared_rank(&last_flag, q) = last;
    }
  }
  cluster.sync();  // after this no CTA reads another's shared memory
  if (!last_flag) return;
  // every CTA of the last cluster adds the tile totals in tile order (the
  // same value in every CTA and whichever cluster is last) ...
  const double invT = 1.0 / (double)tail.T_total;
  if (tid < 32) {
    double t = 0.0;
    for (int b = tid; b < (int)gridDim.x; b += 32) {
      const uint32_t lo = __float_as_uint(__ldcg(tail.s + 2 * b));
      const uint32_t hi = __float_as_uint(__ldcg(tail.s + 2 * b + 1));
      t += __longlong_as_double(
          (long long)(((unsigned long long)hi << 32) | lo));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (tid == 0) tile_part[0] = t;
  }
  cluster.sync();  // every tile total read before s is overwritten
  const double mbar = tile_part[0] * invT / (double)K;
  // ... then the scales of its share of the channels, four at a time
  const int64_t stride = (int64_t)C * kThreads;
  for (int64_t j0 = (int64_t)rank * kThreads + tid; j0 < K; j0 += 4 * stride) {
    float sj[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * stride;
      sj[u] = j < K ? __ldcg(sum_out + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * stride;
      if (j < K)
        awq_scale_one(sj[u], invT, mbar, tail.alpha, tail.lambda, tail.p,
                      tail.s[j], tail.inv_s[j]);
    }
  }
}

template <typename TX, int PK>
ttq_status launch_typed(const void* X, int64_t T, int64_t K, int64_t ldx,
                        float p, int accumulate, float* sum_out,
                        const ScalesTail& tail, cudaStream_t st) {
  const int cw = K >= 1024 ? 128 : 64;
  const int64_t col_tiles = (K + cw - 1) / cw;
  const int target = 2 * sm_count();
  int C = (int)std::min<int64_t>(
      8, std::max<int64_t>(1, (target + col_tiles - 1) / col_tiles));
  // keep at least 32 rows per CTA
  C = (int)std::min<int64_t>(C, std::max<int64_t>(1, (T + 31) / 32));
  const int rows_per_pass = kThreads / (cw / 8);
  const size_t smem = sizeof(float) * ((size_t)rows_per_pass * cw + cw);

  LaunchShape ls;
  ls.grid = dim3((unsigned)col_tiles, (unsigned)C, 1);
  ls.block = dim3(kThreads, 1, 1);
  ls.smem = smem;
  ls.cluster_y = (unsigned)C;
  return launch(ls, st, act_stats_kernel<TX, PK>, static_cast<const TX*>(X),
                T, K, ldx, p, accumulate, cw, sum_out, tail);
}

template <typename TX>
ttq_status launch_p(const void* X, int64_t T, int64_t K, int64_t ldx, float p,
                    int accumulate, float* sum_out, const ScalesTail& tail,
                    cudaStream_t st) {
  if (p == 2.0f)
    return launch_typed<TX, 2>(X, T, K, ldx, p, accumulate, sum_out, tail,
                               st);
  if (p == 1.0f)
    return launch_typed<TX, 1>(X, T, K, ldx, p, accumulate, sum_out, tail,
                               st);
  return launch_typed<TX, 0>(X, T, K, ldx, p, accumulate, sum_out, tail, st);
}

ttq_status launch_x(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                    int64_t ldx, float p, int accumulate, float* sum_out,
                    const ScalesTail& tail, cudaStream_t st) {
  switch (xt) {
    case TTQ_F32:
      return launch_p<float>(X, T, K, ldx, p, accumulate, sum_out, tail, st);
    case TTQ_BF16:
      return launch_p<__nv_bfloat16>(X, T, K, ldx, p, accumulate, sum_out,
                                     tail, st);
    case TTQ_F16:
      return launch_p<__half>(X, T, K, ldx, p, accumulate, sum_out, tail, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

// sum_out[n] (+)= sum_p partials[p][n] over the P partial rows in order:
// one thread per channel, consecutive threads on consecutive channels.
__global__ void stats_reduce_kernel(const float* __restrict__ partials,
                                    int64_t P, int64_t N, int accumulate,
                                    float* __restrict__ sum_out) {
  griddep_enter();
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float acc = 0.f;
  for (int64_t q = 0; q < P; ++q) acc += __ldcg(partials + q * N + n);
  sum_out[n] = accumulate ? sum_out[n] + acc : acc;
}

}  // namespace

ttq_status launch_stats_reduce(const float* partials, int64_t P, int64_t N,
                               int accumulate, float* sum_out,
                               cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3((unsigned)((N + 255) / 256));
  ls.block = dim3(256);
  return launch(ls, st, stats_reduce_kernel, partials, P, N, accumulate,
                sum_out);
}

ttq_status launch_act_stats(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                            int64_t ldx, float p, int accumulate,
                            float* sum_out, cudaStream_t st) {
  const ScalesTail none = {nullptr, nullptr, nullptr, 0, 0.0, 0.0, 0.0};
  return launch_x(X, xt, T, K, ldx, p, accumulate, sum_out, none, st);
}

ttq_status launch_act_stats_scales(const void* X, ttq_dtype xt, int64_t T,
                                   int64_t K, int64_t ldx, int accumulate,
                                   int64_t T_total, double alpha,
                                   double lambda, double p, float* sum_out,
                                   float* s, float* inv_s,
                                   unsigned int* counter, cudaStream_t st) {
  const ScalesTail tail = {s, inv_s, counter, T_total, alpha, lambda, p};
  return launch_x(X, xt, T, K, ldx, (float)p, accumulate, sum_out, tail, st);
}

}  // namespace ttq
