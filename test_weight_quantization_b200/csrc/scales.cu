// scales.cu — step 2 of TTQ: AWQ scales from the shrunk diagonal covariance.
//
// TTQ review, "Proposed method", bullets 2-4 (arithmetic in awq_scale.cuh).
// O(K) work in one CTA; the mean reduced in a fixed order. For a layer whose
// input channels are split over several GPUs (row-parallel), the channel
// total of each shard is formed here, added across the GPUs by the caller,
// and the scales of each shard take the mean from that sum.
#include "awq_scale.cuh"
#include "kernels.h"

namespace ttq {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
    awq_scales_kernel(const float* __restrict__ sum, int64_t T_total,
                      int64_t K, double alpha, double lambda, double p,
                      float* __restrict__ s, float* __restrict__ inv_s) {
  __shared__ double warp_sums[kThreads / 32];
  griddep_enter();
  const double invT = 1.0 / (double)T_total;
  const double mbar = awq_channel_mean<kThreads>(sum, K, invT, warp_sums);
  // four independent channels per iteration to overlap their latencies
  for (int64_t j0 = threadIdx.x; j0 < K; j0 += 4 * kThreads) {
    float sj[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * kThreads;
      sj[u] = j < K ? __ldcg(sum + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * kThreads;
      if (j < K) awq_scale_one(sj[u], invT, mbar, alpha, lambda, p, s[j], inv_s[j]);
    }
  }
}

// The same scales with the channel mean taken from a total over a larger
// set of channels (this shard's and the others'): mbar = *total / K_total.
__global__ void __launch_bounds__(kThreads)
    awq_scales_sharded_kernel(const float* __restrict__ sum, int64_t T_total,
                              int64_t K, int64_t K_total,
                              const double* __restrict__ total, double alpha,
                              double lambda, double p, float* __restrict__ s,
                              float* __restrict__ inv_s) {
  griddep_enter();
  const double invT = 1.0 / (double)T_total;
  const double mbar = __ldcg(total) / (double)K_total;
  for (int64_t j0 = threadIdx.x; j0 < K; j0 += 4 * kThreads) {
    float sj[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * kThreads;
      sj[u] = j < K ? __ldcg(sum + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + u * kThreads;
      if (j < K) awq_scale_one(sj[u], invT, mbar, alpha, lambda, p, s[j], inv_s[j]);
    }
  }
}

// *out = sum_j sum[j] / T_total in fp64, in the fixed order of
// awq_channel_total (one CTA).
__global__ void __launch_bounds__(kThreads)
    channel_total_kernel(const float* __restrict__ sum, int64_t T_total,
                         int64_t K, double* __restrict__ out) {
  __shared__ double warp_sums[kThreads / 32];
  griddep_enter();
  const double t =
      awq_channel_total<kThreads>(sum, K, 1.0 / (double)T_total, warp_sums);
  if (threadIdx.x == 0) *out = t;
}

}  // namespace

ttq_status launch_channel_total(const float* sum, int64_t T_total, int64_t K,
                                double* out, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3(1);
  ls.block = dim3(kThreads);
  return launch(ls, st, channel_total_kernel, sum, T_total, K, out);
}

ttq_status launch_awq_scales_sharded(const float* sum, int64_t T_total,
                                     int64_t K, int64_t K_total,
                                     const double* total, double alpha,
                                     double lambda, double p, float* s,
                                     float* inv_s, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3(1);
  ls.block = dim3(kThreads);
  return launch(ls, st, awq_scales_sharded_kernel, sum, T_total, K, K_total,
                total, alpha, lambda, p, s, inv_s);
}

ttq_status launch_awq_scales(const float* sum, int64_t T_total, int64_t K,
                             double alpha, double lambda, double p, float* s,
                             float* inv_s, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3(1);
  ls.block = dim3(kThreads);
  return launch(ls, st, awq_scales_kernel, sum, T_total, K, alpha, lambda, p,
                s, inv_s);
}

}  // namespace ttq
