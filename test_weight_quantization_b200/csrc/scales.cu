// scales.cu — step 2 of TTQ: AWQ scales from the shrunk diagonal covariance.
//
// TTQ review, "Proposed method", bullets 2-4 (arithmetic in awq_scale.cuh).
// O(K) work in one CTA; the mean reduced in a fixed order.
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

}  // namespace

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
