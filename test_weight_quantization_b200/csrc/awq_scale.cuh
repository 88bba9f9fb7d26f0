// awq_scale.cuh — device arithmetic of step 2 of TTQ, shared by the scales
// kernel and the statistics kernel's fused tail.
//
// TTQ review, "Proposed method", bullets 2-4: AWQ with a closed form on the
// diagonal input covariance, shrunk by lambda. With m_j = sum_j / T:
//   c_j = (1 - lambda) m_j + lambda mean_k(m_k),   s_j = c_j^(alpha/p).
#pragma once

#include "common.cuh"

namespace ttq {

// sum_k (sum_k / T) in fp64 by the NT threads of one CTA, in a fixed order
// (thread-strided partials, a butterfly inside each warp, warps in order),
// so every CTA that runs it gets the same value. warp_sums holds NT/32
// doubles of shared memory; sum is read through L2 (other CTAs wrote it).
template <int NT>
__device__ double awq_channel_total(const float* sum, int64_t K, double invT,
                                    double* warp_sums) {
  double local = 0.0;
  int64_t j = threadIdx.x;
  for (; j + 3 * NT < K; j += 4 * NT) {
    const float a = __ldcg(sum + j), b = __ldcg(sum + j + NT),
                c = __ldcg(sum + j + 2 * NT), d = __ldcg(sum + j + 3 * NT);
    local += (double)a * invT;
    local += (double)b * invT;
    local += (double)c * invT;
    local += (double)d * invT;
  }
  for (; j < K; j += NT) local += (double)__ldcg(sum + j) * invT;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = local;
  __syncthreads();
  double total = 0.0;
  for (int w = 0; w < NT / 32; ++w) total += warp_sums[w];
  __syncthreads();  // warp_sums may be reused by the caller
  return total;
}

// mean_k(sum_k / T): the total above divided by K.
template <int NT>
__device__ double awq_channel_mean(const float* sum, int64_t K, double invT,
                                   double* warp_sums) {
  return awq_channel_total<NT>(sum, K, invT, warp_sums) / (double)K;
}

// s_j and 1/s_j of one channel. c_j is formed in fp64; the power runs in
// fp32 on c_j rounded to fp32 (relative error below 1e-6, far inside the
// 1e-5 agreement with the fp64 definition): square or fourth roots for the
// exponents 1/2 and 1/4 (alpha = 0.5 with p = 1 or 2), powf otherwise, and
// fp64 pow outside the range where fp32 keeps full precision.
__device__ __forceinline__ void awq_scale_one(float sum_j, double invT,
                                              double mbar, double alpha,
                                              double lambda, double p,
                                              float& s, float& inv_s) {
  const double m = (double)sum_j * invT;
  const double c = (1.0 - lambda) * m + lambda * mbar;
  float sj = 1.f, ij = 1.f;
  if (alpha != 0.0 && c > 0.0 && isfinite(c)) {
    const float cf = (float)c;
    const double e = alpha / p;
    if (!(cf > 1e-30f && cf < 1e30f))
      sj = (float)pow(c, e);
    else if (e == 0.5)  // square and fourth roots: within 2 ulp, cheaper
      sj = sqrtf(cf);
    else if (e == 0.25)
      sj = sqrtf(sqrtf(cf));
    else
      sj = powf(cf, (float)e);
    ij = 1.f / sj;
  }
  s = sj;
  inv_s = ij;
}

}  // namespace ttq
