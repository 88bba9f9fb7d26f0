// lowrank.cu — the low-rank term as a call of its own.
//
// TTQ review, "Proposed method", bullet 5 and "Main results", bullet 4:
// with W = W_q + B A the projection adds (X A^T) B^T. ttq_w_lowbit_gemm
// folds this term into its tensor-core K loop; this kernel serves callers
// that add it to an existing Y (Y += (X A^T) B^T), in fp32 arithmetic.
//
// One CTA per 16 tokens: U = X A^T for those tokens (rank <= 64) is reduced
// by warps into shared memory, then every thread walks output channels and
// adds sum_rho U[t][rho] B[n][rho] for the 16 tokens.
#include "common.cuh"
#include "kernels.h"

namespace ttq {
namespace {

constexpr int kTok = 16;
constexpr int kThreads = 256;

template <typename TX, typename TY>
__global__ void __launch_bounds__(kThreads)
    lowrank_add_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                       int64_t ldx, const TX* __restrict__ A,
                       const TX* __restrict__ B, int r, int64_t N,
                       TY* __restrict__ Y, int64_t ldy) {
  __shared__ float U[kTok][64];
  griddep_enter();
  const int64_t t0 = (int64_t)blockIdx.x * kTok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int item = warp; item < kTok * r; item += kThreads / 32) {
    const int tt = item / r, rho = item % r;
    const int64_t t = t0 + tt;
    float acc = 0.f;
    if (t < T)
      for (int64_t j = lane; j < K; j += 32)
        acc = fmaf(to_f32(X[t * ldx + j]), to_f32(A[(int64_t)rho * K + j]),
                   acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) U[tt][rho] = acc;
  }
  __syncthreads();
  for (int64_t n = threadIdx.x; n < N; n += kThreads) {
    float acc[kTok];
#pragma unroll
    for (int tt = 0; tt < kTok; ++tt) acc[tt] = 0.f;
    for (int rho = 0; rho < r; ++rho) {
      const float b = to_f32(B[n * r + rho]);
#pragma unroll
      for (int tt = 0; tt < kTok; ++tt) acc[tt] = fmaf(U[tt][rho], b, acc[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < kTok; ++tt) {
      const int64_t t = t0 + tt;
      if (t < T) {
        TY* y = Y + t * ldy + n;
        *y = from_f32<TY>(to_f32(*y) + acc[tt]);
      }
    }
  }
}

template <typename TX, typename TY>
ttq_status launch_typed(const void* X, int64_t T, int64_t K, int64_t ldx,
                        const void* A, const void* B, int r, int64_t N,
                        void* Y, int64_t ldy, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3((unsigned)((T + kTok - 1) / kTok));
  ls.block = dim3(kThreads);
  return launch(ls, st, lowrank_add_kernel<TX, TY>, static_cast<const TX*>(X),
                T, K, ldx, static_cast<const TX*>(A),
                static_cast<const TX*>(B), r, N, static_cast<TY*>(Y), ldy);
}

template <typename TX>
ttq_status launch_y(ttq_dtype yt, const void* X, int64_t T, int64_t K,
                    int64_t ldx, const void* A, const void* B, int r,
                    int64_t N, void* Y, int64_t ldy, cudaStream_t st) {
  switch (yt) {
    case TTQ_F32:
      return launch_typed<TX, float>(X, T, K, ldx, A, B, r, N, Y, ldy, st);
    case TTQ_BF16:
      return launch_typed<TX, __nv_bfloat16>(X, T, K, ldx, A, B, r, N, Y, ldy,
                                             st);
    case TTQ_F16:
      return launch_typed<TX, __half>(X, T, K, ldx, A, B, r, N, Y, ldy, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

}  // namespace

ttq_status launch_lowrank_add(const void* X, ttq_dtype xt, int64_t T,
                              int64_t K, int64_t ldx, const void* A,
                              const void* B, int r, int64_t N, void* Y,
                              ttq_dtype yt, int64_t ldy, cudaStream_t st) {
  switch (xt) {
    case TTQ_F32:
      return launch_y<float>(yt, X, T, K, ldx, A, B, r, N, Y, ldy, st);
    case TTQ_BF16:
      return launch_y<__nv_bfloat16>(yt, X, T, K, ldx, A, B, r, N, Y, ldy, st);
    case TTQ_F16:
      return launch_y<__half>(yt, X, T, K, ldx, A, B, r, N, Y, ldy, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

}  // namespace ttq
