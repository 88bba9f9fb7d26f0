// kernels.h — internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ttq.h"

namespace ttq {

ttq_status launch_act_stats(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                            int64_t ldx, float p, int accumulate,
                            float* sum_out, cudaStream_t st);

ttq_status launch_act_stats_scales(const void* X, ttq_dtype xt, int64_t T,
                                   int64_t K, int64_t ldx, int accumulate,
                                   int64_t T_total, double alpha,
                                   double lambda, double p, float* sum_out,
                                   float* s, float* inv_s,
                                   unsigned int* counter, cudaStream_t st);

ttq_status launch_channel_total(const float* sum, int64_t T_total, int64_t K,
                                double* out, cudaStream_t st);
ttq_status launch_awq_scales_sharded(const float* sum, int64_t T_total,
                                     int64_t K, int64_t K_total,
                                     const double* total, double alpha,
                                     double lambda, double p, float* s,
                                     float* inv_s, cudaStream_t st);
ttq_status launch_awq_scales(const float* sum, int64_t T_total, int64_t K,
                             double alpha, double lambda, double p, float* s,
                             float* inv_s, cudaStream_t st);

ttq_status launch_quantize(const void* W, ttq_dtype wt, int64_t N, int64_t K,
                           int64_t ldw, const float* s, int bits, int group,
                           uint32_t* codes, float* delta, uint8_t* zero,
                           cudaStream_t st);

ttq_status launch_unpack(const uint32_t* codes, int64_t N, int64_t K, int bits,
                         uint8_t* q_out, cudaStream_t st);

// Workspace carve-up of the projection.
size_t gemm_workspace_bytes(int64_t T, int64_t K, int r);

ttq_status launch_lowbit_gemm(const void* X, ttq_dtype xt, int64_t T,
                              int64_t K, int64_t ldx, const float* inv_s,
                              const uint32_t* codes, const float* delta,
                              const uint8_t* zero, int64_t N, int bits,
                              int group, const void* A, const void* B, int r,
                              void* Y, ttq_dtype yt, int64_t ldy,
                              void* workspace, cudaStream_t st);

ttq_status launch_prepare(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                          int64_t ldx, const float* inv_s, int bits,
                          const void* A, int r, void* Xs, void* U,
                          cudaStream_t st);

// The decode projection on CUDA cores (T <= 2), used by
// launch_gemm_prepared when it applies.
bool gemv_applies(int64_t T, int64_t K);
ttq_status launch_gemv(const void* Xs, const void* U, int64_t T, int64_t K,
                       const uint32_t* codes, const float* delta,
                       const uint8_t* zero, int64_t N, int bits, int group,
                       const void* B, ttq_dtype bt, int r, void* Y,
                       ttq_dtype yt, int64_t ldy, cudaStream_t st);

ttq_status launch_gemm_prepared(const void* Xs, const void* U, int64_t T,
                                int64_t K, const uint32_t* codes,
                                const float* delta, const uint8_t* zero,
                                int64_t N, int bits, int group, const void* B,
                                ttq_dtype bt, int r, void* Y, ttq_dtype yt,
                                int64_t ldy, cudaStream_t st,
                                float* stats = nullptr, float stats_p = 2.f);
// The fused (QDQ) projection: group RTN of the bf16 weights W (pitch ldw)
// with scales s inside the tensor-core projection; codes, delta and zero of
// the quantized weights are stored when not null. Prefill (T > 32) only.
ttq_status launch_quantize_gemm_prepared(
    const void* W, int64_t ldw, const float* s, const void* Xs, const void* U,
    int64_t T, int64_t K, int64_t N, int bits, int group, const void* B,
    ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy, uint32_t* codes,
    float* delta, uint8_t* zero, cudaStream_t st);
// Partial rows of the fused output statistic for a prefill projection
// (0 when the shape has none), and the rows per token tile.
int64_t gemm_stats_rows(int64_t T, int64_t N, int64_t K, int bits);
int stats_parts_of(int dqw, int bn);
// sum_out[n] (+)= sum_p partials[p][n], p in order.
ttq_status launch_stats_reduce(const float* partials, int64_t P, int64_t N,
                               int accumulate, float* sum_out,
                               cudaStream_t st);

// One thread runs the library's bounded mbarrier wait; *out = 1 if the
// phase completed, 0 if the wait gave up (selftest.cu).
ttq_status launch_bounded_wait_check(int arrive, uint32_t* out,
                                     cudaStream_t st);

ttq_status launch_lowrank_add(const void* X, ttq_dtype xt, int64_t T,
                              int64_t K, int64_t ldx, const void* A,
                              const void* B, int r, int64_t N, void* Y,
                              ttq_dtype yt, int64_t ldy, cudaStream_t st);

// 2D TMA descriptor of a [rows][inner] tensor with a row pitch of
// pitch_bytes, copied in boxes of box_inner x box_rows; out-of-range
// elements read as zero (gemm.cu).
bool make_tensor_map_2d(CUtensorMap* m, CUtensorMapDataType dt,
                        const void* ptr, uint64_t inner, uint64_t rows,
                        uint64_t pitch_bytes, uint32_t box_inner,
                        uint32_t box_rows, CUtensorMapSwizzle swz);

// Per-prompt low-rank factors of the bf16 weight W (lowrank_dyn.cu).
size_t lowrank_factors_workspace_bytes(int64_t N, int64_t K, int r);
ttq_status launch_lowrank_factors(const void* W, int64_t N, int64_t K,
                                  int64_t ldw, const float* s,
                                  const float* omega, int r, int iters,
                                  void* B, void* A, void* workspace,
                                  cudaStream_t st);
ttq_status launch_lowrank_residual(const void* W, int64_t N, int64_t K,
                                   int64_t ldw, const void* B, const void* A,
                                   int r, void* R, int64_t ldr,
                                   cudaStream_t st);

}  // namespace ttq
