// api.cu — the exported C ABI of libttq (declared in include/ttq.h).
//
// Every entry point validates its arguments on the host before enqueuing
// anything, then calls an internal launcher. Nothing here allocates device
// memory; the library's device state is the sticky error word below and the
// built-in scratch array of noalloc.cu (host side: cached SM counts).
#include <math.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

#define TTQ_EXPORT extern "C" __attribute__((visibility("default")))

// Sticky error bits raised by kernels (TTQ_DEVERR_*), one word per device.
__device__ uint32_t g_ttq_device_error;

namespace ttq {
namespace {

constexpr int kMaxDevices = 64;
std::atomic<uint32_t*> g_err_ptr[kMaxDevices];
std::atomic<int> g_sms[kMaxDevices];
std::mutex g_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

bool valid_dtype(ttq_dtype t) {
  return t == TTQ_F32 || t == TTQ_BF16 || t == TTQ_F16;
}

// A [rows, cols] matrix with row pitch ld elements whose rows all start on a
// 16-byte boundary.
bool rows_aligned(const void* p, ttq_dtype t, int64_t ld) {
  return aligned(p, 16) && ((ld * dtype_bytes(t)) % 16) == 0;
}

bool valid_group(int g) { return g == 16 || g == 32 || g == 64 || g == 128; }

// Whether byte ranges [a, a + na) and [b, b + nb) overlap.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a);
  const uintptr_t y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

uint32_t* device_error_word() {
  const int d = current_device();
  if (d < 0) return nullptr;
  uint32_t* p = g_err_ptr[d].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_mu);
  p = g_err_ptr[d].load(std::memory_order_relaxed);
  if (!p) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_ttq_device_error) != cudaSuccess)
      return nullptr;
    p = static_cast<uint32_t*>(addr);
    g_err_ptr[d].store(p, std::memory_order_release);
  }
  return p;
}

int sm_count() {
  const int d = current_device();
  if (d < 0) return 148;
  int n = g_sms[d].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) !=
          cudaSuccess ||
      n <= 0)
    n = 148;
  g_sms[d].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace ttq

using namespace ttq;

TTQ_EXPORT int ttq_abi_version(void) { return 8; }

TTQ_EXPORT int64_t ttq_codes_ld(int64_t K, int bits) {
  if (K < 32 || K % 32 != 0 || bits < 2 || bits > 8) return 0;
  return codes_ld(K, bits);
}

TTQ_EXPORT int64_t ttq_groups_ld(int64_t K, int group) {
  if (K < 1 || !valid_group(group) || K % group != 0) return 0;
  return groups_ld(K, group);
}

TTQ_EXPORT const char* ttq_status_string(ttq_status s) {
  switch (s) {
    case TTQ_OK: return "TTQ_OK";
    case TTQ_ERR_INVALID_ARG: return "TTQ_ERR_INVALID_ARG";
    case TTQ_ERR_UNSUPPORTED: return "TTQ_ERR_UNSUPPORTED";
    case TTQ_ERR_CUDA: return "TTQ_ERR_CUDA";
    case TTQ_ERR_TIMEOUT: return "TTQ_ERR_TIMEOUT";
    case TTQ_ERR_RANGE: return "TTQ_ERR_RANGE";
  }
  return "TTQ_ERR_UNKNOWN";
}

TTQ_EXPORT int ttq_device_error(int clear) {
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ttq_device_error, sizeof(v)) != cudaSuccess)
    return -1;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_ttq_device_error, &zero, sizeof(zero)) !=
        cudaSuccess)
      return -1;
  }
  return (int)v;
}

TTQ_EXPORT ttq_status ttq_act_stats(const void* X, ttq_dtype xt, int64_t T,
                                    int64_t K, int64_t ldx, float p,
                                    int accumulate, float* sum_out,
                                    void* stream) {
  if (!X || !sum_out || !valid_dtype(xt) || T < 1 || K < 8 || K % 8 != 0 ||
      ldx < K || !rows_aligned(X, xt, ldx) || !aligned(sum_out, 4) ||
      !(p > 0.f) || !isfinite(p) || (accumulate != 0 && accumulate != 1))
    return TTQ_ERR_INVALID_ARG;
  return launch_act_stats(X, xt, T, K, ldx, p, accumulate, sum_out,
                          as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_awq_scales(const float* sum, int64_t T_total,
                                     int64_t K, const ttq_params* prm,
                                     float* s, float* inv_s, void* stream) {
  if (!sum || !s || !inv_s || !prm || T_total < 1 || K < 1 ||
      !(prm->alpha >= 0.f) || !isfinite(prm->alpha) ||
      !(prm->lambda >= 0.f && prm->lambda <= 1.f) || !(prm->p > 0.f) ||
      !isfinite(prm->p) || !aligned(sum, 4) || !aligned(s, 4) ||
      !aligned(inv_s, 4))
    return TTQ_ERR_INVALID_ARG;
  return launch_awq_scales(sum, T_total, K, prm->alpha, prm->lambda, prm->p,
                           s, inv_s, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_channel_moment_total(const float* sum,
                                               int64_t T_total, int64_t K,
                                               double* total, void* stream) {
  if (!sum || !total || T_total < 1 || K < 1 || !aligned(sum, 4) ||
      !aligned(total, 8))
    return TTQ_ERR_INVALID_ARG;
  return launch_channel_total(sum, T_total, K, total, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_awq_scales_sharded(const float* sum, int64_t T_total,
                                             int64_t K, int64_t K_total,
                                             const ttq_params* prm,
                                             const double* total, float* s,
                                             float* inv_s, void* stream) {
  if (!sum || !total || !s || !inv_s || !prm || T_total < 1 || K < 1 ||
      K_total < K || !(prm->alpha >= 0.f) || !isfinite(prm->alpha) ||
      !(prm->lambda >= 0.f && prm->lambda <= 1.f) || !(prm->p > 0.f) ||
      !isfinite(prm->p) || !aligned(sum, 4) || !aligned(total, 8) ||
      !aligned(s, 4) || !aligned(inv_s, 4))
    return TTQ_ERR_INVALID_ARG;
  return launch_awq_scales_sharded(sum, T_total, K, K_total, total,
                                   prm->alpha, prm->lambda, prm->p, s, inv_s,
                                   as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_act_stats_scales(
    const void* X, ttq_dtype xt, int64_t T, int64_t K, int64_t ldx,
    int accumulate, int64_t T_total, const ttq_params* prm, float* sum_out,
    float* s, float* inv_s, uint32_t* counter, void* stream) {
  if (!X || !sum_out || !s || !inv_s || !prm || !counter || !valid_dtype(xt) ||
      T < 1 || K < 8 || K % 8 != 0 || ldx < K || !rows_aligned(X, xt, ldx) ||
      !aligned(sum_out, 4) || !aligned(s, 4) || !aligned(inv_s, 4) ||
      !aligned(counter, 4) || (accumulate != 0 && accumulate != 1) ||
      T_total < T || !(prm->alpha >= 0.f) || !isfinite(prm->alpha) ||
      !(prm->lambda >= 0.f && prm->lambda <= 1.f) || !(prm->p > 0.f) ||
      !isfinite(prm->p))
    return TTQ_ERR_INVALID_ARG;
  // the launch keeps partial results in s until the scales are written:
  // the sums, the two scale arrays and the counter must not overlap
  const size_t kb = (size_t)K * sizeof(float);
  if (overlaps(sum_out, kb, s, kb) || overlaps(sum_out, kb, inv_s, kb) ||
      overlaps(s, kb, inv_s, kb) || overlaps(counter, 4, sum_out, kb) ||
      overlaps(counter, 4, s, kb) || overlaps(counter, 4, inv_s, kb))
    return TTQ_ERR_INVALID_ARG;
  return launch_act_stats_scales(X, xt, T, K, ldx, accumulate, T_total,
                                 prm->alpha, prm->lambda, prm->p, sum_out, s,
                                 inv_s, counter, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_quantize_rtn_grouped(
    const void* W, ttq_dtype wt, int64_t N, int64_t K, int64_t ldw,
    const float* s, int bits, int group, uint32_t* codes, float* delta,
    uint8_t* zero, void* stream) {
  if (!W || !codes || !delta || !zero || !valid_dtype(wt) || N < 1 ||
      K < 32 || K % 32 != 0 || bits < 2 || bits > 8 || !valid_group(group) ||
      K % group != 0 || ldw < K || !rows_aligned(W, wt, ldw) ||
      (s && !aligned(s, 16)) || !aligned(codes, 16) || !aligned(delta, 16) ||
      !aligned(zero, 16) || N * (K / 32) >= ((int64_t)1 << 31))
    return TTQ_ERR_INVALID_ARG;
  return launch_quantize(W, wt, N, K, ldw, s, bits, group, codes, delta, zero,
                         as_stream(stream));
}

TTQ_EXPORT size_t ttq_w_lowbit_gemm_workspace_size(int64_t T, int64_t K,
                                                   int r) {
  if (T < 1 || K < 1 || r < 0) return 0;
  return gemm_workspace_bytes(T, K, r);
}

TTQ_EXPORT ttq_status ttq_w_lowbit_gemm(
    const void* X, ttq_dtype xt, int64_t T, int64_t K, int64_t ldx,
    const float* inv_s, const uint32_t* codes, const float* delta,
    const uint8_t* zero, int64_t N, int bits, int group, const void* A,
    const void* B, int r, void* Y, ttq_dtype yt, int64_t ldy, void* workspace,
    size_t workspace_bytes, void* stream) {
  if (!X || !inv_s || !codes || !delta || !zero || !Y || !workspace ||
      !valid_dtype(xt) || !valid_dtype(yt) || T < 1 || N < 1 || K < 32 ||
      K % 32 != 0 || bits < 2 || bits > 8 || !valid_group(group) ||
      K % group != 0 || r < 0 || r > 64 || ((r > 0) != (A && B)) ||
      (r == 0 && (A || B)) || ldx < K || ldy < N ||
      !rows_aligned(X, xt, ldx) || !aligned(inv_s, 16) ||
      !aligned(codes, 16) || !aligned(delta, 16) || !aligned(zero, 16) ||
      !aligned(Y, dtype_bytes(yt)) || !aligned(workspace, 256) ||
      (r > 0 && (!rows_aligned(A, xt, K) || !aligned(B, dtype_bytes(xt)))) ||
      T >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) ||
      N >= ((int64_t)1 << 31))
    return TTQ_ERR_INVALID_ARG;
  if (workspace_bytes < gemm_workspace_bytes(T, K, r))
    return TTQ_ERR_INVALID_ARG;
  return launch_lowbit_gemm(X, xt, T, K, ldx, inv_s, codes, delta, zero, N,
                            bits, group, A, B, r, Y, yt, ldy, workspace,
                            as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_prepare_activations(const void* X, ttq_dtype xt,
                                              int64_t T, int64_t K, int64_t ldx,
                                              const float* inv_s, int bits,
                                              const void* A, int r, void* Xs,
                                              void* U, void* stream) {
  if (!X || !inv_s || !Xs || !valid_dtype(xt) || T < 1 || K < 32 ||
      K % 32 != 0 || bits < 2 || bits > 8 || ldx < K || r < 0 || r > 64 ||
      T * (K / 16) >= ((int64_t)1 << 31) ||
      ((r > 0) != (A && U)) ||
      (r == 0 && (A || U)) || !rows_aligned(X, xt, ldx) ||
      !aligned(inv_s, 16) || !aligned(Xs, 16) || (U && !aligned(U, 16)) ||
      (r > 0 && !rows_aligned(A, xt, K)))
    return TTQ_ERR_INVALID_ARG;
  return launch_prepare(X, xt, T, K, ldx, inv_s, bits, A, r, Xs, U,
                        as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_w_lowbit_gemm_prepared(
    const void* Xs, const void* U, int64_t T, int64_t K, const uint32_t* codes,
    const float* delta, const uint8_t* zero, int64_t N, int bits, int group,
    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
    void* stream) {
  if (!Xs || !codes || !delta || !zero || !Y || !valid_dtype(yt) || T < 1 ||
      N < 1 || K < 32 || K % 32 != 0 || bits < 2 || bits > 8 ||
      !valid_group(group) || K % group != 0 || r < 0 || r > 64 ||
      ((r > 0) != (U && B)) || (r == 0 && (U || B)) ||
      (r > 0 && !valid_dtype(bt)) || ldy < N || !aligned(Xs, 16) ||
      (U && !aligned(U, 16)) || !aligned(codes, 16) || !aligned(delta, 16) ||
      !aligned(zero, 16) || !aligned(Y, dtype_bytes(yt)) ||
      (r > 0 && !aligned(B, dtype_bytes(bt))) || T >= ((int64_t)1 << 31) ||
      K >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31))
    return TTQ_ERR_INVALID_ARG;
  return launch_gemm_prepared(Xs, U, T, K, codes, delta, zero, N, bits, group,
                              B, bt, r, Y, yt, ldy, as_stream(stream));
}

TTQ_EXPORT int64_t ttq_projection_stats_rows(int64_t T, int64_t N, int64_t K,
                                            int bits) {
  if (T < 1 || N < 1 || K < 32 || K % 32 != 0 || bits < 2 || bits > 8 ||
      T >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) ||
      K >= ((int64_t)1 << 31))
    return 0;
  return gemm_stats_rows(T, N, K, bits);
}

TTQ_EXPORT ttq_status ttq_w_lowbit_gemm_prepared_stats(
    const void* Xs, const void* U, int64_t T, int64_t K, const uint32_t* codes,
    const float* delta, const uint8_t* zero, int64_t N, int bits, int group,
    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
    float p, float* stats, int64_t stats_rows, void* stream) {
  if (!stats || !(p > 0.f) || !isfinite(p) || !aligned(stats, 4))
    return TTQ_ERR_INVALID_ARG;
  const int64_t rows = ttq_projection_stats_rows(T, N, K, bits);
  if (rows == 0) return TTQ_ERR_UNSUPPORTED;
  if (stats_rows != rows) return TTQ_ERR_INVALID_ARG;
  if (!Xs || !codes || !delta || !zero || !Y || !valid_dtype(yt) ||
      !valid_group(group) || K % group != 0 || r < 0 || r > 64 ||
      ((r > 0) != (U && B)) || (r == 0 && (U || B)) ||
      (r > 0 && !valid_dtype(bt)) || ldy < N || !aligned(Xs, 16) ||
      (U && !aligned(U, 16)) || !aligned(codes, 16) || !aligned(delta, 16) ||
      !aligned(zero, 16) || !aligned(Y, dtype_bytes(yt)) ||
      (r > 0 && !aligned(B, dtype_bytes(bt))))
    return TTQ_ERR_INVALID_ARG;
  return launch_gemm_prepared(Xs, U, T, K, codes, delta, zero, N, bits, group,
                              B, bt, r, Y, yt, ldy, as_stream(stream), stats,
                              p);
}

TTQ_EXPORT ttq_status ttq_quantize_gemm_prepared(
    const void* W, ttq_dtype wt, int64_t ldw, const float* s, const void* Xs,
    const void* U, int64_t T, int64_t K, int64_t N, int bits, int group,
    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
    uint32_t* codes, float* delta, uint8_t* zero, void* stream) {
  if (!W || !s || !Xs || !Y || !valid_dtype(wt) || !valid_dtype(yt) || T < 1 ||
      N < 1 || K < 32 || K % 32 != 0 || bits < 2 || bits > 8 ||
      !valid_group(group) || K % group != 0 || r < 0 || r > 64 ||
      ((r > 0) != (U && B)) || (r == 0 && (U || B)) ||
      (r > 0 && !valid_dtype(bt)) || ldw < K || ldy < N ||
      !rows_aligned(W, wt, ldw) || !aligned(s, 16) || !aligned(Xs, 16) ||
      (U && !aligned(U, 16)) || !aligned(Y, dtype_bytes(yt)) ||
      (r > 0 && !aligned(B, dtype_bytes(bt))) ||
      ((codes != nullptr) != (delta != nullptr)) ||
      ((codes != nullptr) != (zero != nullptr)) ||
      (codes && (!aligned(codes, 16) || !aligned(delta, 16) ||
                 !aligned(zero, 16))) ||
      T >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) ||
      N >= ((int64_t)1 << 31))
    return TTQ_ERR_INVALID_ARG;
  // the fused form reads bf16 weight tiles and runs the prefill tile only
  if (wt != TTQ_BF16 || T <= 32) return TTQ_ERR_UNSUPPORTED;
  return launch_quantize_gemm_prepared(W, ldw, s, Xs, U, T, K, N, bits, group,
                                       B, bt, r, Y, yt, ldy, codes, delta,
                                       zero, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_stats_reduce(const float* partials, int64_t P,
                                       int64_t N, int accumulate,
                                       float* sum_out, void* stream) {
  if (!partials || !sum_out || P < 1 || N < 1 ||
      (accumulate != 0 && accumulate != 1) || !aligned(partials, 4) ||
      !aligned(sum_out, 4))
    return TTQ_ERR_INVALID_ARG;
  return launch_stats_reduce(partials, P, N, accumulate, sum_out,
                             as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_lowrank_add(const void* X, ttq_dtype xt, int64_t T,
                                      int64_t K, int64_t ldx, const void* A,
                                      const void* B, int r, int64_t N, void* Y,
                                      ttq_dtype yt, int64_t ldy,
                                      void* stream) {
  if (!X || !A || !B || !Y || !valid_dtype(xt) || !valid_dtype(yt) || T < 1 ||
      K < 1 || N < 1 || r < 1 || r > 64 || ldx < K || ldy < N ||
      !aligned(X, dtype_bytes(xt)) || !aligned(A, dtype_bytes(xt)) ||
      !aligned(B, dtype_bytes(xt)) || !aligned(Y, dtype_bytes(yt)))
    return TTQ_ERR_INVALID_ARG;
  return launch_lowrank_add(X, xt, T, K, ldx, A, B, r, N, Y, yt, ldy,
                            as_stream(stream));
}

TTQ_EXPORT size_t ttq_lowrank_factors_workspace_size(int64_t N, int64_t K,
                                                     int r) {
  if (N < 1 || K < 1 || r < 1 || r > 64 || N > (1LL << 30) ||
      K > (1LL << 30))
    return 0;
  return lowrank_factors_workspace_bytes(N, K, r);
}

TTQ_EXPORT ttq_status ttq_lowrank_factors(const void* W, int64_t N, int64_t K,
                                          int64_t ldw, const float* s,
                                          const float* omega, int r, int iters,
                                          void* B, void* A, void* workspace,
                                          size_t workspace_bytes,
                                          void* stream) {
  if (!W || !s || !omega || !B || !A || !workspace || N < 1 || K < 1 ||
      N > (1LL << 30) || K > (1LL << 30) || r < 1 || r > 64 || iters < 0 ||
      iters > 16 || ldw < K || !rows_aligned(W, TTQ_BF16, ldw) ||
      !aligned(s, 4) || !aligned(omega, 4) || !aligned(B, 2) ||
      !aligned(A, 2) || !aligned(workspace, 256) ||
      workspace_bytes < lowrank_factors_workspace_bytes(N, K, r))
    return TTQ_ERR_INVALID_ARG;
  const size_t nb = (size_t)N * r * 2, na = (size_t)r * K * 2,
               nw = (size_t)((N - 1) * ldw + K) * 2;
  if (overlaps(B, nb, A, na) || overlaps(B, nb, W, nw) ||
      overlaps(A, na, W, nw) || overlaps(workspace, workspace_bytes, B, nb) ||
      overlaps(workspace, workspace_bytes, A, na))
    return TTQ_ERR_INVALID_ARG;
  return launch_lowrank_factors(W, N, K, ldw, s, omega, r, iters, B, A,
                                workspace, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_lowrank_residual(const void* W, int64_t N, int64_t K,
                                           int64_t ldw, const void* B,
                                           const void* A, int r, void* R,
                                           int64_t ldr, void* stream) {
  if (!W || !B || !A || !R || N < 1 || K < 1 || N > (1LL << 30) ||
      K > (1LL << 30) || r < 1 || r > 64 || ldw < K || ldr < K ||
      !rows_aligned(W, TTQ_BF16, ldw) || !rows_aligned(R, TTQ_BF16, ldr) ||
      !aligned(B, 2) || !aligned(A, 2))
    return TTQ_ERR_INVALID_ARG;
  const size_t nb = (size_t)N * r * 2, na = (size_t)r * K * 2,
               nw = (size_t)((N - 1) * ldw + K) * 2,
               nr = (size_t)((N - 1) * ldr + K) * 2;
  const bool in_place = R == W && ldr == ldw;
  if ((!in_place && overlaps(R, nr, W, nw)) || overlaps(R, nr, B, nb) ||
      overlaps(R, nr, A, na))
    return TTQ_ERR_INVALID_ARG;
  return launch_lowrank_residual(W, N, K, ldw, B, A, r, R, ldr,
                                 as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_unpack_codes(const uint32_t* codes, int64_t N,
                                       int64_t K, int bits, uint8_t* q_out,
                                       void* stream) {
  if (!codes || !q_out || N < 1 || K < 32 || K % 32 != 0 || bits < 2 ||
      bits > 8 || !aligned(codes, 4))
    return TTQ_ERR_INVALID_ARG;
  return launch_unpack(codes, N, K, bits, q_out, as_stream(stream));
}

TTQ_EXPORT ttq_status ttq_selftest_bounded_wait(int arrive, uint32_t* out,
                                                void* stream) {
  if (!out || !aligned(out, sizeof(uint32_t))) return TTQ_ERR_INVALID_ARG;
  return launch_bounded_wait_check(arrive ? 1 : 0, out, as_stream(stream));
}
