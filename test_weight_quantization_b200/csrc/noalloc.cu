// noalloc.cu — the quantized projection without a caller-provided workspace.
//
// ttq_w_lowbit_gemm needs T*K*2 (+T*128) bytes of device scratch for the
// prepared fp16 activations, which the caller allocates. Some callers cannot
// allocate device memory at the point where they run the projection: a
// plugin that an inference engine calls after the engine has fixed its
// memory plan, or host code that only receives device pointers from another
// runtime and has no allocator of its own. This entry point serves them with
// a scratch buffer built into the library: a file-scope __device__ array of
// TTQ_NOALLOC_SCRATCH_BYTES, present on every GPU that loads the library
// until the process exits.
//
// Set-up: the first call on a device looks up the array's device address
// with cudaGetSymbolAddress (with that device current) and caches it; that
// first call should therefore come before any stream capture. The array is
// shared by every call and keeps the last call's contents; everything the
// kernels read from it is written earlier in the same call, so nothing needs
// clearing. Calls whose execution overlaps on the GPU (different streams,
// or other threads) race on the array.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

#define TTQ_EXPORT extern "C" __attribute__((visibility("default")))

static __device__ __align__(256) uint8_t g_ttq_noalloc_scratch[TTQ_NOALLOC_SCRATCH_BYTES];

namespace ttq {
namespace {

constexpr int kMaxDev = 64;
std::atomic<void*> g_scratch[kMaxDev];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, or null.
void* scratch_address() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDev) return nullptr;
  void* p = g_scratch[d].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  p = g_scratch[d].load(std::memory_order_relaxed);
  if (!p) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_ttq_noalloc_scratch) != cudaSuccess ||
        addr == nullptr)
      return nullptr;
    p = addr;
    g_scratch[d].store(p, std::memory_order_release);
  }
  return p;
}

bool is_aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

bool dtype_ok(ttq_dtype t) {
  return t == TTQ_F32 || t == TTQ_BF16 || t == TTQ_F16;
}

}  // namespace
}  // namespace ttq

using namespace ttq;

TTQ_EXPORT ttq_status ttq_w_lowbit_gemm_noalloc(
    const void* X, ttq_dtype xt, int64_t T, int64_t K, int64_t ldx,
    const float* inv_s, const uint32_t* codes, const float* delta,
    const uint8_t* zero, int64_t N, int bits, int group, const void* A,
    const void* B, int r, void* Y, ttq_dtype yt, int64_t ldy, void* stream) {
  const bool group_ok =
      group == 16 || group == 32 || group == 64 || group == 128;
  if (!X || !inv_s || !codes || !delta || !zero || !Y || !dtype_ok(xt) ||
      !dtype_ok(yt) || T < 1 || N < 1 || K < 32 || K % 32 != 0 || bits < 2 ||
      bits > 8 || !group_ok || K % group != 0 || r < 0 || r > 64 ||
      ((r > 0) != (A && B)) || (r == 0 && (A || B)) || ldx < K || ldy < N ||
      !is_aligned(X, 16) || (ldx * dtype_bytes(xt)) % 16 != 0 ||
      !is_aligned(inv_s, 16) || !is_aligned(codes, 16) ||
      !is_aligned(delta, 16) || !is_aligned(zero, 16) ||
      !is_aligned(Y, dtype_bytes(yt)) ||
      (r > 0 && (!is_aligned(A, 16) || (K * dtype_bytes(xt)) % 16 != 0 ||
                 !is_aligned(B, dtype_bytes(xt)))) ||
      T >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) ||
      N >= ((int64_t)1 << 31))
    return TTQ_ERR_INVALID_ARG;
  // The built-in scratch holds the prepared activations of at most
  // TTQ_NOALLOC_SCRATCH_BYTES; larger inputs need ttq_w_lowbit_gemm.
  if (gemm_workspace_bytes(T, K, r) > (size_t)TTQ_NOALLOC_SCRATCH_BYTES)
    return TTQ_ERR_UNSUPPORTED;
  void* scratch = scratch_address();
  if (!scratch) return TTQ_ERR_CUDA;
  return launch_lowbit_gemm(X, xt, T, K, ldx, inv_s, codes, delta, zero, N,
                            bits, group, A, B, r, Y, yt, ldy, scratch,
                            static_cast<cudaStream_t>(stream));
}
