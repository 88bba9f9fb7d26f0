// gemm.cu — step 4 of TTQ: the quantized projection on 5th-generation
// tensor cores, with dequantisation inside the GEMM.
//
// TTQ review, "Proposed method", bullets 1 and 7 (QDQ weights; a GPU kernel
// for the quantized projection) and bullet 5 (optional W = W_q + B A):
//   Y = (X diag(1/s)) W_hat_s^T + (X A^T) B^T,  W_hat_s = (q - z) * D.
//
// Orientation: the weight rows are the MMA's M dimension (128 TMEM lanes)
// and the tokens its N dimension (16..256 TMEM columns), so one dequantised
// 128 x 64 weight tile feeds up to 256 tokens. Operands are fp16: the
// activations are scaled by 1/s and rounded once to fp16 by a pre-pass
// (prescale_kernel), each weight (q - z) * D is rounded once to fp16 in the
// dequantiser; products accumulate in fp32 in TMEM.
//
// CTA = 6 warps:
//   warp 0      TMA producer: fp16 activation tiles (64 x BN, 128B swizzle)
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//   warps 2-5   dequantisers (one weight row per thread: codes, delta, zero
//               arrive by cp.async into a private ring; fp16 pairs are built
//               with the 1024+q exponent trick and written in the 128B
//               swizzled K-major layout), then the epilogue (TMEM -> Y)
// Decode (T <= 16) splits K over a cluster of up to 8 CTAs; partial tiles
// are summed by cluster rank 0 through distributed shared memory in a fixed
// order. The rank-r low-rank term is one extra K stage: [X~ | U] [W | B]^T
// with U = X A^T (fp16, computed by lowrank_u_kernel).
// Every wait is bounded (TTQ_DEVERR_TIMEOUT, then the CTA winds down).
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace ttq {
namespace {

constexpr int kBM = 128;       // weight rows per CTA
constexpr int kBK = 64;        // K per stage: one 128-byte fp16 row
constexpr int kThreads = 192;  // 6 warps
constexpr int kATileBytes = kBM * kBK * 2;
constexpr int kMaxStages = 8;
constexpr int kSmemBudget = 220 * 1024;

// Words each dequantiser thread stages per K step: 2 blocks of codes,
// up to 4 deltas, 2 words holding the zero bytes.
__host__ __device__ constexpr int ring_words(int bits) { return 2 * bits + 6; }

struct GemmArgs {
  const uint32_t* codes;
  const float* delta;
  const uint8_t* zero;
  const void* Blr;  // low-rank B [N][r] in dtype blr_t, or null
  int blr_t;        // ttq_dtype of Blr
  int r;
  int64_t N, K, T;
  void* Y;
  int yt;  // ttq_dtype of Y
  int64_t ldy;
  int bn;      // tokens per tile (MMA N)
  int stages;  // pipeline depth
  int group;
  int64_t k_steps;  // ceil(K / 64)
  uint32_t* err;
};

struct SmemLayout {
  uint32_t a, b, ring, bars, tmem_slot, abort_flag, total;
};

__host__ __device__ inline SmemLayout smem_layout(int bits, int bn,
                                                  int stages) {
  SmemLayout L;
  L.a = 0;
  L.b = L.a + stages * kATileBytes;
  L.ring = L.b + stages * bn * 128;
  L.bars = L.ring + stages * ring_words(bits) * 128 * 4;
  L.tmem_slot = L.bars + (3 * stages + 1) * 8;
  L.abort_flag = L.tmem_slot + 4;
  L.total = L.abort_flag + 4;
  return L;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a,
                                             uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a),
               "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void cp_async_wait_dyn(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

__device__ __forceinline__ void store_y(void* Y, int yt, int64_t idx,
                                        float v) {
  if (yt == TTQ_BF16)
    static_cast<__nv_bfloat16*>(Y)[idx] = __float2bfloat16_rn(v);
  else if (yt == TTQ_F16)
    static_cast<__half*>(Y)[idx] = __float2half_rn(v);
  else
    static_cast<float*>(Y)[idx] = v;
}

__device__ __forceinline__ float load_any(const void* p, int t, int64_t idx) {
  if (t == TTQ_BF16)
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[idx]);
  if (t == TTQ_F16) return __half2float(static_cast<const __half*>(p)[idx]);
  return static_cast<const float*>(p)[idx];
}

// GMODE: 0 -> g = 16 (4 groups per K step), 1 -> g = 32 (2 groups),
// 2 -> g >= 64 (one group per K step).
template <int BITS, int GMODE>
__global__ void __launch_bounds__(kThreads, 1)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_u,
                       const GemmArgs p) {
  constexpr int GPS = GMODE == 0 ? 4 : (GMODE == 1 ? 2 : 1);
  constexpr int RW = ring_words(BITS);
  constexpr uint32_t QMASK = (1u << BITS) - 1u;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw_base);

  const int stages = p.stages;
  const SmemLayout L = smem_layout(BITS, p.bn, stages);
  const uint32_t bar_full_x = base + L.bars;
  const uint32_t bar_full_a = bar_full_x + 8 * stages;
  const uint32_t bar_empty = bar_full_a + 8 * stages;
  const uint32_t bar_accum = bar_empty + 8 * stages;
  volatile uint32_t* tmem_slot =
      reinterpret_cast<volatile uint32_t*>(gbase + L.tmem_slot);
  volatile int* aborted = reinterpret_cast<volatile int*>(gbase + L.abort_flag);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t t0 = (int64_t)blockIdx.y * p.bn;
  const int split = (int)gridDim.z;
  const int rank = (int)blockIdx.z;

  // K steps of this split; rank 0 also runs the low-rank stage.
  const int64_t per = (p.k_steps + split - 1) / split;
  const int64_t ks_begin =
      rank * per < p.k_steps ? rank * per : p.k_steps;
  const int64_t ks_end =
      ks_begin + per < p.k_steps ? ks_begin + per : p.k_steps;
  const int n_main = (int)(ks_end - ks_begin);
  const int n_total = n_main + ((p.r > 0 && rank == 0) ? 1 : 0);
  const uint32_t tmem_cols = p.bn < 32 ? 32u : (uint32_t)p.bn;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(bar_full_x + 8 * i, 1);
      mbar_init(bar_full_a + 8 * i, kBM);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_accum, 1);
    *aborted = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L.tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      if (p.r > 0) tma_prefetch_desc(&tmap_u);
      int issued = 0;
      const uint32_t tx = (uint32_t)p.bn * 128u;
      for (int s = 0; s < n_total; ++s) {
        const int slot = s % stages;
        const uint32_t it = (uint32_t)(s / stages);
        if (s >= stages && !mbar_wait(bar_empty + 8 * slot, (it - 1) & 1,
                                      p.err)) {
          *aborted = 1;
          break;
        }
        if (*aborted) break;
        const uint32_t dst = base + L.b + slot * p.bn * 128;
        mbar_arrive_expect_tx(bar_full_x + 8 * slot, tx);
        if (s < n_main)
          tma_load_2d(dst, &tmap_x, (int32_t)((ks_begin + s) * kBK),
                      (int32_t)t0, bar_full_x + 8 * slot);
        else
          tma_load_2d(dst, &tmap_u, 0, (int32_t)t0, bar_full_x + 8 * slot);
        issued = s + 1;
      }
      // never leave a bulk copy in flight into shared memory at exit
      for (int s = max(0, issued - stages); s < issued; ++s)
        mbar_wait(bar_full_x + 8 * (s % stages), (uint32_t)(s / stages) & 1,
                  p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kBM, p.bn);
      for (int s = 0; s < n_total; ++s) {
        const int slot = s % stages;
        const uint32_t par = (uint32_t)(s / stages) & 1;
        if (!mbar_wait(bar_full_x + 8 * slot, par, p.err) ||
            !mbar_wait(bar_full_a + 8 * slot, par, p.err)) {
          *aborted = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad = smem_desc_sw128(base + L.a + slot * kATileBytes);
        const uint64_t bd = smem_desc_sw128(base + L.b + slot * p.bn * 128);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          tc_mma_f16(tmem, ad + 2 * k, bd + 2 * k, idesc,
                     (s > 0 || k > 0) ? 1u : 0u);
        tc_commit(bar_empty + 8 * slot);
      }
      tc_commit(bar_accum);
    }
  } else {
    // ------------------------------------------------ dequantisers ----
    const int i = 32 * (warp & 3) + lane;  // weight row in the tile = TMEM lane
    const int64_t n = m0 + i;
    const bool row_ok = n < p.N;
    const int64_t row_words = p.K * BITS / 32;
    const int64_t G = p.K / p.group;
    const uint32_t* crow = p.codes + (row_ok ? n : 0) * row_words;
    const float* drow = p.delta + (row_ok ? n : 0) * G;
    const int64_t zrow = (row_ok ? n : 0) * G;
    const int64_t zend = p.N * G;
    const uint32_t ring0 = base + L.ring + 4u * i;

    auto ring_addr = [&](int slot, int w) -> uint32_t {
      return ring0 + (uint32_t)((slot * RW + w) * 128 * 4);
    };
    auto first_group = [&](int64_t k0) -> int64_t { return k0 / p.group; };

    // Stage s's codes, deltas and zero bytes into ring slot s % stages.
    auto issue = [&](int s) {
      if (s < n_main) {
        const int slot = s % stages;
        const int64_t k0 = (ks_begin + s) * kBK;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const bool ok = row_ok && (k0 + 32 * b < p.K);
#pragma unroll
          for (int w = 0; w < BITS; ++w)
            cp_async_4(ring_addr(slot, b * BITS + w),
                       ok ? crow + (k0 / 32 + b) * BITS + w : p.codes,
                       ok ? 4u : 0u);
        }
        const int64_t g0 = first_group(k0);
#pragma unroll
        for (int j = 0; j < GPS; ++j) {
          const bool ok = row_ok && (g0 + j) * p.group < p.K;
          cp_async_4(ring_addr(slot, 2 * BITS + j), ok ? drow + g0 + j : p.delta,
                     ok ? 4u : 0u);
        }
        const int64_t wa = (zrow + g0) & ~(int64_t)3;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int64_t wq = wa + 4 * q;
          const uint32_t dst = ring_addr(slot, 2 * BITS + 4 + q);
          if (row_ok && wq + 4 <= zend) {
            cp_async_4(dst, p.zero + wq, 4u);
          } else if (row_ok && wq < zend) {
            uint32_t v = 0;
            for (int b = 0; b < 4; ++b)
              if (wq + b < zend) v |= (uint32_t)p.zero[wq + b] << (8 * b);
            st_shared_u32(dst, v);
          } else {
            cp_async_4(dst, p.zero, 0u);
          }
        }
      }
      cp_async_commit();
    };

    for (int s = 0; s < stages - 1; ++s) issue(s);
    for (int s = 0; s < n_total; ++s) {
      issue(s + stages - 1);
      cp_async_wait_dyn(stages - 1);
      const int slot = s % stages;
      const uint32_t it = (uint32_t)(s / stages);
      if (s >= stages &&
          !mbar_wait(bar_empty + 8 * slot, (it - 1) & 1, p.err)) {
        *aborted = 1;
        break;
      }
      if (*aborted) break;
      const uint32_t arow = base + L.a + slot * kATileBytes + i * 128;
      const uint32_t swz = (uint32_t)(i & 7);

      if (s < n_main) {
        const int64_t k0 = (ks_begin + s) * kBK;
        uint32_t cw[2 * BITS];
#pragma unroll
        for (int w = 0; w < 2 * BITS; ++w) cw[w] = ld_shared_u32(ring_addr(slot, w));
        __half2 zsub[GPS], dh[GPS];
        const int64_t g0 = first_group(k0);
        const uint64_t zz =
            (((uint64_t)ld_shared_u32(ring_addr(slot, 2 * BITS + 5)) << 32) |
             ld_shared_u32(ring_addr(slot, 2 * BITS + 4))) >>
            (8 * ((zrow + g0) & 3));
#pragma unroll
        for (int j = 0; j < GPS; ++j) {
          const uint32_t zj = (uint32_t)(zz >> (8 * j)) & 0xFFu;
          zsub[j] = bits_h2((0x6400u | zj) * 0x00010001u);  // 1024 + z
          dh[j] = __float2half2_rn(
              __uint_as_float(ld_shared_u32(ring_addr(slot, 2 * BITS + j))));
        }
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const bool ok = k0 + 32 * blk < p.K;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[4];
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              const int c = 8 * cc + 2 * pp;  // code index in the block
              const int bit = c * BITS, wd = bit >> 5, sh = bit & 31;
              uint32_t x;
              if (sh + 2 * BITS <= 32)
                x = cw[blk * BITS + wd] >> sh;
              else
                x = __funnelshift_r(cw[blk * BITS + wd],
                                    cw[blk * BITS + wd + 1], sh);
              const uint32_t h = (x & QMASK) |
                                 ((x << (16 - BITS)) & (QMASK << 16)) |
                                 0x64006400u;  // fp16 pair (1024+q0, 1024+q1)
              const int gl = GMODE == 0 ? (32 * blk + c) / 16
                                        : (GMODE == 1 ? blk : 0);
              o[pp] = h2_bits(__hmul2(__hsub2(bits_h2(h), zsub[gl]), dh[gl]));
            }
            if (!ok) o[0] = o[1] = o[2] = o[3] = 0u;
            const uint32_t chunk = (uint32_t)(4 * blk + cc);
            st_shared_v4(arow + ((chunk ^ swz) << 4), o[0], o[1], o[2], o[3]);
          }
        }
      } else {
        // low-rank stage: row n of B (r <= 64 values) as fp16, zero padded
#pragma unroll 1
        for (int chunk = 0; chunk < 8; ++chunk) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int rho = chunk * 8 + 2 * e;
            float lo = 0.f, hi = 0.f;
            if (row_ok && rho < p.r) lo = load_any(p.Blr, p.blr_t, n * p.r + rho);
            if (row_ok && rho + 1 < p.r)
              hi = load_any(p.Blr, p.blr_t, n * p.r + rho + 1);
            o[e] = h2_bits(__floats2half2_rn(lo, hi));
          }
          st_shared_v4(arow + (((uint32_t)chunk ^ swz) << 4), o[0], o[1], o[2],
                       o[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_full_a + 8 * slot);
    }
    cp_async_wait_all();
    __syncwarp();

    // ------------------------------------------------------ epilogue ----
    const bool acc_ok = mbar_wait(bar_accum, 0, p.err);
    tc_fence_after();
    const bool ok = acc_ok && !*aborted && n_total > 0;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    if (split == 1) {
      for (int j = 0; j < p.bn; j += 16) {
        float v[16];
        tmem_ld16(t_lane + (uint32_t)j, v);
        if (ok && row_ok) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int64_t t = t0 + j + c;
            if (t < p.T) store_y(p.Y, p.yt, t * p.ldy + n, v[c]);
          }
        }
      }
    } else {
      float* part = reinterpret_cast<float*>(gbase + L.a);
      for (int j = 0; j < p.bn; j += 16) {
        float v[16];
        tmem_ld16(t_lane + (uint32_t)j, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) part[(j + c) * kBM + i] = ok ? v[c] : 0.f;
      }
    }
  }

  if (split > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && warp >= 2) {
      const int i = 32 * (warp & 3) + lane;
      const int64_t n = m0 + i;
      float* part = reinterpret_cast<float*>(gbase + L.a);
      if (n < p.N && !*aborted) {
        for (int c = 0; c < p.bn; ++c) {
          const int64_t t = t0 + c;
          if (t >= p.T) break;
          float acc = 0.f;
          for (int q = 0; q < split; ++q)
            acc += cluster.map_shared_rank(part, q)[c * kBM + i];
          store_y(p.Y, p.yt, t * p.ldy + n, acc);
        }
      }
    }
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

// X~ = fp16(X * inv_s), one thread per 8 channels.
template <typename TX>
__global__ void prescale_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                                int64_t ldx, const float* __restrict__ inv_s,
                                __half* __restrict__ Xs, uint32_t* err) {
  const int64_t chunks = K / 8;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= T * chunks) return;
  const int64_t t = id / chunks, c = (id % chunks) * 8;
  float v[8];
  load8<TX>(X + t * ldx + c, v);
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(inv_s + c));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(inv_s + c + 4));
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  uint32_t o[4];
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a = __fmul_rn(v[2 * e], sv[2 * e]);
    const float b = __fmul_rn(v[2 * e + 1], sv[2 * e + 1]);
    bad |= !(fabsf(a) < 65520.f) || !(fabsf(b) < 65520.f);
    o[e] = h2_bits(__floats2half2_rn(a, b));
  }
  *reinterpret_cast<uint4*>(Xs + t * K + c) = make_uint4(o[0], o[1], o[2], o[3]);
  if (bad) flag_error(err, TTQ_DEVERR_FP16_RANGE);
}

// U[t][rho] = fp16(sum_j X[t][j] A[rho][j]) for rho < r, 0 up to 64.
template <typename TX>
__global__ void __launch_bounds__(256)
    lowrank_u_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                     int64_t ldx, const TX* __restrict__ A, int r,
                     __half* __restrict__ U) {
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rho = warp; rho < 64; rho += 8) {
    float acc = 0.f;
    if (rho < r) {
      for (int64_t j = (int64_t)lane * 8; j < K; j += 256) {
        float xv[8], av[8];
        load8<TX>(X + t * ldx + j, xv);
        load8<TX>(A + (int64_t)rho * K + j, av);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(xv[e], av[e], acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
    }
    if (lane == 0) U[t * 64 + rho] = __float2half_rn(acc);
  }
}

// ------------------------------------------------------------ host side ---

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType,
                                   cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2D fp16 tensor [rows][inner] with the given row pitch (elements); box of
// 64 x box_rows with 128-byte swizzle; out-of-range elements read as zero.
bool make_tmap_f16(CUtensorMap* m, const void* ptr, uint64_t inner,
                   uint64_t rows, uint64_t pitch, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int BITS, int GMODE>
ttq_status launch_kernel(const CUtensorMap& tx, const CUtensorMap& tu,
                         const GemmArgs& a, dim3 grid, int split,
                         size_t smem, cudaStream_t st) {
  auto kern = lowbit_gemm_kernel<BITS, GMODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return TTQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tx, tu, a));
}

template <int GMODE>
ttq_status dispatch_bits(int bits, const CUtensorMap& tx, const CUtensorMap& tu,
                         const GemmArgs& a, dim3 grid, int split, size_t smem,
                         cudaStream_t st) {
  switch (bits) {
    case 2: return launch_kernel<2, GMODE>(tx, tu, a, grid, split, smem, st);
    case 3: return launch_kernel<3, GMODE>(tx, tu, a, grid, split, smem, st);
    case 4: return launch_kernel<4, GMODE>(tx, tu, a, grid, split, smem, st);
    case 5: return launch_kernel<5, GMODE>(tx, tu, a, grid, split, smem, st);
    case 6: return launch_kernel<6, GMODE>(tx, tu, a, grid, split, smem, st);
    case 7: return launch_kernel<7, GMODE>(tx, tu, a, grid, split, smem, st);
    case 8: return launch_kernel<8, GMODE>(tx, tu, a, grid, split, smem, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

template <typename TX>
ttq_status launch_pre(const void* X, int64_t T, int64_t K, int64_t ldx,
                      const float* inv_s, const void* A, int r, __half* Xs,
                      __half* U, cudaStream_t st) {
  const int64_t items = T * (K / 8);
  const int threads = 256;
  prescale_kernel<TX><<<(unsigned)((items + threads - 1) / threads), threads,
                        0, st>>>(static_cast<const TX*>(X), T, K, ldx, inv_s,
                                 Xs, device_error_word());
  ttq_status e = launch_status();
  if (e != TTQ_OK || r == 0) return e;
  lowrank_u_kernel<TX><<<(unsigned)T, 256, 0, st>>>(
      static_cast<const TX*>(X), T, K, ldx, static_cast<const TX*>(A), r, U);
  return launch_status();
}

}  // namespace

size_t gemm_workspace_bytes(int64_t T, int64_t K, int r) {
  size_t b = align_up((size_t)T * (size_t)K * 2, 1024);
  if (r > 0) b += align_up((size_t)T * 64 * 2, 1024);
  return b;
}

ttq_status launch_prepare(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                          int64_t ldx, const float* inv_s, const void* A,
                          int r, void* Xs, void* U, cudaStream_t st) {
  __half* xs = static_cast<__half*>(Xs);
  __half* u = static_cast<__half*>(U);
  switch (xt) {
    case TTQ_F32: return launch_pre<float>(X, T, K, ldx, inv_s, A, r, xs, u, st);
    case TTQ_BF16:
      return launch_pre<__nv_bfloat16>(X, T, K, ldx, inv_s, A, r, xs, u, st);
    case TTQ_F16: return launch_pre<__half>(X, T, K, ldx, inv_s, A, r, xs, u, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

ttq_status launch_gemm_prepared(const void* Xs, const void* U, int64_t T,
                                int64_t K, const uint32_t* codes,
                                const float* delta, const uint8_t* zero,
                                int64_t N, int bits, int group, const void* B,
                                ttq_dtype bt, int r, void* Y, ttq_dtype yt,
                                int64_t ldy, cudaStream_t st) {
  // Tile shape: decode splits K over a cluster; prefill picks the widest
  // token tile that still gives at least one CTA per SM.
  const int sms = sm_count();
  const int64_t tiles_m = (N + kBM - 1) / kBM;
  const int64_t k_steps = (K + kBK - 1) / kBK;
  int bn = 16, split = 1;
  if (T <= 16) {
    split = (int)std::min<int64_t>(
        8, std::max<int64_t>(1, (2 * sms + tiles_m - 1) / tiles_m));
    split = (int)std::min<int64_t>(split, k_steps);
    const int64_t per = (k_steps + split - 1) / split;
    split = (int)((k_steps + per - 1) / per);  // every rank gets >= 1 step
  } else if (T <= 32) {
    bn = 32;
  } else {
    bn = 64;
    const int cand[2] = {256, 128};
    for (int c : cand)
      if (tiles_m * ((T + c - 1) / c) >= sms) {
        bn = c;
        break;
      }
  }
  const int64_t tiles_t = (T + bn - 1) / bn;

  const int per_stage = kATileBytes + bn * 128 + ring_words(bits) * 128 * 4;
  const int stages = std::min(kMaxStages, (kSmemBudget - 2048) / per_stage);
  if (stages < 2) return TTQ_ERR_UNSUPPORTED;
  const SmemLayout L = smem_layout(bits, bn, stages);
  const size_t smem = L.total + 1024;

  CUtensorMap tx, tu;
  if (!make_tmap_f16(&tx, Xs, (uint64_t)K, (uint64_t)T, (uint64_t)K,
                     (uint32_t)bn))
    return TTQ_ERR_CUDA;
  if (r > 0) {
    if (!make_tmap_f16(&tu, U, 64, (uint64_t)T, 64, (uint32_t)bn))
      return TTQ_ERR_CUDA;
  } else {
    tu = tx;  // never read without a low-rank stage
  }

  GemmArgs a;
  a.codes = codes;
  a.delta = delta;
  a.zero = zero;
  a.Blr = B;
  a.blr_t = (int)bt;
  a.r = r;
  a.N = N;
  a.K = K;
  a.T = T;
  a.Y = Y;
  a.yt = (int)yt;
  a.ldy = ldy;
  a.bn = bn;
  a.stages = stages;
  a.group = group;
  a.k_steps = k_steps;
  a.err = device_error_word();
  const dim3 grid((unsigned)tiles_m, (unsigned)tiles_t, (unsigned)split);
  if (group == 16)
    return dispatch_bits<0>(bits, tx, tu, a, grid, split, smem, st);
  if (group == 32)
    return dispatch_bits<1>(bits, tx, tu, a, grid, split, smem, st);
  return dispatch_bits<2>(bits, tx, tu, a, grid, split, smem, st);
}

ttq_status launch_lowbit_gemm(const void* X, ttq_dtype xt, int64_t T,
                              int64_t K, int64_t ldx, const float* inv_s,
                              const uint32_t* codes, const float* delta,
                              const uint8_t* zero, int64_t N, int bits,
                              int group, const void* A, const void* B, int r,
                              void* Y, ttq_dtype yt, int64_t ldy,
                              void* workspace, cudaStream_t st) {
  void* Xs = workspace;
  void* U = r > 0 ? static_cast<void*>(static_cast<char*>(workspace) +
                                       align_up((size_t)T * (size_t)K * 2,
                                                1024))
                  : nullptr;
  ttq_status e = launch_prepare(X, xt, T, K, ldx, inv_s, A, r, Xs, U, st);
  if (e != TTQ_OK) return e;
  return launch_gemm_prepared(Xs, U, T, K, codes, delta, zero, N, bits, group,
                              B, xt, r, Y, yt, ldy, st);
}

}  // namespace ttq
