// gemv.cu — step 4 of TTQ for one or two tokens: the low-bit projection as
// a CUDA-core matrix-vector product (TTQ review, "Proposed method",
// bullets 1 and 7; bullet 5 for the low-rank term).
//
// For a decoding step the projection reads every packed weight once and
// does one multiply-add per weight and token, so it is bound by HBM, not by
// arithmetic; a tensor-core tile would spend a 128 x 16 x 16 MMA (~45-117
// cycles from one issuing thread) on 16 real products per weight. Here:
//   - a warp owns one weight row at a time and its lanes take the row's
//     32-code blocks (lane l: blocks l, l + 32, ...), the codes and group
//     parameters of several blocks in flight per lane;
//   - a code q of b bits that sits at bit p < 24 - b of its word (or of the
//     word shifted right by 9, or, straddling two words, funnel-shifted to
//     bit 0) is read in place: OR-ing its field into the mantissa of 1.0
//     gives 1 + q 2^(p-23), and subtracting 1 is exact. The activation of
//     that channel is staged pre-multiplied by 2^(23-p), so one logic op,
//     one FADD and one FMA per token make x_j q_j exactly (integer work is
//     the scarce pipe here):
//       sum_{j in blk} x_j (q_j - z) D = D sum_j x_j q_j - D z sum_j x_j;
//   - the activations (fp16, as prepared for the tensor path) are staged
//     once per CTA as fp32 in shared memory in natural channel order, with
//     the sums of every 16-channel span (of the unscaled values);
//   - the row's lanes reduce by shuffles in a fixed order (deterministic).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "kperm.cuh"

namespace ttq {
namespace {

constexpr int kGvThreads = 1024;   // one CTA per SM
constexpr int kBlkPitch = 36;      // floats per staged 32-channel block
constexpr int kMaxGvTokens = 2;

// Where code I of a 32-code block is read: kind 0 in place in its word,
// kind 1 in the word shifted right by 9, kind 2 funnel-shifted to bit 0
// (it straddles two words); pos is the field's bit in the source.
template <int BITS, int I>
struct CodeAt {
  static constexpr int bit = I * BITS, wd = bit >> 5, sh = bit & 31;
  static constexpr int kind = sh + BITS <= 23 ? 0 : sh + BITS <= 32 ? 1 : 2;
  static constexpr int pos = kind == 0 ? sh : kind == 1 ? sh - 9 : 0;
};

__host__ __device__ constexpr int code_pos(int bits, int i) {
  return ((i * bits) & 31) + bits <= 23
             ? ((i * bits) & 31)
             : ((i * bits) & 31) + bits <= 32 ? ((i * bits) & 31) - 9 : 0;
}

// q * 2^(pos - 23) for code I (exact). cwo and cw9o are the code words
// (and the words shifted right by 9) with the exponent bits of 1.0 already
// OR-ed in, once per word: since those bits lie outside every field's mask,
// (w | E) & (mask | E) = (w & mask) | E, and a code in place costs a single
// AND with one immediate.
template <int BITS, int I>
__device__ __forceinline__ float code_val(const uint32_t (&cw)[BITS],
                                          const uint32_t (&cwo)[BITS],
                                          const uint32_t (&cw9o)[BITS]) {
  using C = CodeAt<BITS, I>;
  constexpr uint32_t kOne = 0x3F800000u;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << C::pos;
  uint32_t bits;
  if constexpr (C::kind == 0)
    bits = cwo[C::wd] & (mask | kOne);
  else if constexpr (C::kind == 1)
    bits = cw9o[C::wd] & (mask | kOne);
  else
    bits = (__funnelshift_r(cw[C::wd], cw[C::wd + 1], C::sh) & mask) | kOne;
  return __fsub_rn(__uint_as_float(bits), 1.f);
}

template <int BITS>
__device__ __forceinline__ void load_codes(const uint32_t* p,
                                           uint32_t (&cw)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS; i += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p + i));
      cw[i] = v.x;
      cw[i + 1] = v.y;
      cw[i + 2] = v.z;
      cw[i + 3] = v.w;
    }
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int i = 0; i < BITS; i += 2) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p + i));
      cw[i] = v.x;
      cw[i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) cw[i] = __ldg(p + i);
  }
}

// sum over codes [I, HI) of the block of x'_j q_j 2^(pos_j - 23) = x_j q_j
// for the NT tokens whose staged (pre-scaled) blocks start at xb[t].
template <int BITS, int NT, int I, int HI>
__device__ __forceinline__ void dot_range(const uint32_t (&cw)[BITS],
                                          const uint32_t (&cwo)[BITS],
                                          const uint32_t (&cw9o)[BITS],
                                          const float* const (&xb)[NT],
                                          float (&acc)[NT]) {
  if constexpr (I < HI) {
    float4 xv[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
      xv[t] = *reinterpret_cast<const float4*>(xb[t] + I);
    const float f0 = code_val<BITS, I>(cw, cwo, cw9o);
    const float f1 = code_val<BITS, I + 1>(cw, cwo, cw9o);
    const float f2 = code_val<BITS, I + 2>(cw, cwo, cw9o);
    const float f3 = code_val<BITS, I + 3>(cw, cwo, cw9o);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      acc[t] = fmaf(f0, xv[t].x, acc[t]);
      acc[t] = fmaf(f1, xv[t].y, acc[t]);
      acc[t] = fmaf(f2, xv[t].z, acc[t]);
      acc[t] = fmaf(f3, xv[t].w, acc[t]);
    }
    dot_range<BITS, NT, I + 4, HI>(cw, cwo, cw9o, xb, acc);
  }
}

template <typename TY>
__device__ __forceinline__ void put_y(void* Y, int64_t idx, float v) {
  static_cast<TY*>(Y)[idx] = from_f32<TY>(v);
}

// Y[t][n] for t < NT. U: [NT][64] fp16 (r > 0); B: [N][r] of dtype bt.
template <int BITS, int NT, bool G16, int PERM, typename TY>
__global__ void __launch_bounds__(kGvThreads, 1)
    gemv_kernel(const __half* __restrict__ Xs, const __half* __restrict__ U,
                int64_t K, const uint32_t* __restrict__ codes,
                const float* __restrict__ delta,
                const uint8_t* __restrict__ zero, int64_t N, int group,
                const void* __restrict__ B, int bt, int r, void* Y,
                int64_t ldy) {
  // blocks in flight per lane (about 16 code words)
  constexpr int U_BLK = BITS <= 2 ? 8 : BITS <= 4 ? 4 : 2;
  extern __shared__ __align__(16) float xs_sm[];  // [NT][K/32][kBlkPitch]
  const int bpr = (int)(K / 32);
  float* span_sum = xs_sm + (size_t)NT * bpr * kBlkPitch;  // [NT][K/16]
  griddep_enter();

  // stage x in natural channel order (undoing the K permutation) as fp32
  for (int64_t q = threadIdx.x; q < (int64_t)NT * (K / 16);
       q += kGvThreads) {
    const int t = (int)(q / (K / 16));
    const int64_t span = q - (int64_t)t * (K / 16);
    const uint4* src = reinterpret_cast<const uint4*>(Xs + t * K + span * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float v[16];
#pragma unroll
    for (int e = 0; e < 8; ++e) f16x2_to_f32(w[e], v[2 * e], v[2 * e + 1]);
    // the span's sum (natural values, any order: a sum of 16 inputs)
    float sum = 0.f;
#pragma unroll
    for (int pp = 0; pp < 16; ++pp) sum += v[pp];
    span_sum[t * 2 * bpr + span] = sum;
    float* dst = xs_sm + ((size_t)t * bpr + (span >> 1)) * kBlkPitch +
                 (span & 1) * 16;
#pragma unroll
    for (int pp = 0; pp < 16; ++pp) {
      const int ch = k_perm<PERM>(pp);              // channel in the span
      const int i = (int)(span & 1) * 16 + ch;      // code index in the block
      dst[ch] = ldexpf(v[pp], 23 - code_pos(BITS, i));
    }
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t ldc = codes_ld(K, BITS), ldg = groups_ld(K, group);
  const int warps = gridDim.x * (kGvThreads / 32);
  const int cpr = (bpr + 32 * U_BLK - 1) / (32 * U_BLK);  // chunks per row
  const int blk_shift = 31 - __clz(group) - 5;  // block -> group: >> (lg g - 5)

  struct Item {
    uint32_t cw[U_BLK][BITS];
    float d0[U_BLK], d1[U_BLK];
    uint32_t zz[U_BLK];
  };
  auto fetch = [&](int64_t n, int ch, Item& it) {
    const uint32_t* crow = codes + n * ldc;
    const float* drow = delta + n * ldg;
    const uint8_t* zrow = zero + n * ldg;
#pragma unroll
    for (int u = 0; u < U_BLK; ++u) {
      const int bk = ch * 32 * U_BLK + lane + 32 * u;
      if (bk < bpr) {
        load_codes<BITS>(crow + (int64_t)bk * BITS, it.cw[u]);
        if constexpr (G16) {
          const float2 d2 = __ldg(reinterpret_cast<const float2*>(drow) + bk);
          it.d0[u] = d2.x;
          it.d1[u] = d2.y;
          it.zz[u] = __ldg(reinterpret_cast<const uint16_t*>(zrow) + bk);
        } else {
          const int gi = bk >> blk_shift;  // g >= 32: whole blocks per group
          it.d0[u] = __ldg(drow + gi);
          it.d1[u] = 0.f;
          it.zz[u] = __ldg(zrow + gi);
        }
      }
    }
  };
  float y[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) y[t] = 0.f;
  // the chunk's products, added into y
  auto compute = [&](int ch, const Item& it) {
#pragma unroll
    for (int u = 0; u < U_BLK; ++u) {
      const int bk = ch * 32 * U_BLK + lane + 32 * u;
      if (bk < bpr) {
        uint32_t cwo[BITS], cw9o[BITS];
#pragma unroll
        for (int w = 0; w < BITS; ++w) {
          cwo[w] = it.cw[u][w] | 0x3F800000u;
          cw9o[w] = (it.cw[u][w] >> 9) | 0x3F800000u;
        }
        const float* xb[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) xb[t] = xs_sm + (t * bpr + bk) * kBlkPitch;
        const float* ss = span_sum + 2 * bk;
        if constexpr (G16) {
          // two groups of 16 in the block
          float a0[NT], a1[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) a0[t] = a1[t] = 0.f;
          dot_range<BITS, NT, 0, 16>(it.cw[u], cwo, cw9o, xb, a0);
          dot_range<BITS, NT, 16, 32>(it.cw[u], cwo, cw9o, xb, a1);
          const float z0 = (float)(it.zz[u] & 0xFFu);
          const float z1 = (float)(it.zz[u] >> 8);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            y[t] = fmaf(it.d0[u], fmaf(-z0, ss[t * 2 * bpr], a0[t]), y[t]);
            y[t] = fmaf(it.d1[u], fmaf(-z1, ss[t * 2 * bpr + 1], a1[t]), y[t]);
          }
        } else {
          float a[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) a[t] = 0.f;
          dot_range<BITS, NT, 0, 32>(it.cw[u], cwo, cw9o, xb, a);
          const float z = (float)it.zz[u];
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float sb = ss[t * 2 * bpr] + ss[t * 2 * bpr + 1];
            y[t] = fmaf(it.d0[u], fmaf(-z, sb, a[t]), y[t]);
          }
        }
      }
    }
  };
  // the row's lanes add their partial sums (and the low-rank term) in a
  // fixed order; lane 0 stores the NT outputs
  auto finish = [&](int64_t n) {
    if (r > 0 && lane < r) {
      const float bv =
          bt == TTQ_F32
              ? static_cast<const float*>(B)[n * r + lane]
              : bt == TTQ_BF16
                    ? __bfloat162float(
                          static_cast<const __nv_bfloat16*>(B)[n * r + lane])
                    : __half2float(static_cast<const __half*>(B)[n * r + lane]);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        y[t] = fmaf(__half2float(U[t * 64 + lane]), bv, y[t]);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        y[t] += __shfl_xor_sync(0xffffffffu, y[t], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < NT; ++t) put_y<TY>(Y, t * ldy + n, y[t]);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) y[t] = 0.f;
  };

  for (int64_t n = blockIdx.x * (kGvThreads / 32) + (threadIdx.x >> 5); n < N;
       n += warps) {
    for (int ch = 0; ch < cpr; ++ch) {
      Item it;
      fetch(n, ch, it);
      compute(ch, it);
    }
    finish(n);
  }
}

template <int BITS, int NT, bool G16, int PERM>
ttq_status launch_y(const void* Xs, const void* U, int64_t K,
                    const uint32_t* codes, const float* delta,
                    const uint8_t* zero, int64_t N, int group, const void* B,
                    ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
                    size_t smem, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3((unsigned)std::min<int64_t>(sm_count(), (N + 31) / 32));
  ls.block = dim3(kGvThreads);
  ls.smem = smem;
  auto go = [&](auto kern) -> ttq_status {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return TTQ_ERR_CUDA;
    return launch(ls, st, kern, static_cast<const __half*>(Xs),
                  static_cast<const __half*>(U), K, codes, delta, zero, N,
                  group, B, (int)bt, r, Y, ldy);
  };
  switch (yt) {
    case TTQ_F32: return go(gemv_kernel<BITS, NT, G16, PERM, float>);
    case TTQ_BF16: return go(gemv_kernel<BITS, NT, G16, PERM, __nv_bfloat16>);
    case TTQ_F16: return go(gemv_kernel<BITS, NT, G16, PERM, __half>);
  }
  return TTQ_ERR_INVALID_ARG;
}

template <int BITS, int NT>
ttq_status launch_g(bool g16, const void* Xs, const void* U, int64_t K,
                    const uint32_t* codes, const float* delta,
                    const uint8_t* zero, int64_t N, int group, const void* B,
                    ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
                    size_t smem, cudaStream_t st) {
  constexpr int PERM = (BITS == 2 || BITS == 4 || BITS == 8) ? BITS : 0;
  return g16 ? launch_y<BITS, NT, true, PERM>(Xs, U, K, codes, delta, zero, N,
                                              group, B, bt, r, Y, yt, ldy,
                                              smem, st)
             : launch_y<BITS, NT, false, PERM>(Xs, U, K, codes, delta, zero,
                                               N, group, B, bt, r, Y, yt, ldy,
                                               smem, st);
}

template <int NT>
ttq_status launch_t(const void* Xs, const void* U, int64_t K,
                    const uint32_t* codes, const float* delta,
                    const uint8_t* zero, int64_t N, int bits, int group,
                    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt,
                    int64_t ldy, size_t smem, cudaStream_t st) {
  const bool g16 = group == 16;
#define TTQ_GV(BB)                                                           \
  case BB:                                                                   \
    return launch_g<BB, NT>(g16, Xs, U, K, codes, delta, zero, N, group, B,  \
                            bt, r, Y, yt, ldy, smem, st);
  switch (bits) {
    TTQ_GV(2) TTQ_GV(3) TTQ_GV(4) TTQ_GV(5) TTQ_GV(6) TTQ_GV(7) TTQ_GV(8)
  }
#undef TTQ_GV
  return TTQ_ERR_INVALID_ARG;
}

}  // namespace

size_t gemv_smem_bytes(int64_t T, int64_t K) {
  return (size_t)T * (size_t)(K / 32) * (kBlkPitch + 2) * sizeof(float);
}

bool gemv_applies(int64_t T, int64_t K) {
  return T >= 1 && T <= kMaxGvTokens && gemv_smem_bytes(T, K) <= 200 * 1024;
}

ttq_status launch_gemv(const void* Xs, const void* U, int64_t T, int64_t K,
                       const uint32_t* codes, const float* delta,
                       const uint8_t* zero, int64_t N, int bits, int group,
                       const void* B, ttq_dtype bt, int r, void* Y,
                       ttq_dtype yt, int64_t ldy, cudaStream_t st) {
  const size_t smem = gemv_smem_bytes(T, K);
  if (T == 1)
    return launch_t<1>(Xs, U, K, codes, delta, zero, N, bits, group, B, bt, r,
                       Y, yt, ldy, smem, st);
  return launch_t<2>(Xs, U, K, codes, delta, zero, N, bits, group, B, bt, r,
                     Y, yt, ldy, smem, st);
}

}  // namespace ttq
