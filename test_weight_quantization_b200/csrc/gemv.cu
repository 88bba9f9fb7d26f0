// gemv.cu — step 4 of TTQ for one or two tokens: the low-bit projection as
// a CUDA-core matrix-vector product (TTQ review, "Proposed method",
// bullets 1 and 7; bullet 5 for the low-rank term).
//
// A decoding step reads every packed weight once and does one multiply-add
// per weight and token, so it is bound by HBM, not by arithmetic; a
// tensor-core tile would spend a 128 x 16 x 16 MMA on a handful of real
// products per weight. The design keeps the instructions per weight few
// and every SM busy to the end:
//   - a code q of b bits that sits at bit p < 24 - b of its word (or of the
//     word shifted right by 9, or, straddling two words, funnel-shifted to
//     bit 0) is read in place: OR-ing its field into the mantissa of 1.0
//     gives 1 + q 2^(p-23). One packed subtraction of 1 (FADD2) makes two
//     codes exact q 2^(p-23), and one packed multiply-add (FFMA2) per token
//     adds x'_j q_j 2^(p_j-23) = x_j q_j for both, because the activation
//     of channel j is staged pre-multiplied by 2^(23-p_j);
//       sum_{j in grp} x_j (q_j - z) D = D (sum_j x_j q_j - z sum_j x_j);
//   - the activations (fp16, as prepared for the tensor path) are staged
//     once per CTA as fp32 in shared memory in natural channel order, with
//     the sums of every 16-channel span of the unscaled values;
//   - every CTA owns a contiguous, near-equal range of weight rows. Their
//     32-code blocks, in row-major order, are cut into one contiguous range
//     per warp of equal length (to a block), so all warps finish together;
//     a warp walks its range in chunks of 32 consecutive blocks, a lane per
//     block, with the next chunks' codes and group parameters in flight;
//   - a lane accumulates its blocks' products while they stay in the row
//     the warp is on; where a chunk crosses into the next row the warp adds
//     its lanes' sums by shuffles (fixed order) into a per-warp slot of the
//     row, and after the pass each row adds its (at most a few) warp slots
//     in warp order, with the low-rank term. The result does not depend on
//     timing.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "kperm.cuh"

namespace ttq {
namespace {

// one CTA per SM: 32 warps for one or two tokens (16 warps with twice the
// registers each for more)
__host__ __device__ constexpr int gv_threads(int nt) {
  return nt <= 2 ? 1024 : 512;
}
constexpr int kBlkPitch = 36;     // floats per staged 32-channel block
constexpr int kMaxGvTokens = 2;
constexpr int kPassRows = 1024;   // rows per pass over a CTA's range
constexpr size_t kGvSmemLimit = 200 * 1024;

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

// 1 + q 2^(pos - 23) for code I: its field OR-ed into the mantissa of 1.0.
template <int BITS, int I>
__device__ __forceinline__ float code_one(const uint32_t (&cw)[BITS],
                                          const uint32_t (&cw9)[BITS]) {
  using C = CodeAt<BITS, I>;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << C::pos;
  uint32_t src;
  if constexpr (C::kind == 0)
    src = cw[C::wd];
  else if constexpr (C::kind == 1)
    src = cw9[C::wd];
  else
    src = __funnelshift_r(cw[C::wd], cw[C::wd + 1], C::sh);
  return __uint_as_float((src & mask) | 0x3F800000u);
}

// q 2^(pos - 23) of codes I and I + 1 (exact): one packed subtraction.
template <int BITS, int I>
__device__ __forceinline__ float2 code_pair(const uint32_t (&cw)[BITS],
                                            const uint32_t (&cw9)[BITS]) {
  return __fadd2_rn(make_float2(code_one<BITS, I>(cw, cw9),
                                code_one<BITS, I + 1>(cw, cw9)),
                    make_float2(-1.f, -1.f));
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

// Adds x_j q_j over codes [I, HI) of a block, for the NT tokens whose staged
// (pre-scaled) blocks start at xb[t], into packed (even, odd) sums.
template <int BITS, int NT, int I, int HI>
__device__ __forceinline__ void dot_range(const uint32_t (&cw)[BITS],
                                          const uint32_t (&cw9)[BITS],
                                          const float* const (&xb)[NT],
                                          float2 (&acc)[NT]) {
  if constexpr (I < HI) {
    float4 xv[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
      xv[t] = *reinterpret_cast<const float4*>(xb[t] + I);
    const float2 f01 = code_pair<BITS, I>(cw, cw9);
    const float2 f23 = code_pair<BITS, I + 2>(cw, cw9);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      acc[t] = __ffma2_rn(f01, make_float2(xv[t].x, xv[t].y), acc[t]);
      acc[t] = __ffma2_rn(f23, make_float2(xv[t].z, xv[t].w), acc[t]);
    }
    dot_range<BITS, NT, I + 4, HI>(cw, cw9, xb, acc);
  }
}

template <typename TY>
__device__ __forceinline__ void put_y(void* Y, int64_t idx, float v) {
  static_cast<TY*>(Y)[idx] = from_f32<TY>(v);
}

__device__ __forceinline__ float load_b(const void* B, int bt, int64_t idx) {
  if (bt == TTQ_F32) return static_cast<const float*>(B)[idx];
  if (bt == TTQ_BF16)
    return __bfloat162float(static_cast<const __nv_bfloat16*>(B)[idx]);
  return __half2float(static_cast<const __half*>(B)[idx]);
}

// One lane's 32-code block of one chunk: its codes and group parameters.
template <int BITS>
struct BlockRegs {
  uint32_t cw[BITS];
  float d0, d1;
  uint32_t zz;
};

// Chunks of 32 blocks in flight per lane (the one being computed included),
// as many as the registers allow.
__host__ __device__ constexpr int gv_depth(int bits, int nt) {
  return bits <= 4 && nt == 1 ? 3 : 2;
}

// A lane's position in the row range of a pass: local row and block.
struct Cursor {
  int row, col;
  __device__ __forceinline__ void advance(int bpr) {
    col += 32;
    while (col >= bpr) {
      col -= bpr;
      ++row;
    }
  }
};

// Y[t][n] for t < NT. U: [NT][64] fp16 (r > 0); B: [N][r] of dtype bt.
template <int BITS, int NT, bool G16, int PERM, typename TY>
__global__ void __launch_bounds__(gv_threads(NT), 1)
    gemv_kernel(const __half* __restrict__ Xs, const __half* __restrict__ U,
                int64_t K, const uint32_t* __restrict__ codes,
                const float* __restrict__ delta,
                const uint8_t* __restrict__ zero, int64_t N, int group,
                const void* __restrict__ B, int bt, int r, void* Y,
                int64_t ldy) {
  constexpr int kThreads = gv_threads(NT);
  constexpr int kWarps = kThreads / 32;
  constexpr int D = gv_depth(BITS, NT);
  constexpr int M = kPassRows / kWarps + 2;  // rows one warp touches per pass
  extern __shared__ __align__(16) float xs_sm[];  // [NT][K/32][kBlkPitch]
  const int bpr = (int)(K / 32);
  float* span_sum = xs_sm + (size_t)NT * bpr * kBlkPitch;  // [NT][K/16]
  float* part = span_sum + (size_t)NT * 2 * bpr;         // [warps][M][NT]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t ldc = codes_ld(K, BITS), ldg = groups_ld(K, group);
  const int blk_shift = 31 - __clz(group) - 5;  // block -> group (g >= 32)
  // this CTA's rows: a near-equal contiguous share
  const int64_t row_lo = N * (int64_t)blockIdx.x / gridDim.x;
  const int64_t row_hi = N * (int64_t)(blockIdx.x + 1) / gridDim.x;

  auto load = [&](int64_t p_lo, const Cursor& c, BlockRegs<BITS>& it) {
    const int64_t n = p_lo + c.row;
    load_codes<BITS>(codes + n * ldc + (int64_t)c.col * BITS, it.cw);
    if constexpr (G16) {
      const float2 d2 =
          __ldg(reinterpret_cast<const float2*>(delta + n * ldg) + c.col);
      it.d0 = d2.x;
      it.d1 = d2.y;
      it.zz = __ldg(reinterpret_cast<const uint16_t*>(zero + n * ldg) + c.col);
    } else {
      const int gi = c.col >> blk_shift;  // g >= 32: whole blocks per group
      it.d0 = __ldg(delta + n * ldg + gi);
      it.d1 = 0.f;
      it.zz = __ldg(zero + n * ldg + gi);
    }
  };
  // sum_j x_j (q_j - z) D over the block `col` of one lane, per token
  auto block_dot = [&](const BlockRegs<BITS>& it, int col, float (&v)[NT]) {
    uint32_t cw9[BITS];
#pragma unroll
    for (int w = 0; w < BITS; ++w) cw9[w] = it.cw[w] >> 9;
    const float* xb[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) xb[t] = xs_sm + (t * bpr + col) * kBlkPitch;
    const float* ss = span_sum + 2 * col;
    if constexpr (G16) {
      // two groups of 16 in the block
      float2 a0[NT], a1[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) a0[t] = a1[t] = make_float2(0.f, 0.f);
      dot_range<BITS, NT, 0, 16>(it.cw, cw9, xb, a0);
      dot_range<BITS, NT, 16, 32>(it.cw, cw9, xb, a1);
      const float z0 = (float)(it.zz & 0xFFu);
      const float z1 = (float)(it.zz >> 8);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float s0 = a0[t].x + a0[t].y, s1 = a1[t].x + a1[t].y;
        v[t] = fmaf(it.d1, fmaf(-z1, ss[t * 2 * bpr + 1], s1),
                    it.d0 * fmaf(-z0, ss[t * 2 * bpr], s0));
      }
    } else {
      float2 a[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) a[t] = make_float2(0.f, 0.f);
      dot_range<BITS, NT, 0, 32>(it.cw, cw9, xb, a);
      const float z = (float)it.zz;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float sb = ss[t * 2 * bpr] + ss[t * 2 * bpr + 1];
        v[t] = it.d0 * fmaf(-z, sb, a[t].x + a[t].y);
      }
    }
  };

  griddep_enter();

  // Pass over up to kPassRows rows of the CTA's range. Its blocks, row-major,
  // are split into kWarps contiguous equal ranges; a warp walks its range in
  // chunks of 32 consecutive blocks (lane l takes block 32 k + l).
  int64_t p_lo = row_lo;
  int rows = (int)std::min<int64_t>(kPassRows, row_hi - p_lo);
  int nb = rows * bpr;
  int s0 = (int)((int64_t)nb * warp / kWarps);
  int s1 = (int)((int64_t)nb * (warp + 1) / kWarps);
  int n_chunks = (s1 - s0 + 31) / 32;
  Cursor ld = {(s0 + lane) / bpr, (s0 + lane) % bpr};
  BlockRegs<BITS> slot[D];
  // the first chunks' codes are requested before the activations are
  // staged (they do not depend on them)
#pragma unroll
  for (int d = 0; d < D; ++d) {
    if (d < n_chunks && s0 + 32 * d + lane < s1) load(p_lo, ld, slot[d]);
    ld.advance(bpr);
  }

  // stage x in natural channel order (undoing the K permutation) as fp32,
  // each channel pre-multiplied by 2^(23 - p) for its code's position p
  for (int64_t q = threadIdx.x; q < (int64_t)NT * (K / 16); q += kThreads) {
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

  for (;;) {
    const int first_row = s0 / bpr;
    Cursor cp = {(s0 + lane) / bpr, (s0 + lane) % bpr};
    int wr = first_row;  // the row the warp accumulates (warp-uniform)
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    // the lanes' sums of row wr, added in a fixed order, to its slot
    auto flush = [&]() {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float y = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
        if (lane == 0) part[((warp * M) + (wr - first_row)) * NT + t] = y;
      }
    };
    for (int k = 0; k < n_chunks; k += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        if (k + d < n_chunks) {
          const bool valid = s0 + 32 * (k + d) + lane < s1;
          float v[NT];
          block_dot(slot[d], valid ? cp.col : 0, v);
          // refill the slot with the chunk D ahead
          if (k + d + D < n_chunks && s0 + 32 * (k + d + D) + lane < s1)
            load(p_lo, ld, slot[d]);
          ld.advance(bpr);
          const int rb = valid ? cp.row : wr;
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[t] += (valid && rb == wr) ? v[t] : 0.f;
          while (__any_sync(0xffffffffu, rb > wr)) {
            flush();
            ++wr;
#pragma unroll
            for (int t = 0; t < NT; ++t)
              acc[t] = (valid && rb == wr) ? v[t] : 0.f;
          }
          cp.advance(bpr);
        }
      }
    }
    if (n_chunks > 0) flush();
    __syncthreads();
    // every row of the pass: the warps that cover it, in order, then the
    // low-rank term
    for (int q = threadIdx.x; q < rows * NT; q += kThreads) {
      const int lr = q / NT, t = q - lr * NT;
      const int64_t n = p_lo + lr;
      const int b0 = lr * bpr, b1 = b0 + bpr;
      float total = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const int w0 = (int)((int64_t)nb * w / kWarps);
        const int w1 = (int)((int64_t)nb * (w + 1) / kWarps);
        if (w0 < w1 && w0 < b1 && w1 > b0)
          total += part[((w * M) + (lr - w0 / bpr)) * NT + t];
      }
      if (r > 0) {
        float lr_acc = 0.f;
        for (int rho = 0; rho < r; ++rho)
          lr_acc = fmaf(__half2float(U[t * 64 + rho]),
                        load_b(B, bt, n * r + rho), lr_acc);
        total += lr_acc;
      }
      put_y<TY>(Y, t * ldy + n, total);
    }
    p_lo += rows;
    if (p_lo >= row_hi) break;
    __syncthreads();  // the partial sums were read
    rows = (int)std::min<int64_t>(kPassRows, row_hi - p_lo);
    nb = rows * bpr;
    s0 = (int)((int64_t)nb * warp / kWarps);
    s1 = (int)((int64_t)nb * (warp + 1) / kWarps);
    n_chunks = (s1 - s0 + 31) / 32;
    ld = {(s0 + lane) / bpr, (s0 + lane) % bpr};
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (d < n_chunks && s0 + 32 * d + lane < s1) load(p_lo, ld, slot[d]);
      ld.advance(bpr);
    }
  }
}

template <int BITS, int NT, bool G16, int PERM>
ttq_status launch_y(const void* Xs, const void* U, int64_t K,
                    const uint32_t* codes, const float* delta,
                    const uint8_t* zero, int64_t N, int group, const void* B,
                    ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
                    size_t smem, cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3((unsigned)std::min<int64_t>(sm_count(), N));
  ls.block = dim3(gv_threads(NT));
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
  const int warps = gv_threads((int)T) / 32;
  return (size_t)T * (size_t)(K / 32) * (kBlkPitch + 2) * sizeof(float) +
         (size_t)warps * (kPassRows / warps + 2) * (size_t)T * sizeof(float);
}

bool gemv_applies(int64_t T, int64_t K) {
  return T >= 1 && T <= kMaxGvTokens && gemv_smem_bytes(T, K) <= kGvSmemLimit;
}

ttq_status launch_gemv(const void* Xs, const void* U, int64_t T, int64_t K,
                       const uint32_t* codes, const float* delta,
                       const uint8_t* zero, int64_t N, int bits, int group,
                       const void* B, ttq_dtype bt, int r, void* Y,
                       ttq_dtype yt, int64_t ldy, cudaStream_t st) {
  const size_t smem = gemv_smem_bytes(T, K);
  switch (T) {
    case 1:
      return launch_t<1>(Xs, U, K, codes, delta, zero, N, bits, group, B, bt,
                         r, Y, yt, ldy, smem, st);
    case 2:
      return launch_t<2>(Xs, U, K, codes, delta, zero, N, bits, group, B, bt,
                         r, Y, yt, ldy, smem, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

}  // namespace ttq
