// quantize.cu — step 3 of TTQ: group-wise RTN of the scaled weights.
//
// TTQ review, "Proposed method", bullet 1: weights are quantized on the fly
// with group-wise round-to-nearest. Per group of g input channels of one
// weight row, in fp32 with explicit round-to-nearest-even operations (no
// contraction into FMA), as ttq.h states:
//   w = W*s;  mn = min(0, min w);  mx = max(0, max w);
//   D = (mx - mn)/(2^b - 1) (1 if 0);
//   z = clamp(rint(-mn/D));  q = clamp(rint(w*r) + z),  r = RN(1/D),
// where rint(w*r) rounds the exact product (one fused multiply-add with the
// round-to-integer offset below). The zero point takes the IEEE quotient,
// once per group. The exact product w*r lies within 2^-24 |w/D| of the
// quotient w/D, so a code can differ from rint(w/D) + z only where the
// IEEE quotient is within one fp32 step of a half-integer (a near-tie).
//
// Design (HBM-bound, kept below the instruction budget): one lane per
// 32-code block, i.e. 32 consecutive channels of one weight row, loaded as
// 64 contiguous bytes (bf16/fp16) and packed by the lane itself into its
// `bits` words, which it stores directly. Consecutive lanes take consecutive
// blocks of the [N, K/32] block grid, so a warp reads and writes contiguous
// spans. A group of g >= 32 channels spans g/32 neighbouring lanes and its
// range is a 1- or 2-level shuffle; with g = 16 a lane holds two groups.
// The IEEE divides and the reciprocal of a group run once per 32 elements.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ttq {
namespace {

constexpr int kWarpsPerCta = 8;
// scales staged in shared memory up to this size (two CTAs per SM)
constexpr int64_t kMaxStagedScaleBytes = 96 * 1024;

// Raw bytes of one block's 32 weights: 4 x 16 bytes for 16-bit types,
// 8 x 16 bytes for fp32.
template <typename TW>
struct RawBlock {
  static constexpr int V = sizeof(TW) * 32 / 16;
  uint4 v[V];
};

template <typename TW>
__device__ __forceinline__ void load_raw(const TW* p, RawBlock<TW>& r) {
#pragma unroll
  for (int i = 0; i < RawBlock<TW>::V; ++i)
    r.v[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
}

template <typename TW>
__device__ __forceinline__ void unpack_raw(const RawBlock<TW>& r,
                                           float (&w)[32]);
template <>
__device__ __forceinline__ void unpack_raw<float>(const RawBlock<float>& r,
                                                  float (&w)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w[4 * i] = __uint_as_float(r.v[i].x);
    w[4 * i + 1] = __uint_as_float(r.v[i].y);
    w[4 * i + 2] = __uint_as_float(r.v[i].z);
    w[4 * i + 3] = __uint_as_float(r.v[i].w);
  }
}
template <>
__device__ __forceinline__ void unpack_raw<__nv_bfloat16>(
    const RawBlock<__nv_bfloat16>& r, float (&w)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bf16x2_to_f32(r.v[i].x, w[8 * i], w[8 * i + 1]);
    bf16x2_to_f32(r.v[i].y, w[8 * i + 2], w[8 * i + 3]);
    bf16x2_to_f32(r.v[i].z, w[8 * i + 4], w[8 * i + 5]);
    bf16x2_to_f32(r.v[i].w, w[8 * i + 6], w[8 * i + 7]);
  }
}
template <>
__device__ __forceinline__ void unpack_raw<__half>(const RawBlock<__half>& r,
                                                   float (&w)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f16x2_to_f32(r.v[i].x, w[8 * i], w[8 * i + 1]);
    f16x2_to_f32(r.v[i].y, w[8 * i + 2], w[8 * i + 3]);
    f16x2_to_f32(r.v[i].z, w[8 * i + 4], w[8 * i + 5]);
    f16x2_to_f32(r.v[i].w, w[8 * i + 6], w[8 * i + 7]);
  }
}

// The block's BITS words at `out` (4 * BITS bytes, aligned to the largest
// power of two dividing 4 * BITS times the block index).
template <int BITS>
__device__ __forceinline__ void store_words(uint32_t* out,
                                            const uint32_t (&cw)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS; i += 4)
      *reinterpret_cast<uint4*>(out + i) =
          make_uint4(cw[i], cw[i + 1], cw[i + 2], cw[i + 3]);
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int i = 0; i < BITS; i += 2)
      *reinterpret_cast<uint2*>(out + i) = make_uint2(cw[i], cw[i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) out[i] = cw[i];
  }
}

// Row and block of the warp-relative item `lane` of a warp whose first
// item is item0: one division per warp, then at most 32/bpr + 1 steps.
__device__ __forceinline__ void locate(uint32_t item0, uint32_t bpr, int lane,
                                       uint32_t& n, uint32_t& k) {
  n = item0 / bpr;
  k = item0 - n * bpr + (uint32_t)lane;
  while (k >= bpr) {
    k -= bpr;
    ++n;
  }
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Shared-memory layout of the staged scales: block b's 32 scales at float
// offset 36 b (16 bytes of padding), so the eight lanes of a quarter-warp
// (eight consecutive blocks) read eight disjoint bank quadruples.
constexpr int kScalePitch = 36;

struct QuantCtx {
  const float* s;     // global scales (null: s = 1)
  const float* s_sm;  // staged scales, or null
  int64_t K, ldc, ldg;
  int group, lpg, lg;  // lg = log2(group)
  uint32_t* codes;
  float* delta;
  uint8_t* zero;
};

// The packing is additive: bits(M + v) = bits(M) + v for |v| < 2^22, so a
// code q placed at bit sh of a word contributes (bits(M + q - z) << sh)
// and the word is corrected once by the constant sum of (bits(M) << sh)
// minus z times the sum of (1 << sh); all mod 2^32 and exact because the
// codes' fields are disjoint. A code that straddles two words is formed
// explicitly and split.
template <int BITS>
struct PackConst {
  uint32_t cm[BITS];     // sum of bits(M) << sh over whole codes
  uint32_t sz[2][BITS];  // sum of 1 << sh over whole codes of group half
  __host__ __device__ constexpr PackConst() : cm(), sz() {
    for (int e = 0; e < 32; ++e) {
      const int bit = e * BITS, wd = bit >> 5, sh = bit & 31;
      if (sh + BITS <= 32) {
        cm[wd] += 0x4B400000u << sh;
        sz[e / 16][wd] += 1u << sh;
      }
    }
  }
};

// STAGED: the scales come from shared memory (staged per CTA, ones when s
// is null); otherwise from global memory (null: no scaling).
template <int BITS, bool G16, bool STAGED>
__device__ __forceinline__ void quantize_item(const QuantCtx& c,
                                              float (&w)[32], uint32_t n,
                                              uint32_t k, bool live) {
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int NG = G16 ? 2 : 1;  // groups held by one lane
  constexpr int E = 32 / NG;       // elements per held group
  // rint(x) for |x| < 2^22 is exactly (x + 1.5*2^23) - 1.5*2^23 under
  // round-to-nearest-even (the sum lands in [2^23, 2^24), where the ulp is
  // 1, and the offset is even).
  constexpr float kMagic = 12582912.0f;  // M = 1.5 * 2^23
  constexpr uint32_t kMagicBits = 0x4B400000u;
  constexpr float kTop = kMagic + (float)QMAX;
  constexpr PackConst<BITS> pc;

  const int64_t col0 = (int64_t)k * 32;
  if (!live) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = 0.f;
  } else if (STAGED || c.s != nullptr) {
    const float* sb = c.s_sm + k * kScalePitch;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 sv =
          STAGED ? *reinterpret_cast<const float4*>(sb + 4 * i)
                 : __ldg(reinterpret_cast<const float4*>(c.s + col0) + i);
      // two correctly rounded products per packed multiply
      const float2 p01 = __fmul2_rn(make_float2(w[4 * i], w[4 * i + 1]),
                                    make_float2(sv.x, sv.y));
      const float2 p23 = __fmul2_rn(make_float2(w[4 * i + 2], w[4 * i + 3]),
                                    make_float2(sv.z, sv.w));
      w[4 * i] = p01.x;
      w[4 * i + 1] = p01.y;
      w[4 * i + 2] = p23.x;
      w[4 * i + 3] = p23.y;
    }
  }
  // groups never straddle warp-items (32 is a multiple of group/32 and a
  // row holds whole groups), so a lane past the end never shares one with
  // a live lane

  float d[NG], r[NG], zf[NG], topz[NG], botz[NG];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    // group range, widened to contain 0 (min and max are exact, so the
    // order of the comparisons does not matter)
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int e = gi * E; e < (gi + 1) * E; e += 2) {
      mn = min3f(mn, w[e], w[e + 1]);
      mx = max3f(mx, w[e], w[e + 1]);
    }
    if constexpr (!G16) {
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {  // g <= 128: at most 4 lanes
        if (o < c.lpg) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
      }
    }
    float dd = __fdiv_rn(__fsub_rn(mx, mn), (float)QMAX);
    if (dd == 0.f) dd = 1.f;
    d[gi] = dd;
    r[gi] = __frcp_rn(dd);
    // clamp(rint(-mn / D), 0, 2^b - 1); rint(-mn / D) lies in that range
    // already because -mn <= mx - mn, the clamp matches the definition
    zf[gi] = fminf(fmaxf(__fadd_rn(__fdiv_rn(-mn, dd), kMagic), kMagic),
                   kTop) - kMagic;
    // q = clamp(rint(w*r) + z, 0, 2^b - 1) <=> M + q - z =
    // clamp(M + rint(w*r), M - z, M + 2^b - 1 - z). The lower clamp matters:
    // z is the IEEE quotient's rint(-mn/D), and where that is a near-tie
    // rint(mn*r) can fall one below -z.
    topz[gi] = kTop - zf[gi];
    botz[gi] = kMagic - zf[gi];
  }

  // code e at bits [e*BITS, e*BITS + BITS) of the block's little-endian
  // stream
  uint32_t cw[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) cw[i] = 0u;
  auto put = [&](int e, int gi, float m) {
    const float t = fmaxf(fminf(m, topz[gi]), botz[gi]);
    const uint32_t tb = __float_as_uint(t);  // bits(M) + q - z
    const int bit = e * BITS, wd = bit >> 5, sh = bit & 31;
    if (sh + BITS <= 32) {
      cw[wd] += tb << sh;
    } else {
      const uint32_t q = tb - kMagicBits + (uint32_t)zf[gi];
      cw[wd] += q << sh;
      cw[wd + 1] += q >> (32 - sh);
    }
  };
  // M + w r, two correctly rounded fused multiply-adds per instruction
  // (E is even, so a pair never straddles two groups)
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const int gi = e / E;
    const float2 m = __ffma2_rn(make_float2(w[e], w[e + 1]),
                                make_float2(r[gi], r[gi]),
                                make_float2(kMagic, kMagic));
    put(e, gi, m.x);
    put(e + 1, gi, m.y);
  }
  const uint32_t z0 = (uint32_t)zf[0], z1 = (uint32_t)zf[NG - 1];
#pragma unroll
  for (int i = 0; i < BITS; ++i)
    cw[i] = cw[i] - pc.cm[i] + z0 * pc.sz[0][i] + z1 * pc.sz[1][i];
  if (!live) return;

  uint32_t* crow = c.codes + (int64_t)n * c.ldc;
  store_words<BITS>(crow + (int64_t)k * BITS, cw);
  if (G16) {
    const int64_t gi = (int64_t)n * c.ldg + 2 * (int64_t)k;
    *reinterpret_cast<float2*>(c.delta + gi) = make_float2(d[0], d[NG - 1]);
    *reinterpret_cast<uint16_t*>(c.zero + gi) = (uint16_t)(z0 | (z1 << 8));
  } else if ((k & (uint32_t)(c.lpg - 1)) == 0) {
    const int64_t gi = (int64_t)n * c.ldg + (col0 >> c.lg);
    c.delta[gi] = d[0];
    c.zero[gi] = (uint8_t)z0;
  }
  // the lane holding the row's first block zeroes the row's padding
  if (k == 0) {
    for (int64_t w2 = c.K * BITS / 32; w2 < c.ldc; ++w2) crow[w2] = 0u;
    for (int64_t gi = c.K / c.group; gi < c.ldg; ++gi) {
      c.delta[(int64_t)n * c.ldg + gi] = 0.f;
      c.zero[(int64_t)n * c.ldg + gi] = 0;
    }
  }
}

// Position of one lane in the [N, K/32] block grid, advanced by a fixed
// number of blocks at a time (no division after the first).
struct BlockPos {
  uint32_t n, k;
  __device__ __forceinline__ void advance(uint32_t dn, uint32_t dk,
                                          uint32_t bpr) {
    n += dn;
    k += dk;
    if (k >= bpr) {
      k -= bpr;
      ++n;
    }
  }
};

// G16: group = 16 (two groups per lane); otherwise group >= 32 spans
// group/32 lanes. A persistent grid: every warp walks warp-items (32
// consecutive blocks of the [N, K/32] block grid) with a stride of the
// grid's warp count and keeps the raw weights of its next two warp-items
// in flight (one for fp32) while it quantizes the current one, so the
// loads overlap the arithmetic (about 64 KB in flight per SM).
template <typename TW, int BITS, bool G16, bool STAGED>
__global__ void __launch_bounds__(kWarpsPerCta * 32, 2)
    quantize_kernel(const TW* __restrict__ W, int64_t N, int64_t K,
                    int64_t ldw, const float* __restrict__ s, int group,
                    uint32_t* __restrict__ codes, float* __restrict__ delta,
                    uint8_t* __restrict__ zero) {
  extern __shared__ __align__(16) float s_sm[];
  griddep_enter();
  QuantCtx c;
  c.s = s;
  c.s_sm = s_sm;
  c.K = K;
  c.ldc = codes_ld(K, BITS);
  c.ldg = groups_ld(K, group);
  c.group = group;
  c.lpg = G16 ? 1 : group >> 5;
  c.lg = 31 - __clz(group);
  c.codes = codes;
  c.delta = delta;
  c.zero = zero;
  const int lane = threadIdx.x & 31;
  // warp-items are < 2^26 (the host checks N * K / 32 < 2^31)
  const uint32_t bpr = (uint32_t)(K / 32);
  const uint32_t total = (uint32_t)N * bpr;
  const uint32_t n_items = (total + 31u) / 32u;
  const uint32_t stride = gridDim.x * kWarpsPerCta;
  uint32_t wi = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const bool has_work = wi < n_items;
  // one stride of warp-items is 32 * stride blocks
  const uint32_t dn = (32u * stride) / bpr, dk = (32u * stride) % bpr;
  auto is_live = [&](uint32_t item) {
    return item * 32u + (uint32_t)lane < total;
  };
  auto load = [&](const BlockPos& q, bool live, RawBlock<TW>& raw) {
    if (live) load_raw<TW>(W + (int64_t)q.n * ldw + (int64_t)q.k * 32, raw);
  };

  // locate this lane's first block (one division per warp) and start the
  // first loads before the scales are staged: they do not depend on them.
  // Slot 0 holds the warp-item in hand, slot 1 the next one (16-bit
  // weights only; fp32 rows are twice the bytes and keep one slot).
  constexpr bool kTwoSlots = sizeof(TW) == 2;
  BlockPos p0 = {0u, 0u}, p1 = {0u, 0u};
  bool l0 = false, l1 = false;
  RawBlock<TW> raw0, raw1;
  if (has_work) {
    const uint32_t item0 = wi * 32u;
    p0.n = item0 / bpr;
    p0.k = item0 - p0.n * bpr + (uint32_t)lane;
    while (p0.k >= bpr) {
      p0.k -= bpr;
      ++p0.n;
    }
    l0 = is_live(wi);
    load(p0, l0, raw0);
    if constexpr (kTwoSlots) {
      p1 = p0;
      p1.advance(dn, dk, bpr);
      l1 = wi + stride < n_items && is_live(wi + stride);
      load(p1, l1, raw1);
    }
  }
  if constexpr (STAGED) {
    const int64_t chunks = K / 4;
    for (int64_t q = threadIdx.x; q < chunks; q += blockDim.x) {
      const float4 v = s ? __ldg(reinterpret_cast<const float4*>(s) + q)
                         : make_float4(1.f, 1.f, 1.f, 1.f);
      *reinterpret_cast<float4*>(s_sm + (q >> 3) * kScalePitch + 4 * (q & 7)) =
          v;
    }
    __syncthreads();
  }
  if (!has_work) return;  // whole warp

  float w[32];
  if constexpr (kTwoSlots) {
    // the two slots used alternately; a slot is unpacked, then refilled
    // with the warp-item two strides ahead before the arithmetic starts
    for (;;) {
      {
        unpack_raw<TW>(raw0, w);
        const BlockPos cp = p0;
        const bool cl = l0;
        p0 = p1;
        p0.advance(dn, dk, bpr);
        l0 = wi + 2 * stride < n_items && is_live(wi + 2 * stride);
        load(p0, l0, raw0);
        quantize_item<BITS, G16, STAGED>(c, w, cp.n, cp.k, cl);
      }
      wi += stride;
      if (wi >= n_items) break;
      {
        unpack_raw<TW>(raw1, w);
        const BlockPos cp = p1;
        const bool cl = l1;
        p1 = p0;
        p1.advance(dn, dk, bpr);
        l1 = wi + 2 * stride < n_items && is_live(wi + 2 * stride);
        load(p1, l1, raw1);
        quantize_item<BITS, G16, STAGED>(c, w, cp.n, cp.k, cl);
      }
      wi += stride;
      if (wi >= n_items) break;
    }
  } else {
    for (; wi < n_items; wi += stride) {
      unpack_raw<TW>(raw0, w);
      const BlockPos cp = p0;
      const bool cl = l0;
      p0.advance(dn, dk, bpr);
      l0 = wi + stride < n_items && is_live(wi + stride);
      load(p0, l0, raw0);
      quantize_item<BITS, G16, STAGED>(c, w, cp.n, cp.k, cl);
    }
  }
}

template <typename TW>
ttq_status launch_bits(const void* W, int64_t N, int64_t K, int64_t ldw,
                       const float* s, int bits, int group, uint32_t* codes,
                       float* delta, uint8_t* zero, cudaStream_t st) {
  const int64_t items = N * (K / 32);
  const int64_t warps = (items + 31) / 32;
  // persistent: as many CTAs as stay resident (2 per SM)
  const int64_t resident = (int64_t)sm_count() * 2;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  LaunchShape ls;
  ls.grid = dim3((unsigned)std::min(ctas, resident));
  ls.block = dim3(kWarpsPerCta * 32);
  // the scales go to shared memory when two CTAs per SM still fit
  const size_t s_bytes = (size_t)(K / 32) * kScalePitch * 4;
  const bool staged = (int64_t)s_bytes <= kMaxStagedScaleBytes;
  ls.smem = staged ? s_bytes : 0;
  const TW* w = static_cast<const TW*>(W);
  auto go = [&](auto kern) -> ttq_status {
    if (ls.smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)ls.smem) != cudaSuccess)
      return TTQ_ERR_CUDA;
    return launch(ls, st, kern, w, N, K, ldw, s, group, codes, delta, zero);
  };
#define TTQ_Q(B)                                                          \
  case B:                                                                 \
    return group == 16                                                    \
               ? (staged ? go(quantize_kernel<TW, B, true, true>)         \
                         : go(quantize_kernel<TW, B, true, false>))       \
               : (staged ? go(quantize_kernel<TW, B, false, true>)        \
                         : go(quantize_kernel<TW, B, false, false>));
  switch (bits) {
    TTQ_Q(2) TTQ_Q(3) TTQ_Q(4) TTQ_Q(5) TTQ_Q(6) TTQ_Q(7) TTQ_Q(8)
  }
#undef TTQ_Q
  return TTQ_ERR_INVALID_ARG;
}

// q_out[n][j] = code of channel j; one thread per 32-code block.
__global__ void unpack_kernel(const uint32_t* __restrict__ codes, int64_t N,
                              int64_t K, int bits,
                              uint8_t* __restrict__ q_out) {
  griddep_enter();
  const int64_t blocks = K / 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= N * blocks) return;
  const int64_t n = id / blocks, b = id % blocks;
  const uint32_t* w = codes + n * codes_ld(K, bits) + b * bits;
  const uint32_t mask = (1u << bits) - 1u;
  uint8_t* out = q_out + n * K + b * 32;
  for (int c = 0; c < 32; ++c) {
    const int bit = c * bits, wi = bit >> 5, sh = bit & 31;
    uint64_t v = w[wi] >> sh;
    if (sh + bits > 32) v |= (uint64_t)w[wi + 1] << (32 - sh);
    out[c] = (uint8_t)(v & mask);
  }
}

}  // namespace

ttq_status launch_quantize(const void* W, ttq_dtype wt, int64_t N, int64_t K,
                           int64_t ldw, const float* s, int bits, int group,
                           uint32_t* codes, float* delta, uint8_t* zero,
                           cudaStream_t st) {
  switch (wt) {
    case TTQ_F32:
      return launch_bits<float>(W, N, K, ldw, s, bits, group, codes, delta,
                                zero, st);
    case TTQ_BF16:
      return launch_bits<__nv_bfloat16>(W, N, K, ldw, s, bits, group, codes,
                                        delta, zero, st);
    case TTQ_F16:
      return launch_bits<__half>(W, N, K, ldw, s, bits, group, codes, delta,
                                 zero, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

ttq_status launch_unpack(const uint32_t* codes, int64_t N, int64_t K, int bits,
                         uint8_t* q_out, cudaStream_t st) {
  const int64_t total = N * (K / 32);
  LaunchShape ls;
  ls.grid = dim3((unsigned)((total + 255) / 256));
  ls.block = dim3(256);
  return launch(ls, st, unpack_kernel, codes, N, K, bits, q_out);
}

}  // namespace ttq
