// quantize.cu — step 3 of TTQ: group-wise RTN of the scaled weights.
//
// TTQ review, "Proposed method", bullet 1: weights are quantized on the fly
// with group-wise round-to-nearest. Per group of g input channels of one
// weight row, in fp32 with explicit round-to-nearest-even operations (no
// contraction into FMA), exactly as ttq.h states:
//   w = W*s;  mn = min(0, min w);  mx = max(0, max w);
//   D = (mx - mn)/(2^b - 1) (1 if 0);  r = 1/D;
//   z = clamp(rint(-mn*r));  q = clamp(rint(w*r) + z).
//
// Design (HBM-bound): one warp per 256-channel segment of a row; a lane owns
// 8 consecutive channels loaded as one 16-byte vector. A group spans g/8
// lanes and its min/max is a butterfly shuffle inside that lane segment.
// Four lanes hold one 32-code block; they exchange their 8*b-bit chunks by
// shuffles and each lane stores the one or two packed words it owns, so a
// warp writes 8*b consecutive words. Delta and zero go out from the first
// lane of each group.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ttq {
namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kSegsPerWarp = 2;  // 256-channel segments per warp

// Packs this lane's eight BITS-bit codes (chunk, codes at BITS*i) into the
// 32-code block shared by the four lanes of its quad and stores the words
// the lane owns (block words qpos and qpos + 4).
template <int BITS>
__device__ __forceinline__ void store_block(uint64_t chunk, int lane,
                                            uint32_t* out, bool active) {
  const int qpos = lane & 3;
  if constexpr (BITS == 4) {
    // eight 4-bit codes are exactly block word qpos
    if (active) out[qpos] = (uint32_t)chunk;
  } else if constexpr (BITS == 8) {
    if (active)
      *reinterpret_cast<uint2*>(out + 2 * qpos) =
          make_uint2((uint32_t)chunk, (uint32_t)(chunk >> 32));
  } else if constexpr (BITS == 2) {
    // two lanes (16 bits each) make one word
    const uint32_t hi = __shfl_down_sync(0xffffffffu, (uint32_t)chunk, 1);
    if (active && (qpos & 1) == 0)
      out[qpos >> 1] = (uint32_t)chunk | (hi << 16);
  } else {
    const int qbase = lane & ~3;
    uint64_t c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)chunk, qbase + j);
      const uint32_t hi =
          __shfl_sync(0xffffffffu, (uint32_t)(chunk >> 32), qbase + j);
      c[j] = ((uint64_t)hi << 32) | lo;
    }
    if (!active) return;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int wi = qpos + 4 * half;  // word index inside the block
      if (wi >= BITS) continue;
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int lo_bit = 8 * BITS * j;  // chunk j spans [lo_bit, +8*BITS)
        const int shift = lo_bit - 32 * wi;
        if (lo_bit + 8 * BITS <= 32 * wi || lo_bit >= 32 * wi + 32) continue;
        word |= shift >= 0 ? (uint32_t)(c[j] << shift)
                           : (uint32_t)(c[j] >> (-shift));
      }
      out[wi] = word;
    }
  }
}

template <typename TW, int BITS>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    quantize_kernel(const TW* __restrict__ W, int64_t N, int64_t K,
                    int64_t ldw, const float* __restrict__ s, int group,
                    uint32_t* __restrict__ codes, float* __restrict__ delta,
                    uint8_t* __restrict__ zero) {
  constexpr int QMAX = (1 << BITS) - 1;
  // rint(x) for |x| < 2^22 is exactly (x + 1.5*2^23) - 1.5*2^23 under
  // round-to-nearest-even (the sum lands in [2^23, 2^24), where the ulp is
  // 1, and the offset is even); the integer is the sum's low bits. Here
  // |w*r| and |mn*r| are at most 2^b - 1 + 1/2.
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr int kMagicBits = 0x4B400000;
  using chunk_t = typename std::conditional<(8 * BITS <= 32), uint32_t,
                                            uint64_t>::type;
  griddep_enter();
  const int lane = threadIdx.x & 31;
  // work items are (row, 256-channel segment) pairs, < 2^31 (checked on
  // the host); 32-bit index math keeps the per-item cost small
  const uint32_t segs = (uint32_t)((K + 255) / 256);
  const uint32_t items = (uint32_t)N * segs;
  const uint32_t item0 =
      (blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5)) * kSegsPerWarp;
  if (item0 >= items) return;  // whole warp exits together
  const int64_t ldc = codes_ld(K, BITS), ldg = groups_ld(K, group);
  const int lanes_per_group = group >> 3;

  // issue every segment's loads first
  float w[kSegsPerWarp][8];
  int64_t n_[kSegsPerWarp], col_[kSegsPerWarp];
  bool act_[kSegsPerWarp];
  const uint32_t row0 = item0 / segs, seg0 = item0 - row0 * segs;
#pragma unroll
  for (int u = 0; u < kSegsPerWarp; ++u) {
    const uint32_t item = item0 + u;
    const bool live = item < items;
    uint32_t row = row0, seg = seg0 + u;
    if (seg >= segs) {  // kSegsPerWarp <= segs is not required
      row += seg / segs;
      seg %= segs;
    }
    n_[u] = live ? row : 0;
    col_[u] = live ? (int64_t)seg * 256 + lane * 8 : K;
    act_[u] = live && col_[u] < K;  // K % 32 == 0: blocks/groups agree
    if (act_[u]) {
      load8<TW>(W + n_[u] * ldw + col_[u], w[u]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[u][i] = 0.f;
    }
  }

#pragma unroll
  for (int u = 0; u < kSegsPerWarp; ++u) {
    const int64_t n = n_[u], col0 = col_[u];
    const bool active = act_[u];
    if (active && s != nullptr) {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + col0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + col0 + 4));
      w[u][0] = __fmul_rn(w[u][0], s0.x); w[u][1] = __fmul_rn(w[u][1], s0.y);
      w[u][2] = __fmul_rn(w[u][2], s0.z); w[u][3] = __fmul_rn(w[u][3], s0.w);
      w[u][4] = __fmul_rn(w[u][4], s1.x); w[u][5] = __fmul_rn(w[u][5], s1.y);
      w[u][6] = __fmul_rn(w[u][6], s1.z); w[u][7] = __fmul_rn(w[u][7], s1.w);
    }
    // group range, widened to contain 0
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mn = fminf(mn, w[u][i]);
      mx = fmaxf(mx, w[u][i]);
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {  // g <= 128: at most 16 lanes
      if (o < lanes_per_group) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
    }
    float d = __fdiv_rn(__fsub_rn(mx, mn), (float)QMAX);
    if (d == 0.f) d = 1.f;
    const float r = __frcp_rn(d);
    // z = rint(-mn * r) lies in [0, 2^b - 1] because -mn <= mx - mn; the
    // clamp below matches the definition and never changes a value
    const int zi = min(max(__float_as_int(__fadd_rn(__fmul_rn(-mn, r), kMagic)) -
                               kMagicBits,
                           0),
                       QMAX);
    // q = rint(w*r) + z >= rint(mn*r) + z = 0 since rint is odd and the
    // products are monotone in w; only the upper clamp can act
    chunk_t chunk = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int qi = __float_as_int(__fadd_rn(__fmul_rn(w[u][i], r), kMagic)) -
                     (kMagicBits - zi);
      chunk |= (chunk_t)(uint32_t)min(qi, QMAX) << (BITS * i);
    }
    store_block<BITS>((uint64_t)chunk, lane,
                      codes + n * ldc + (col0 / 32) * BITS, active);
    if (active && (lane & (lanes_per_group - 1)) == 0) {
      const int64_t gi = n * ldg + col0 / group;
      delta[gi] = d;
      zero[gi] = (uint8_t)zi;
    }
    // the warp holding the row's first segment zeroes the row's padding
    if (col0 == lane * 8 && item0 + u < items) {
      for (int64_t w2 = K * BITS / 32 + lane; w2 < ldc; w2 += 32)
        codes[n * ldc + w2] = 0u;
      for (int64_t gi = K / group + lane; gi < ldg; gi += 32) {
        delta[n * ldg + gi] = 0.f;
        zero[n * ldg + gi] = 0;
      }
    }
  }
}

template <typename TW>
ttq_status launch_bits(const void* W, int64_t N, int64_t K, int64_t ldw,
                       const float* s, int bits, int group, uint32_t* codes,
                       float* delta, uint8_t* zero, cudaStream_t st) {
  const int64_t items = N * ((K + 255) / 256);
  const int64_t warps = (items + kSegsPerWarp - 1) / kSegsPerWarp;
  LaunchShape ls;
  ls.grid = dim3((unsigned)((warps + kWarpsPerCta - 1) / kWarpsPerCta));
  ls.block = dim3(kWarpsPerCta * 32);
  const TW* w = static_cast<const TW*>(W);
#define TTQ_Q(B)                                                            \
  case B:                                                                   \
    return launch(ls, st, quantize_kernel<TW, B>, w, N, K, ldw, s, group,   \
                  codes, delta, zero);
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
