// gemm.cu — step 4 of TTQ: the quantized projection on 5th-generation
// tensor cores, with dequantisation inside the GEMM.
//
// TTQ review, "Proposed method", bullets 1 and 7 (QDQ weights; a GPU kernel
// for the quantized projection) and bullet 5 (optional W = W_q + B A):
//   Y = (X diag(1/s)) W_hat_s^T + (X A^T) B^T,  W_hat_s = (q - z) * D.
//
// Orientation: the weight rows are the MMA's M dimension (128 TMEM lanes)
// and the tokens its N dimension (16..256 TMEM columns), so one dequantised
// 128 x 128 weight stage feeds up to 256 tokens. Operands are fp16: the
// activations are scaled by 1/s and rounded once to fp16 by a pre-pass
// (prescale_kernel), each weight (q - z) * D is rounded once to fp16 in the
// dequantiser; products accumulate in fp32 in TMEM.
//
// CTA = producer warp + MMA warp + 16 dequantiser warps (prefill, one CTA
// per SM) or 4 (decode, two CTAs per SM). Shared-memory rings filled by the
// tensor memory accelerator (TMA) and drained in K order by stage:
//   X~ ring      two 64-channel fp16 activation boxes (128B swizzle)
//   codes ring   128 rows x 128 channels of packed codes
//   params ring  128 rows x 16 groups of delta (fp32) and zero (u8)
// The dequantisers write each fp16 weight stage straight to a TMEM ring
// (tcgen05.st; a thread = a weight row = a TMEM lane) and the MMA warp's
// elected thread consumes it with the A-from-TMEM form of tcgen05.mma
// (fp16 pairs are built with the 1024+q exponent trick). Epilogue: the
// accumulator leaves TMEM in 16x256b fragment order, is packed to 16-bit
// pairs and written transposed by stmatrix into 128-byte-swizzled boxes of
// the idle activation ring, and a TMA tensor store writes Y. Decode
// (T <= 32 where gemv.cu, which takes one or two tokens, does not apply)
// splits K over a cluster of up to 8 CTAs whose partial tiles every rank
// reduces in part through distributed shared memory, in rank order. The rank-r low-rank term is one
// extra K stage, [X~ | U] [W_hat | B]^T with U = X A^T (fp16, from
// lowrank_u_kernel). Every wait is bounded (TTQ_DEVERR_TIMEOUT, then the CTA
// winds down).
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "kperm.cuh"

namespace cg = cooperative_groups;

namespace ttq {
namespace {

constexpr int kBM = 128;           // weight rows per CTA (TMEM lanes)
constexpr int kSK = 128;           // channels per pipeline stage
constexpr int kSCols = kSK / 2;    // TMEM columns of one fp16 weight stage
constexpr int kParamGroups = 16;   // groups per params chunk
// CTA = producer warp + MMA warp + DQW dequantiser warps (4, 8 or 16; with
// 8 or 16, two or four warps share each TMEM lane quarter and split every
// stage into parts of 64 or 32 channels)
constexpr int kDqWarp0 = 2;  // first dequantiser warp
// dequantiser warps of the prefill form (four per SM sub-partition, so that
// one warp's dependent chain of shared-memory loads, unpacking and TMEM
// stores overlaps the others')
constexpr int kPrefillDequantWarps = 16;
__host__ __device__ constexpr int cta_threads(int dqw) {
  return 32 * (kDqWarp0 + dqw);
}
constexpr int kParamDeltaBytes = kBM * kParamGroups * 4;
constexpr int kParamBytes = kParamDeltaBytes + kBM * kParamGroups;
constexpr int kMaxSmem = 225 * 1024;

struct GemmArgs {
  const void* Blr;  // low-rank B [N][r] in dtype blr_t, or null
  int blr_t;
  int r;
  int N, K, T;
  void* Y;
  int yt;  // ttq_dtype of Y
  long long ldy;
  int bn;         // tokens per tile (MMA N)
  int S;          // shared-memory ring depth (stages of 128 channels)
  int SA;         // TMEM weight-stage ring depth (<= S)
  int tmem_cols;  // TMEM allocation: accumulator + S weight stages
  int acc_cols;   // TMEM columns reserved for the accumulator
  int group;
  int k_stages;   // ceil(K / 128)
  int per;        // stages per split rank
  // fused quantization (QDQ form): the scales, and where the first token
  // tile's CTAs store the codes, delta and zero (null: not stored)
  const float* qs;
  uint32_t* q_codes;
  float* q_delta;
  uint8_t* q_zero;
  long long q_ldc, q_ldg;
  float* stats;   // per-row partial sums of |Y|^stats_p, or null
  float stats_p;
  int stats_parts;  // partial rows per token tile (1 or 2)
  int y_mode;     // 0: per-row stores (rows not 16-byte aligned);
                  // 1: staged tile [tokens][128] stored through tm_y;
                  // 2: 16-bit Y staged by stmatrix in 128-byte swizzled
                  //    boxes of 64 rows, two stores per group
  uint32_t* err;
};

__host__ __device__ inline uint32_t code_chunk_bytes(int bits) {
  return (uint32_t)(kBM * 16 * bits);  // 128 rows x 4*bits words
}

struct Layout {
  uint32_t x, c, p, part, bars, tmem, abort_flag, total, stage_x;
};

// bf16 weight tile of one stage in the fused (QDQ) form: two 64-channel
// boxes of 128 rows, 128-byte swizzled
constexpr uint32_t kWStageBytes = 2u * kBM * 128u;
// group-range exchange of the fused form: [2 stage parities][4 parts]
// [128 rows] (min, max)
constexpr uint32_t kXchgBytes = 2u * 4u * kBM * 8u;

// Shared memory: per stage two 64-channel activation boxes and one codes
// chunk (the bf16 weight tile in the fused form); two params slots (the
// group-range exchange in the fused form); the split-K partial tile
// (decode); barriers. The fp16 weight stages live in TMEM.
__host__ __device__ inline Layout make_layout(int bits, int bn, int S,
                                              bool split, bool qdq = false,
                                              int extra_bars = 0) {
  Layout L;
  L.stage_x = (uint32_t)(2 * bn * 128);
  L.x = 0;
  L.c = L.x + (uint32_t)S * L.stage_x;
  L.p = L.c + (uint32_t)S * (qdq ? kWStageBytes : code_chunk_bytes(bits));
  L.part = L.p + (qdq ? kXchgBytes : 2u * kParamBytes);
  L.bars = L.part + (split ? (uint32_t)(bn * kBM * 4) : 0u);
  // loaded, ready, empty, a_free; params; accumulator; the fused form's
  // group-range exchange (4 lane quarters x 2 stage parities)
  const int nbars = 3 * S + S + 4 + 1 + (qdq ? 8 : 0) + extra_bars;
  L.tmem = L.bars + 8u * nbars;
  L.abort_flag = L.tmem + 4;
  L.total = L.abort_flag + 4;
  return L;
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_shared_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// The BITS words of one 32-code block, with the widest aligned loads.
template <int BITS>
__device__ __forceinline__ void load_block(uint32_t addr, uint32_t (&w)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int k = 0; k < BITS; k += 4)
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(w[k]), "=r"(w[k + 1]), "=r"(w[k + 2]), "=r"(w[k + 3])
                   : "r"(addr + 4 * k)
                   : "memory");
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int k = 0; k < BITS; k += 2)
      asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];"
                   : "=r"(w[k]), "=r"(w[k + 1])
                   : "r"(addr + 4 * k)
                   : "memory");
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = ld_shared_u32(addr + 4 * k);
  }
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

__device__ __forceinline__ void store_y(void* Y, int yt, long long idx,
                                        float v) {
  if (yt == TTQ_BF16)
    static_cast<__nv_bfloat16*>(Y)[idx] = __float2bfloat16_rn(v);
  else if (yt == TTQ_F16)
    static_cast<__half*>(Y)[idx] = __float2half_rn(v);
  else
    static_cast<float*>(Y)[idx] = v;
}

// The value Y stores for v (rounded to its dtype), as fp32.
__device__ __forceinline__ float stored_y(int yt, float v) {
  if (yt == TTQ_BF16) return __bfloat162float(__float2bfloat16_rn(v));
  if (yt == TTQ_F16) return __half2float(__float2half_rn(v));
  return v;
}

// |y|^p of the fused output statistic.
__device__ __forceinline__ float y_moment(float y, float p) {
  if (p == 2.f) return y * y;
  if (p == 1.f) return fabsf(y);
  return powf(fabsf(y), p);
}

__device__ __forceinline__ float load_any(const void* p, int t, long long idx) {
  if (t == TTQ_BF16)
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[idx]);
  if (t == TTQ_F16) return __half2float(static_cast<const __half*>(p)[idx]);
  return static_cast<const float*>(p)[idx];
}

// Dequantises one 32-code block (BITS words in cw) into the 16 fp16 pairs
// o[0..15], o[p] holding block positions 2p and 2p+1: w = (q - z) * D, each
// pair built as fp16 (1024 + q) by OR-ing the code into the mantissa, then
// (1024 + q) - (1024 + z), then times D (one fp16 rounding). Written as
// four passes over all 16 pairs (extract, subtract, multiply) so that the
// independent pairs interleave instead of running as 16 dependent chains.
template <int BITS, int GMODE>
__device__ __forceinline__ void dequant_block(const uint32_t (&cw)[BITS],
                                              const __half2* zsub,
                                              const __half2* dh,
                                              uint32_t* o) {
  constexpr uint32_t QMASK = (1u << BITS) - 1u;
  uint32_t x[16];
  if constexpr (BITS == 2 || BITS == 4 || BITS == 8) {
    // codes c and c + 16/BITS sit 16 bits apart in one word: one shift and
    // mask yield the pair; positions follow k_perm<BITS>
    constexpr int PER_WORD = 32 / BITS;   // codes per word
    constexpr int PAIRS = PER_WORD / 2;   // pairs per word
    constexpr uint32_t PMASK = QMASK | (QMASK << 16);
#pragma unroll
    for (int wd = 0; wd < BITS; ++wd)
#pragma unroll
      for (int j = 0; j < PAIRS; ++j)
        x[wd * PAIRS + j] = ((cw[wd] >> (BITS * j)) & PMASK) | 0x64006400u;
  } else {
#pragma unroll
    for (int pp = 0; pp < 16; ++pp) {
      const int c = 2 * pp;  // code index in the block
      const int bit = c * BITS, wd = bit >> 5, sh = bit & 31;
      uint32_t v;
      if (sh + 2 * BITS <= 32)
        v = cw[wd] >> sh;
      else
        v = __funnelshift_r(cw[wd], cw[wd + 1], sh);
      x[pp] = (v & QMASK) | ((v << (16 - BITS)) & (QMASK << 16)) | 0x64006400u;
    }
  }
  // group of pair p (g = 16 splits a block into two groups)
  auto grp = [&](int pp) -> int {
    if constexpr (GMODE != 0) return 0;
    if constexpr (BITS == 2 || BITS == 4 || BITS == 8)
      return (pp / (16 / BITS)) * (32 / BITS) / 16;  // word's first code
    return (2 * pp) / 16;
  };
  __half2 t[16];
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) t[pp] = __hsub2(bits_h2(x[pp]), zsub[grp(pp)]);
#pragma unroll
  for (int pp = 0; pp < 16; ++pp) o[pp] = h2_bits(__hmul2(t[pp], dh[grp(pp)]));
}

// One arrival on `bar` for the whole warp, made by lane 0 once every lane
// has come here: a barrier then counts warps, not threads, and takes one
// shared-memory update per warp instead of 32.
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Position in a ring of `depth` slots: the slot and how many times the
// ring has wrapped (its parity is the mbarrier phase of the slot's use).
struct Ring {
  int slot = 0;
  uint32_t round = 0;
  __device__ __forceinline__ void next(int depth) {
    if (++slot == depth) {
      slot = 0;
      ++round;
    }
  }
};

// Stage protocol (slot = stage % S):
//   producer   waits `empty` (previous use done), then loads the codes
//              chunk and both activation boxes, completing on `loaded`;
//   dequant    waits `loaded`, writes the fp16 weight stage to TMEM, then
//              arrives on `ready`, once per warp (this also vouches that
//              the activations have landed, since it observed `loaded`);
//   MMA        waits `ready`, issues 8 MMAs, commits to `empty`, which frees
//              the codes, the activations and the TMEM weight stage at once.
// GMODE: 0 -> g = 16 (a 32-code block spans 2 groups), 1 -> g >= 32.
// QDQ: the fused form. The producer loads bf16 weight tiles instead of
// codes, and the dequantiser warps quantize them on the fly (the same
// arithmetic as quantize.cu), store the codes, delta and zero of the first
// token tile for later use, and hand the dequantised fp16 weights to the
// tensor cores as usual (TTQ review, Proposed method, bullet 1: QDQ).
template <int BITS, int GMODE, int DQW, bool QDQ>
__global__ void __launch_bounds__(cta_threads(DQW), DQW >= 16 ? 1 : 2)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_u,
                       const __grid_constant__ CUtensorMap tm_c,
                       const __grid_constant__ CUtensorMap tm_d,
                       const __grid_constant__ CUtensorMap tm_z,
                       const __grid_constant__ CUtensorMap tm_y,
                       const __grid_constant__ CUtensorMap tm_w,
                       const GemmArgs p) {
  constexpr int GPB = GMODE == 0 ? 2 : 1;  // groups per 32-code block
  constexpr uint32_t CHUNK = QDQ ? kWStageBytes : kBM * 16 * BITS;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw_base);

  const int S = p.S, SA = p.SA, bn = p.bn;
  const int split = (int)gridDim.z;
  const Layout L = make_layout(BITS, bn, S, split > 1, QDQ);
  const uint32_t b_loaded = base + L.bars;
  const uint32_t b_ready = b_loaded + 8 * S;
  const uint32_t b_empty = b_ready + 8 * S;
  const uint32_t b_afree = b_empty + 8 * S;
  const uint32_t b_full_p = b_afree + 8 * S;
  const uint32_t b_empty_p = b_full_p + 16;
  const uint32_t b_accum = b_empty_p + 16;
  const uint32_t b_xchg = b_accum + 8;  // fused form: [lane quarter][parity]
  volatile uint32_t* tmem_slot =
      reinterpret_cast<volatile uint32_t*>(gbase + L.tmem);
  volatile int* aborted = reinterpret_cast<volatile int*>(gbase + L.abort_flag);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;
  const int t0 = blockIdx.y * bn;
  const int rank = (int)blockIdx.z;
  const int ks_begin = min(rank * p.per, p.k_stages);
  const int ks_end = min(ks_begin + p.per, p.k_stages);
  const int n_main = ks_end - ks_begin;
  const int n_total = n_main + ((p.r > 0 && rank == 0) ? 1 : 0);
  const int lg = 31 - __clz(p.group);  // log2(g)

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(b_loaded + 8 * i, 1);
      mbar_init(b_ready + 8 * i, DQW);
      mbar_init(b_empty + 8 * i, 1);
      mbar_init(b_afree + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_full_p + 8 * i, 1);
      mbar_init(b_empty_p + 8 * i, DQW);
    }
    mbar_init(b_accum, 1);
    if constexpr (QDQ) {
      for (int i = 0; i < 8; ++i) mbar_init(b_xchg + 8 * i, 128);
    }
    *aborted = 0;
    fence_barrier_init();
    // the tensor maps are kernel parameters: no need to wait for them
    tma_prefetch_desc(&tm_x);
    if constexpr (QDQ) {
      tma_prefetch_desc(&tm_w);
    } else {
      tma_prefetch_desc(&tm_c);
      tma_prefetch_desc(&tm_d);
      tma_prefetch_desc(&tm_z);
    }
    if (p.r > 0) tma_prefetch_desc(&tm_u);
  }
  // The set-up above and the TMEM allocation touch no global memory, so
  // they overlap the previous kernel on the stream. (An allocation can
  // only wait for TMEM of a CTA that is already running on this SM, which
  // releases it when it ends.) Everything after the wait may read what
  // earlier kernels wrote.
  if (warp == 1) {
    tmem_alloc(base + L.tmem, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_enter();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a = tmem + (uint32_t)p.acc_cols;  // weight-stage ring

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      const uint32_t xbytes = (uint32_t)bn * 128u;
      Ring rs, rp;
      int pchunk = -1, issued = 0, np = 0;
      bool ok = true;
      for (int s = 0; s < n_total; ++s) {
        const int k0 = (ks_begin + s) * kSK;
        if (!QDQ && s < n_main) {
          const int pc = k0 >> (lg + 4);  // params chunk: 16 groups
          if (pc != pchunk) {
            if (pchunk >= 0) rp.next(2);
            pchunk = pc;
            if (np >= 2 && !mbar_wait(b_empty_p + 8 * rp.slot,
                                      (rp.round & 1) ^ 1, p.err)) {
              ok = false;
              break;
            }
            const uint32_t bar = b_full_p + 8 * rp.slot;
            const uint32_t dst = base + L.p + rp.slot * kParamBytes;
            mbar_arrive_expect_tx(bar, kParamBytes);
            tma_load_2d(dst, &tm_d, pc * kParamGroups, m0, bar);
            tma_load_2d(dst + kParamDeltaBytes, &tm_z, pc * kParamGroups, m0,
                        bar);
            ++np;
          }
        }
        if (s >= S &&
            !mbar_wait(b_empty + 8 * rs.slot, (rs.round & 1) ^ 1, p.err)) {
          ok = false;
          break;
        }
        if (*aborted) break;
        const uint32_t bar = b_loaded + 8 * rs.slot;
        const uint32_t xdst = base + L.x + rs.slot * L.stage_x;
        if (s < n_main) {
          mbar_arrive_expect_tx(bar, CHUNK + 2 * xbytes);
          const uint32_t cdst = base + L.c + rs.slot * CHUNK;
          if constexpr (QDQ) {
            tma_load_2d(cdst, &tm_w, k0, m0, bar);
            tma_load_2d(cdst + CHUNK / 2, &tm_w, k0 + 64, m0, bar);
          } else {
            tma_load_2d(cdst, &tm_c, (k0 >> 7) * 4 * BITS, m0, bar);
          }
          tma_load_2d(xdst, &tm_x, k0, t0, bar);
          tma_load_2d(xdst + xbytes, &tm_x, k0 + 64, t0, bar);
        } else {
          mbar_arrive_expect_tx(bar, xbytes);
          tma_load_2d(xdst, &tm_u, 0, t0, bar);
        }
        rs.next(S);
        issued = s + 1;
      }
      if (!ok) *aborted = 1;
      // never leave a bulk copy in flight into shared memory at exit: wait
      // for the last use of every slot that was loaded
      for (int i = 0; i < S && i < issued; ++i) {
        const int q = issued - 1 - i;
        mbar_wait(b_loaded + 8 * (q % S), (uint32_t)(q / S) & 1, p.err);
      }
      for (int i = 0; i < 2 && i < np; ++i) {
        const int q = np - 1 - i;
        mbar_wait(b_full_p + 8 * (q & 1), (uint32_t)(q >> 1) & 1, p.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    // (Issuing a stage's MMAs from several warps into separate accumulators
    // was measured slower for the decode tile: 21.9 against 19.3 us on
    // 14336 x 4096 at 16 tokens.)
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kBM, bn);
      const uint32_t xbytes = (uint32_t)bn * 128u;
      Ring rs, ra;
      for (int s = 0; s < n_total; ++s) {
        if (!mbar_wait(b_ready + 8 * rs.slot, rs.round & 1, p.err)) {
          *aborted = 1;
          break;
        }
        tc_fence_after();
        const uint32_t ad = tmem_a + (uint32_t)(ra.slot * kSCols);
        const uint32_t xs = base + L.x + rs.slot * L.stage_x;
        const uint64_t bd0 = smem_desc_sw128(xs);
        const uint64_t bd1 = smem_desc_sw128(xs + xbytes);
        // the stage's eight K steps back to back (four for the low-rank
        // stage)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_f16_ts(tmem, ad + 8 * k, bd0 + 2 * k, idesc,
                        (s > 0 || k > 0) ? 1u : 0u);
        if (s < n_main) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ts(tmem, ad + 32 + 8 * k, bd1 + 2 * k, idesc, 1u);
        }
        tc_commit(b_empty + 8 * rs.slot);
        tc_commit(b_afree + 8 * ra.slot);
        rs.next(S);
        ra.next(SA);
      }
      tc_commit(b_accum);
    }
  } else {
    // ------------------------------------------------ dequantisers ----
    // One thread per weight row (= TMEM lane): a stage is four 32-code
    // blocks, 64 fp16 pairs, written to the TMEM weight ring; the DQW / 4
    // warps of a lane quarter take equal parts of it.
    constexpr int kParts = DQW / 4;
    const int q4 = warp & 3;                // TMEM lane quarter of this warp
    const int h = (warp - kDqWarp0) >> 2;   // which part of a stage
    const int i = 32 * q4 + lane;    // weight row in the tile = TMEM lane
    const int n = m0 + i;
    const bool row_ok = n < p.N;
    const int half_lo = kParts == 2 ? h : 0, half_hi = kParts == 2 ? h + 1 : 2;
    const uint32_t crow = base + L.c + i * 16 * BITS;
    // delta tile: 64-byte rows in the 64B swizzle (16-byte chunk index XOR
    // bits 1-2 of the row); zero tile: plain 16-byte rows
    const uint32_t drow = base + L.p + i * 64;
    const uint32_t dswz = (uint32_t)((i >> 1) & 3);
    const uint32_t zrow = base + L.p + kParamDeltaBytes + i * 16;
    const uint32_t arow = tmem_a + ((uint32_t)(32 * q4) << 16);
    Ring rs, ra, rp;
    int pchunk = -1;
    bool ok_loop = true;

    // The fused (QDQ) form of a main stage: this warp's 32 channels (block
    // h of the stage) of row i, quantized from the bf16 tile exactly as
    // quantize.cu does, dequantised as the codes path does, stored to TMEM;
    // the first token tile also stores the codes, delta and zero.
    auto qdq_stage = [&](int s, int k0, uint32_t acol) {
      if constexpr (QDQ) {
        static_assert(DQW == 16, "the fused form uses 16 dequantiser warps");
        constexpr int QMAX = (1 << BITS) - 1;
        constexpr float kMagic = 12582912.0f;  // rint by 1.5 * 2^23
        constexpr float kTop = kMagic + (float)QMAX;
        constexpr int NG = GMODE == 0 ? 2 : 1;  // groups in the block
        constexpr int E = 32 / NG;
        constexpr int PERM = (BITS == 2 || BITS == 4 || BITS == 8) ? BITS : 0;
        // raw bf16 weights: box h >> 1, 16-byte chunks (h & 1) * 4 .. + 3
        // of row i, stored at chunk ^ (i % 8) (128-byte swizzle)
        const uint32_t wrow = base + L.c + rs.slot * CHUNK +
                              (uint32_t)(h >> 1) * (CHUNK / 2) +
                              (uint32_t)i * 128u;
        float w[32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t c = (uint32_t)((h & 1) * 4 + cc);
          uint32_t v[4];
          asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                       : "r"(wrow + ((c ^ ((uint32_t)i & 7u)) << 4))
                       : "memory");
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[8 * cc + 2 * e] = __uint_as_float(v[e] << 16);
            w[8 * cc + 2 * e + 1] = __uint_as_float(v[e] & 0xFFFF0000u);
          }
        }
        // w = W * s (the same scale for every row: broadcast loads); a
        // block past K (the last stage's tail) holds zeros from the tile
        // load and keeps them
        const bool in_k = k0 + 32 * h < p.K;
        const float4* sp = reinterpret_cast<const float4*>(
            p.qs + (in_k ? k0 + 32 * h : 0));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 sv = in_k ? __ldg(sp + q) : make_float4(0.f, 0.f, 0.f,
                                                               0.f);
          const float2 a = __fmul2_rn(make_float2(w[4 * q], w[4 * q + 1]),
                                      make_float2(sv.x, sv.y));
          const float2 b = __fmul2_rn(make_float2(w[4 * q + 2], w[4 * q + 3]),
                                      make_float2(sv.z, sv.w));
          w[4 * q] = a.x;
          w[4 * q + 1] = a.y;
          w[4 * q + 2] = b.x;
          w[4 * q + 3] = b.y;
        }
        // group ranges widened to contain 0; groups of 64 or 128 channels
        // span two or four warps of this lane quarter, which exchange their
        // parts through shared memory (two slots by stage parity)
        float mn[NG], mx[NG];
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
          mn[gi] = 0.f;
          mx[gi] = 0.f;
#pragma unroll
          for (int e = gi * E; e < (gi + 1) * E; ++e) {
            mn[gi] = fminf(mn[gi], w[e]);
            mx[gi] = fmaxf(mx[gi], w[e]);
          }
        }
        if (NG == 1 && p.group >= 64) {
          const uint32_t xslot =
              base + L.p + (uint32_t)((s & 1) * 4) * kBM * 8u;
          const uint32_t mine = xslot + (uint32_t)(h * kBM + i) * 8u;
          asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(mine),
                       "f"(mn[0]), "f"(mx[0])
                       : "memory");
          // the lane quarter's four warps meet on a bounded barrier (its
          // phase of use s >> 1); a wait that gives up flags the error word
          const uint32_t bx = b_xchg + 8u * (uint32_t)(2 * q4 + (s & 1));
          mbar_arrive(bx);
          mbar_wait(bx, (uint32_t)(s >> 1) & 1u, p.err);
          const int gp = p.group >> 5;  // parts per group: 2 or 4
          const int h0 = h & ~(gp - 1);
          for (int j = 0; j < gp; ++j) {
            float a, b;
            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                         : "=f"(a), "=f"(b)
                         : "r"(xslot + (uint32_t)((h0 + j) * kBM + i) * 8u)
                         : "memory");
            mn[0] = fminf(mn[0], a);
            mx[0] = fmaxf(mx[0], b);
          }
        }
        float dd[NG], r[NG], zf[NG], topz[NG], botz[NG];
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
          float d0 = __fdiv_rn(__fsub_rn(mx[gi], mn[gi]), (float)QMAX);
          if (d0 == 0.f) d0 = 1.f;
          dd[gi] = d0;
          r[gi] = __frcp_rn(d0);
          zf[gi] = fminf(fmaxf(__fadd_rn(__fdiv_rn(-mn[gi], d0), kMagic),
                               kMagic),
                         kTop) - kMagic;
          topz[gi] = kTop - zf[gi];
          botz[gi] = kMagic - zf[gi];
        }
        uint32_t qv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int gi = e / E;
          const float t = fmaxf(
              fminf(__fmaf_rn(w[e], r[gi], kMagic), topz[gi]), botz[gi]);
          qv[e] = __float_as_uint(t) - 0x4B400000u + (uint32_t)zf[gi];
        }
        // fp16 pairs in the codes path's TMEM order: position p of a span
        // holds channel k_perm(p); (1024 + q) - (1024 + z), then times D
        // rounded to fp16: the codes path's exact operations
        uint32_t o[16];
#pragma unroll
        for (int pp = 0; pp < 16; ++pp) {
          const int pa = 2 * pp, pb = 2 * pp + 1;
          const int ca = 16 * (pa >> 4) + k_perm<PERM>(pa & 15);
          const int cb = 16 * (pb >> 4) + k_perm<PERM>(pb & 15);
          const int gi = ca / E;
          const uint32_t x = (0x6400u | qv[ca]) | ((0x6400u | qv[cb]) << 16);
          const uint32_t zz = (0x6400u | (uint32_t)zf[gi]) * 0x00010001u;
          o[pp] = h2_bits(__hmul2(__hsub2(bits_h2(x), bits_h2(zz)),
                                  __float2half2_rn(dd[gi])));
        }
        tmem_st16(acol + 16u * h, o);
        // the codes, delta and zero, once (the first token tile)
        if (blockIdx.y == 0 && p.q_codes != nullptr && row_ok && in_k) {
          uint32_t cw[BITS];
#pragma unroll
          for (int k = 0; k < BITS; ++k) cw[k] = 0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int bit = e * BITS, wd = bit >> 5, sh = bit & 31;
            cw[wd] |= qv[e] << sh;
            if (sh + BITS > 32) cw[wd + 1] |= qv[e] >> (32 - sh);
          }
          uint32_t* dst = p.q_codes + (long long)n * p.q_ldc +
                          (long long)(k0 / 32 + h) * BITS;
#pragma unroll
          for (int k = 0; k < BITS; ++k) dst[k] = cw[k];
          const int c0 = k0 + 32 * h;
          if (NG == 2) {
            const long long gidx = (long long)n * p.q_ldg + c0 / 16;
            p.q_delta[gidx] = dd[0];
            p.q_delta[gidx + 1] = dd[NG - 1];
            p.q_zero[gidx] = (uint8_t)zf[0];
            p.q_zero[gidx + 1] = (uint8_t)zf[NG - 1];
          } else if (c0 % p.group == 0) {
            const long long gidx = (long long)n * p.q_ldg + c0 / p.group;
            p.q_delta[gidx] = dd[0];
            p.q_zero[gidx] = (uint8_t)zf[0];
          }
        }
      }
    };

    for (int s = 0; s < n_total && ok_loop; ++s) {
      const int k0 = (ks_begin + s) * kSK;
      // codes and activations of this stage have landed; its TMEM weight
      // slot is free once the MMA of stage s - SA completed
      if (!mbar_wait(b_loaded + 8 * rs.slot, rs.round & 1, p.err) ||
          (s >= SA &&
           !mbar_wait(b_afree + 8 * ra.slot, (ra.round & 1) ^ 1, p.err)) ||
          *aborted) {
        ok_loop = false;
        break;
      }
      tc_fence_after();
      const uint32_t acol = arow + (uint32_t)(ra.slot * kSCols);
      if (s < n_main) {
        if constexpr (QDQ) {
          qdq_stage(s, k0, acol);
        } else {
        const int pc = k0 >> (lg + 4);
        if (pc != pchunk) {
          if (pchunk >= 0) rp.next(2);
          pchunk = pc;
          if (!mbar_wait(b_full_p + 8 * rp.slot, rp.round & 1, p.err)) {
            ok_loop = false;
            break;
          }
        }
        const uint32_t poff = rp.slot * kParamBytes;
        const uint32_t cbase = crow + rs.slot * CHUNK;
        // the params of one 32-code block as fp16 pairs: (1024 + z), D
        auto block_params = [&](int blk, __half2 (&zsub)[GPB],
                                __half2 (&dh)[GPB]) {
          const int gl0 = ((k0 + 32 * blk) >> lg) & (kParamGroups - 1);
#pragma unroll
          for (int j = 0; j < GPB; ++j) {
            const int gl = gl0 + j;
            const float dl = __uint_as_float(ld_shared_u32(
                drow + poff + ((((uint32_t)gl >> 2) ^ dswz) << 4) +
                4 * (gl & 3)));
            const uint32_t zj = ld_shared_u8(zrow + poff + gl);
            dh[j] = __float2half2_rn(dl);
            zsub[j] = bits_h2((0x6400u | zj) * 0x00010001u);  // 1024 + z
          }
        };
        if constexpr (kParts == 4) {
          // one 32-code block per warp and stage
          uint32_t o[16];
          uint32_t cw[BITS];
          load_block<BITS>(cbase + h * 4 * BITS, cw);
          __half2 zsub[GPB], dh[GPB];
          block_params(h, zsub, dh);
          dequant_block<BITS, GMODE>(cw, zsub, dh, o);
          tmem_st16(acol + 16u * h, o);
        } else {
        // a thread's blocks are consecutive in K: the params are loaded
        // again only where a block starts a new group (every block for
        // g = 16). Decode at 16 tokens, 14336 x 4096, b = 4, g = 128:
        // 20.9 against 22.8 us on one box.
        __half2 zsub[GPB], dh[GPB];
#pragma unroll
        for (int half = half_lo; half < half_hi; ++half) {
          uint32_t o[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int blk = 2 * half + h;  // 32-code block of the stage
            uint32_t cw[BITS];
            load_block<BITS>(cbase + blk * 4 * BITS, cw);
            if (GMODE == 0 || blk == 2 * half_lo ||
                ((32 * blk) & (p.group - 1)) == 0)
              block_params(blk, zsub, dh);
            dequant_block<BITS, GMODE>(cw, zsub, dh, o + 16 * h);
          }
          tmem_st32(acol + 32u * half, o);
        }
        }
        // release the params once their last stage is read
        if (s + 1 >= n_main || ((k0 + kSK) >> (lg + 4)) != pc)
          warp_arrive(b_empty_p + 8 * rp.slot);
        }
      } else {
        // low-rank stage: row n of B (r <= 64 values) as fp16, zero padded
        if (h == 0) {
          uint32_t o[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int rho = 2 * e;
            float lo = 0.f, hi = 0.f;
            if (row_ok && rho < p.r)
              lo = load_any(p.Blr, p.blr_t, (long long)n * p.r + rho);
            if (row_ok && rho + 1 < p.r)
              hi = load_any(p.Blr, p.blr_t, (long long)n * p.r + rho + 1);
            o[e] = h2_bits(__floats2half2_rn(lo, hi));
          }
          tmem_st32(acol, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(b_ready + 8 * rs.slot);
      rs.next(S);
      ra.next(SA);
    }
    if (!ok_loop) *aborted = 1;
    __syncwarp();

    // ------------------------------------------------------ epilogue ----
    // the first two parts' warps drain the accumulator (with 16
    // dequantisers the other eight are done)
    if (kParts == 4 && h >= 2) goto done;
    {  // the epilogue's scope
    const bool acc_ok = mbar_wait(b_accum, 0, p.err);
    tc_fence_after();
    const bool ok = acc_ok && !*aborted && n_total > 0;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);

    // columns of the accumulator this warp drains
    const int c_lo = DQW >= 8 ? (bn >= 32 ? h * (bn / 2) : 0) : 0;
    const int c_hi = DQW >= 8 ? (bn >= 32 ? c_lo + bn / 2 : (h == 0 ? bn : 0))
                              : bn;
    // The statistic of the stored output over this warp's columns (the
    // next layer's input statistic, Proposed method bullets 2-3): row n's
    // sum of |Y[t][n]|^p goes to partial row (tile, part) of p.stats.
    float* const stats_row =
        p.stats ? p.stats + ((int64_t)blockIdx.y * p.stats_parts +
                             (p.stats_parts > 1 ? h : 0)) * p.N
                : nullptr;
    if (split == 1 && p.y_mode == 0) {
      // Y rows not 16-byte aligned: each thread stores its row directly
      float st = 0.f;
      for (int j = c_lo; j < c_hi; j += 16) {
        float v[16];
        tmem_ld16(t_lane + (uint32_t)j, v);
        if (ok && row_ok) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int t = t0 + j + c;
            if (t < p.T) {
              store_y(p.Y, p.yt, (long long)t * p.ldy + n, v[c]);
              if (stats_row) st += y_moment(stored_y(p.yt, v[c]), p.stats_p);
            }
          }
        }
      }
      if (stats_row && ok && row_ok && c_hi > c_lo) stats_row[n] = st;
    } else if (split == 1 && p.y_mode == 2) {
      // 16-bit Y. Each warp reads its 32 rows in two halves of 16 lanes in
      // the 16x256b fragment order, packs column pairs, and writes 8x8
      // blocks transposed into [tokens][64 rows] boxes (128-byte rows,
      // 16-byte chunk index XOR token % 8, the tensor map's 128-byte
      // swizzle), so every store instruction moves 512 bytes without bank
      // conflicts. The activation ring is idle once every MMA completed.
      const int box_t = c_hi - c_lo;
      const uint32_t gtile =
          base + L.x + (uint32_t)h * 2u * (uint32_t)box_t * 128u;
      const bool bf = p.yt == TTQ_BF16;
      const int mi = lane >> 3, mr = lane & 7;  // matrix and row addressed
#pragma unroll
      for (int lh = 0; lh < 2; ++lh) {
        const int nb = 32 * q4 + 16 * lh;  // first row of this lane half
        const uint32_t box = gtile + (uint32_t)(nb >> 6) * (uint32_t)box_t * 128u;
        const int chunk = ((nb & 63) >> 3) + (mi & 1);
        float st_lo = 0.f, st_hi = 0.f;  // rows nb + lane/4 and + 8
        for (int j = 0; j < box_t; j += 32) {
          uint32_t rr[16];
          tmem_ld_16x256b_x4(
              t_lane + ((uint32_t)(16 * lh) << 16) + (uint32_t)(c_lo + j), rr);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a0 = __uint_as_float(rr[4 * k]);
            const float a1 = __uint_as_float(rr[4 * k + 1]);
            const float b0 = __uint_as_float(rr[4 * k + 2]);
            const float b1 = __uint_as_float(rr[4 * k + 3]);
            if (bf) {
              pk[2 * k] = bf2_bits(__floats2bfloat162_rn(a0, a1));
              pk[2 * k + 1] = bf2_bits(__floats2bfloat162_rn(b0, b1));
            } else {
              pk[2 * k] = h2_bits(__floats2half2_rn(a0, a1));
              pk[2 * k + 1] = h2_bits(__floats2half2_rn(b0, b1));
            }
            if (stats_row) {
              // the stored values (columns past T hold zeros)
              float2 lo, hi;
              if (bf) {
                lo = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(
                    &pk[2 * k]));
                hi = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(
                    &pk[2 * k + 1]));
              } else {
                lo = __half22float2(bits_h2(pk[2 * k]));
                hi = __half22float2(bits_h2(pk[2 * k + 1]));
              }
              st_lo += y_moment(lo.x, p.stats_p) + y_moment(lo.y, p.stats_p);
              st_hi += y_moment(hi.x, p.stats_p) + y_moment(hi.y, p.stats_p);
            }
          }
          if (ok) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int row = j + 8 * (2 * q + (mi >> 1)) + mr;
              const uint32_t addr = box + (uint32_t)row * 128u +
                                    ((uint32_t)(chunk ^ (row & 7)) << 4);
              stmatrix_x4_trans(addr, pk[4 * q], pk[4 * q + 1],
                                pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
        }
        if (stats_row) {
          // the four lanes that hold a row's columns add their sums
#pragma unroll
          for (int o = 1; o < 4; o <<= 1) {
            st_lo += __shfl_xor_sync(0xffffffffu, st_lo, o);
            st_hi += __shfl_xor_sync(0xffffffffu, st_hi, o);
          }
          const int r_lo = m0 + nb + (lane >> 2);
          if (ok && box_t > 0 && (lane & 3) == 0) {
            if (r_lo < p.N) stats_row[r_lo] = st_lo;
            if (r_lo + 8 < p.N) stats_row[r_lo + 8] = st_hi;
          }
        }
      }
      fence_proxy_async_smem();
      if (h == 0)
        named_bar_sync<1>(128);
      else
        named_bar_sync<2>(128);
      if (ok && box_t > 0 && t0 + c_lo < p.T && q4 == 0 && lane == 0) {
        tma_store_2d(&tm_y, gtile, m0, t0 + c_lo);
        if (m0 + 64 < p.N)
          tma_store_2d(&tm_y, gtile + (uint32_t)box_t * 128u, m0 + 64,
                       t0 + c_lo);
        bulk_commit_group();
        bulk_wait_read();
      }
    } else if (split == 1) {
      // The accumulator tile goes TMEM -> registers -> shared memory as a
      // [tokens][128 rows] tile of Y's dtype (the activation ring is idle
      // once every MMA completed), then the four warps that drained a
      // column range hand it to the tensor memory accelerator as one box;
      // rows beyond N and tokens beyond T are clipped by the store.
      const uint32_t esz = p.yt == TTQ_F32 ? 4u : 2u;
      const uint32_t ytile = base + L.x;
      float st = 0.f;
      auto put = [&](int col, float v) {
        if (stats_row) st += y_moment(stored_y(p.yt, v), p.stats_p);
        const uint32_t a = ytile + ((uint32_t)col * kBM + (uint32_t)i) * esz;
        if (p.yt == TTQ_F32)
          st_shared_f32(a, v);
        else if (p.yt == TTQ_BF16)
          st_shared_u16(a, __bfloat16_as_ushort(__float2bfloat16_rn(v)));
        else
          st_shared_u16(a, __half_as_ushort(__float2half_rn(v)));
      };
      int j = c_lo;
      for (; j + 32 <= c_hi; j += 32) {
        float v[32];
        tmem_ld32(t_lane + (uint32_t)j, v);
        if (ok) {
#pragma unroll
          for (int c = 0; c < 32; ++c) put(j + c, v[c]);
        }
      }
      if (j < c_hi) {  // a 16-column remainder (decode tiles)
        float v[16];
        tmem_ld16(t_lane + (uint32_t)j, v);
        if (ok) {
#pragma unroll
          for (int c = 0; c < 16; ++c) put(j + c, v[c]);
        }
      }
      // (columns past T hold zeros, which add nothing)
      if (stats_row && ok && row_ok && c_hi > c_lo) stats_row[n] = st;
      fence_proxy_async_smem();
      if (h == 0)
        named_bar_sync<1>(128);
      else
        named_bar_sync<2>(128);
      if (ok && c_hi > c_lo && t0 + c_lo < p.T && q4 == 0 && lane == 0) {
        tma_store_2d(&tm_y, ytile + (uint32_t)c_lo * kBM * esz, m0, t0 + c_lo);
        bulk_commit_group();
        bulk_wait_read();
      }
    } else {
      float* part = reinterpret_cast<float*>(gbase + L.part);
      for (int j = c_lo; j < c_hi; j += 16) {
        float v[16];
        tmem_ld16(t_lane + (uint32_t)j, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) part[(j + c) * kBM + i] = ok ? v[c] : 0.f;
      }
    }
    }
  done:;
  }

  if (split > 1) {
    // Split-K: every rank's partial tile [bn][128] sits in its shared
    // memory. All ranks reduce disjoint 4-row pieces of the tile: each
    // thread issues the `split` 16-byte loads of a piece at once, then
    // sums them in rank order, so the result does not depend on timing.
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (warp >= kDqWarp0 && !*aborted) {
      constexpr int kDqThreads = 32 * DQW;
      const int tid = rank * kDqThreads + (threadIdx.x - 32 * kDqWarp0);
      const int nthr = split * kDqThreads;
      const int pieces = bn * (kBM / 4);
      const float* part = reinterpret_cast<const float*>(gbase + L.part);
      for (int pc = tid; pc < pieces; pc += nthr) {
        const int c = pc / (kBM / 4), i4 = (pc % (kBM / 4)) * 4;
        const int t = t0 + c;
        if (t >= p.T) continue;
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < split)
            v[q] = *reinterpret_cast<const float4*>(
                cluster.map_shared_rank(part, q) + c * kBM + i4);
        float4 acc = v[0];
#pragma unroll
        for (int q = 1; q < 8; ++q)
          if (q < split) {
            acc.x += v[q].x;
            acc.y += v[q].y;
            acc.z += v[q].z;
            acc.w += v[q].w;
          }
        const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (m0 + i4 + e < p.N)
            store_y(p.Y, p.yt, (long long)t * p.ldy + m0 + i4 + e, a4[e]);
      }
    }
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

// The prefill projection as a persistent kernel: one CTA per SM walks the
// output tiles (tile = blockIdx.x + i * gridDim.x, weight tiles fastest),
// so the TMA ring, the dequantisers and the MMA thread run on without a
// break between tiles. The accumulator is double-buffered in TMEM and four
// extra epilogue warps drain tile i (TMEM -> registers -> Y, coalesced
// across a warp's 32 rows for each token) while the MMAs of tile i+1 run.
// Roles and stage protocol are those of lowbit_gemm_kernel (codes path,
// one token tile per CTA at a time); the rings' slots and phases count
// stages over all of a CTA's tiles.
constexpr int kPersistEpiWarps = 4;
constexpr int kPersistBars = 4;  // accumulator full and empty, two buffers
// Eight dequantiser warps, two 32-code blocks per thread and stage. (Sixteen
// warps with one block each measured 327 against 318 us on the Llama-7B up
// layer, 351 against 324 us at b = 2, g = 16: per stage the fixed work of
// a warp, its waits and bookkeeping, weighs as much as a block's
// arithmetic, and sixteen warps kept 68 % of the issue slots busy against
// 55 % for eight. Four warps with four blocks each were slower again for
// b = 2, 3 and 8.)
constexpr int kPersistDequantWarps = 8;
__host__ __device__ constexpr int persist_threads() {
  return cta_threads(kPersistDequantWarps) + 32 * kPersistEpiWarps;
}

template <int BITS, int GMODE>
__global__ void __launch_bounds__(persist_threads(), 1)
    lowbit_gemm_persist_kernel(const __grid_constant__ CUtensorMap tm_x,
                               const __grid_constant__ CUtensorMap tm_u,
                               const __grid_constant__ CUtensorMap tm_c,
                               const __grid_constant__ CUtensorMap tm_d,
                               const __grid_constant__ CUtensorMap tm_z,
                               const GemmArgs p) {
  constexpr int DQW = kPersistDequantWarps;
  constexpr int NB = 16 / DQW;  // 32-code blocks per thread and stage
  constexpr int GPB = GMODE == 0 ? 2 : 1;
  constexpr uint32_t CHUNK = kBM * 16 * BITS;
  constexpr int kEpiWarp0 = kDqWarp0 + DQW;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw_base);

  const int S = p.S, SA = p.SA, bn = p.bn;
  const Layout L = make_layout(BITS, bn, S, false, false, kPersistBars);
  const uint32_t b_loaded = base + L.bars;
  const uint32_t b_ready = b_loaded + 8 * S;
  const uint32_t b_empty = b_ready + 8 * S;
  const uint32_t b_afree = b_empty + 8 * S;
  const uint32_t b_full_p = b_afree + 8 * S;
  const uint32_t b_empty_p = b_full_p + 16;
  // accumulator buffers: full (MMA -> epilogue), empty (epilogue -> MMA),
  // after the single-tile form's accumulator barrier
  const uint32_t b_acc_full = b_empty_p + 16 + 8;
  const uint32_t b_acc_empty = b_acc_full + 16;
  volatile uint32_t* tmem_slot =
      reinterpret_cast<volatile uint32_t*>(gbase + L.tmem);
  volatile int* aborted = reinterpret_cast<volatile int*>(gbase + L.abort_flag);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_main = p.k_stages;
  const int n_total = n_main + (p.r > 0 ? 1 : 0);
  const int lg = 31 - __clz(p.group);
  const int tiles_m = (p.N + kBM - 1) / kBM;
  const int n_tiles = tiles_m * ((p.T + bn - 1) / bn);
  auto tile_of = [&](int it, int& m0, int& t0) -> bool {
    const int tile = (int)blockIdx.x + it * (int)gridDim.x;
    if (tile >= n_tiles) return false;
    m0 = (tile % tiles_m) * kBM;
    t0 = (tile / tiles_m) * bn;
    return true;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(b_loaded + 8 * i, 1);
      mbar_init(b_ready + 8 * i, DQW);
      mbar_init(b_empty + 8 * i, 1);
      mbar_init(b_afree + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_full_p + 8 * i, 1);
      mbar_init(b_empty_p + 8 * i, DQW);
      mbar_init(b_acc_full + 8 * i, 1);
      mbar_init(b_acc_empty + 8 * i, kPersistEpiWarps);
    }
    *aborted = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_d);
    tma_prefetch_desc(&tm_z);
    if (p.r > 0) tma_prefetch_desc(&tm_u);
  }
  if (warp == 1) {
    tmem_alloc(base + L.tmem, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_enter();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a = tmem + (uint32_t)p.acc_cols;  // weight-stage ring

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      const uint32_t xbytes = (uint32_t)bn * 128u;
      Ring rs, rp;
      int issued = 0, np = 0, pchunk = -1;
      bool ok = true;
      int m0, t0;
      for (int it = 0; ok && tile_of(it, m0, t0); ++it) {
        if (pchunk >= 0) rp.next(2);  // a new row tile: a new params chunk
        pchunk = -1;
        for (int s = 0; s < n_total; ++s) {
          const int k0 = s * kSK;
          if (s < n_main) {
            const int pc = k0 >> (lg + 4);
            if (pc != pchunk) {
              if (pchunk >= 0) rp.next(2);
              pchunk = pc;
              if (np >= 2 && !mbar_wait(b_empty_p + 8 * rp.slot,
                                        (rp.round & 1) ^ 1, p.err)) {
                ok = false;
                break;
              }
              const uint32_t bar = b_full_p + 8 * rp.slot;
              const uint32_t dst = base + L.p + rp.slot * kParamBytes;
              mbar_arrive_expect_tx(bar, kParamBytes);
              tma_load_2d(dst, &tm_d, pc * kParamGroups, m0, bar);
              tma_load_2d(dst + kParamDeltaBytes, &tm_z, pc * kParamGroups,
                          m0, bar);
              ++np;
            }
          }
          if (issued >= S && !mbar_wait(b_empty + 8 * rs.slot,
                                        (rs.round & 1) ^ 1, p.err)) {
            ok = false;
            break;
          }
          if (*aborted) {
            ok = false;
            break;
          }
          const uint32_t bar = b_loaded + 8 * rs.slot;
          const uint32_t xdst = base + L.x + rs.slot * L.stage_x;
          if (s < n_main) {
            mbar_arrive_expect_tx(bar, CHUNK + 2 * xbytes);
            tma_load_2d(base + L.c + rs.slot * CHUNK, &tm_c,
                        (k0 >> 7) * 4 * BITS, m0, bar);
            tma_load_2d(xdst, &tm_x, k0, t0, bar);
            tma_load_2d(xdst + xbytes, &tm_x, k0 + 64, t0, bar);
          } else {
            mbar_arrive_expect_tx(bar, xbytes);
            tma_load_2d(xdst, &tm_u, 0, t0, bar);
          }
          rs.next(S);
          ++issued;
        }
      }
      if (!ok) *aborted = 1;
      // no bulk copy may still be writing shared memory at exit
      for (int i = 0; i < S && i < issued; ++i) {
        const int q = issued - 1 - i;
        mbar_wait(b_loaded + 8 * (q % S), (uint32_t)(q / S) & 1, p.err);
      }
      for (int i = 0; i < 2 && i < np; ++i) {
        const int q = np - 1 - i;
        mbar_wait(b_full_p + 8 * (q & 1), (uint32_t)(q >> 1) & 1, p.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kBM, bn);
      const uint32_t xbytes = (uint32_t)bn * 128u;
      Ring rs, ra;
      bool ok = true;
      int m0, t0, it = 0;
      for (; ok && tile_of(it, m0, t0); ++it) {
        const int buf = it & 1;
        // the epilogue has drained this buffer's previous tile
        if (it >= 2 && !mbar_wait(b_acc_empty + 8 * buf,
                                  (uint32_t)((it >> 1) - 1) & 1u, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * bn);
        for (int s = 0; s < n_total; ++s) {
          if (!mbar_wait(b_ready + 8 * rs.slot, rs.round & 1, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ad = tmem_a + (uint32_t)(ra.slot * kSCols);
          const uint32_t xs = base + L.x + rs.slot * L.stage_x;
          const uint64_t bd0 = smem_desc_sw128(xs);
          const uint64_t bd1 = smem_desc_sw128(xs + xbytes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ts(acc, ad + 8 * k, bd0 + 2 * k, idesc,
                          (s > 0 || k > 0) ? 1u : 0u);
          if (s < n_main) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_f16_ts(acc, ad + 32 + 8 * k, bd1 + 2 * k, idesc, 1u);
          }
          tc_commit(b_empty + 8 * rs.slot);
          tc_commit(b_afree + 8 * ra.slot);
          rs.next(S);
          ra.next(SA);
        }
        tc_commit(b_acc_full + 8 * buf);  // every MMA of the tile done
      }
      if (!ok) *aborted = 1;
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------ dequantisers ----
    // Two 32-code blocks of one weight row per thread and stage. A stage's
    // weights are computed from shared memory before the wait for its TMEM
    // slot. (Handing a stage to the MMA only after the next one is computed,
    // to hide the TMEM store wait, measured slower: 392 against 331 us on
    // the Llama-7B up layer, even when done only while the next stage's
    // data had already landed; the MMA waits on each stage's hand-over.)
    const int q4 = warp & 3;
    const int h = (warp - kDqWarp0) >> 2;   // blocks NB h .. NB h + NB - 1
    const int i = 32 * q4 + lane;           // row in the tile = TMEM lane
    const uint32_t crow = base + L.c + i * 16 * BITS;
    const uint32_t drow = base + L.p + i * 64;
    const uint32_t dswz = (uint32_t)((i >> 1) & 3);
    const uint32_t zrow = base + L.p + kParamDeltaBytes + i * 16;
    const uint32_t arow = tmem_a + ((uint32_t)(32 * q4) << 16);
    Ring rs, ra, rp;
    int pchunk = -1, done = 0;
    bool ok = true;
    // the TMEM weight slot of this stage is free (the MMA of stage
    // done - SA completed)
    auto slot_free = [&]() -> bool {
      if (done >= SA &&
          !mbar_wait(b_afree + 8 * ra.slot, (ra.round & 1) ^ 1, p.err))
        return false;
      tc_fence_after();
      return true;
    };
    int m0, t0;
    for (int it = 0; ok && tile_of(it, m0, t0); ++it) {
      if (pchunk >= 0) rp.next(2);
      pchunk = -1;
      const int n = m0 + i;
      const bool row_ok = n < p.N;
      for (int s = 0; s < n_total; ++s) {
        const int k0 = s * kSK;
        if (!mbar_wait(b_loaded + 8 * rs.slot, rs.round & 1, p.err) ||
            *aborted) {
          ok = false;
          break;
        }
        const uint32_t acol = arow + (uint32_t)(ra.slot * kSCols);
        if (s < n_main) {
          const int pc = k0 >> (lg + 4);
          if (pc != pchunk) {
            if (pchunk >= 0) rp.next(2);
            pchunk = pc;
            if (!mbar_wait(b_full_p + 8 * rp.slot, rp.round & 1, p.err)) {
              ok = false;
              break;
            }
          }
          const uint32_t poff = rp.slot * kParamBytes;
          uint32_t o[16 * NB];
          // the params of a 32-code block as fp16 pairs: (1024 + z), D
          auto params = [&](int blk, __half2 (&zsub)[GPB], __half2 (&dh)[GPB]) {
            const int gl0 = ((k0 + 32 * blk) >> lg) & (kParamGroups - 1);
#pragma unroll
            for (int j = 0; j < GPB; ++j) {
              const int gl = gl0 + j;
              const float dl = __uint_as_float(ld_shared_u32(
                  drow + poff + ((((uint32_t)gl >> 2) ^ dswz) << 4) +
                  4 * (gl & 3)));
              const uint32_t zj = ld_shared_u8(zrow + poff + gl);
              dh[j] = __float2half2_rn(dl);
              zsub[j] = bits_h2((0x6400u | zj) * 0x00010001u);
            }
          };
          __half2 zsub[GPB], dh[GPB];
          params(NB * h, zsub, dh);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const int blk = NB * h + b;
            // a thread's blocks share one group when g >= 32 NB (loading
            // the params once measured 336 against 344 us on the Llama-7B
            // up layer, b = 4, g = 128)
            if (b > 0 && (GMODE == 0 || p.group < 32 * NB))
              params(blk, zsub, dh);
            uint32_t cw[BITS];
            load_block<BITS>(crow + rs.slot * CHUNK + blk * 4 * BITS, cw);
            dequant_block<BITS, GMODE>(cw, zsub, dh, o + 16 * b);
          }
          // release the params once their last stage is read
          if (s + 1 >= n_main || ((k0 + kSK) >> (lg + 4)) != pc)
            warp_arrive(b_empty_p + 8 * rp.slot);
          if (!slot_free()) {
            ok = false;
            break;
          }
          static_assert(NB == 2, "one 32-column TMEM store per thread");
          tmem_st32(acol + 32u * h, o);
        } else {
          if (!slot_free()) {
            ok = false;
            break;
          }
          if (h == 0) {
            // low-rank stage: row n of B (r <= 64 values) as fp16, zero
            // padded
            uint32_t o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int rho = 2 * e;
              float lo = 0.f, hi = 0.f;
              if (row_ok && rho < p.r)
                lo = load_any(p.Blr, p.blr_t, (long long)n * p.r + rho);
              if (row_ok && rho + 1 < p.r)
                hi = load_any(p.Blr, p.blr_t, (long long)n * p.r + rho + 1);
              o[e] = h2_bits(__floats2half2_rn(lo, hi));
            }
            tmem_st32(acol, o);
          }
        }
        // hand the stage to the MMA once its TMEM stores landed
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(b_ready + 8 * rs.slot);
        rs.next(S);
        ra.next(SA);
        ++done;
      }
    }
    if (!ok) *aborted = 1;
  } else {
    // -------------------------------------------------- epilogue -------
    // thread = output row (TMEM lane) of its quarter; per token column the
    // warp's 32 lanes store 32 consecutive rows of Y
    const int q4 = warp & 3;
    const int i = 32 * q4 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);
    int m0, t0;
    for (int it = 0; tile_of(it, m0, t0); ++it) {
      const int buf = it & 1;
      if (!mbar_wait(b_acc_full + 8 * buf, (uint32_t)(it >> 1) & 1u, p.err))
        break;
      tc_fence_after();
      const int n = m0 + i;
      const bool ok = !*aborted;
      for (int j = 0; j < bn; j += 16) {
        float v[16];
        tmem_ld16(t_lane + (uint32_t)(buf * bn + j), v);
        if (ok && n < p.N) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int t = t0 + j + c;
            if (t < p.T) store_y(p.Y, p.yt, (long long)t * p.ldy + n, v[c]);
          }
        }
      }
      tc_fence_before();
      warp_arrive(b_acc_empty + 8 * buf);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

// X~ = fp16(X * inv_s), one thread per 16 channels, K-permuted for PERM.
template <typename TX, int PERM>
__global__ void prescale_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                                int64_t ldx, const float* __restrict__ inv_s,
                                __half* __restrict__ Xs, uint32_t* err) {
  griddep_enter();
  // T * K / 16 < 2^31 (checked on the host): 32-bit index math
  const uint32_t spans = (uint32_t)(K / 16);
  const uint32_t id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (uint32_t)T * spans) return;
  const uint32_t tq = id / spans;
  const int64_t t = tq, c = (int64_t)(id - tq * spans) * 16;
  float v[16], sv[16];
  load8<TX>(X + t * ldx + c, *reinterpret_cast<float(*)[8]>(v));
  load8<TX>(X + t * ldx + c + 8, *reinterpret_cast<float(*)[8]>(v + 8));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 s4 = __ldg(reinterpret_cast<const float4*>(inv_s + c) + q);
    sv[4 * q] = s4.x;
    sv[4 * q + 1] = s4.y;
    sv[4 * q + 2] = s4.z;
    sv[4 * q + 3] = s4.w;
  }
  uint32_t o[8];
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int la = k_perm<PERM>(2 * e), lb = k_perm<PERM>(2 * e + 1);
    const float fa = __fmul_rn(v[la], sv[la]);
    const float fb = __fmul_rn(v[lb], sv[lb]);
    bad |= !(fabsf(fa) < 65520.f) || !(fabsf(fb) < 65520.f);
    o[e] = h2_bits(__floats2half2_rn(fa, fb));
  }
  uint4* dst = reinterpret_cast<uint4*>(Xs + t * K + c);
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  if (bad) flag_error(err, TTQ_DEVERR_FP16_RANGE);
}

// The K permutations that keep each 8-channel half of a 16-channel span in
// that half (natural order, 4- and 8-bit codes).
template <int PERM>
__host__ __device__ constexpr bool perm_in_halves() {
  for (int p = 0; p < 8; ++p)
    if (k_perm<PERM>(p) >= 8 || k_perm<PERM>(p + 8) != 8 + k_perm<PERM>(p))
      return false;
  return true;
}

// X~ = fp16(X * inv_s) as prescale_kernel computes it, for the permutations
// that stay inside 8-channel halves. A thread owns 8 channels (one 16-byte
// vector of 16-bit X, two of fp32) for kPreRows consecutive tokens and
// keeps their scales in registers; a warp reads and writes 512 contiguous
// bytes of each row. (One thread per 16 channels and token read its 16
// scales again for every token and touched twice the cache lines per
// instruction: ncu showed the L1 pipeline 80-90 % busy and DRAM 37 %.)
constexpr int kPreRows = 32;
constexpr int kPreInFlight = 8;  // rows loaded before the first is used
template <typename TX, int PERM>
__global__ void __launch_bounds__(256)
    prescale8_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                     int64_t ldx, const float* __restrict__ inv_s,
                     __half* __restrict__ Xs, uint32_t* err) {
  static_assert(perm_in_halves<PERM>(), "permutation leaves the half");
  griddep_enter();
  const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c >= K) return;
  const int64_t t_end = min(T, ((int64_t)blockIdx.y + 1) * kPreRows);
  float sv[8];
  {
    const float4 a = __ldg(reinterpret_cast<const float4*>(inv_s + c));
    const float4 b = __ldg(reinterpret_cast<const float4*>(inv_s + c) + 1);
    sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w;
    sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
  }
  bool bad = false;
  for (int64_t t0 = (int64_t)blockIdx.y * kPreRows; t0 < t_end;
       t0 += kPreInFlight) {
    // raw 16-byte vectors in flight, converted only when used
    constexpr int V = sizeof(TX) == 4 ? 2 : 1;
    uint4 raw[kPreInFlight][V];
#pragma unroll
    for (int u = 0; u < kPreInFlight; ++u)
      if (t0 + u < t_end) {
#pragma unroll
        for (int q = 0; q < V; ++q)
          raw[u][q] = ld_stream_v4(X + (t0 + u) * ldx + c + q * 4);
      }
#pragma unroll
    for (int u = 0; u < kPreInFlight; ++u) {
      if (t0 + u >= t_end) break;
      float v[8];
      if constexpr (V == 2) {
        const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z,
                               raw[u][0].w, raw[u][1].x, raw[u][1].y,
                               raw[u][1].z, raw[u][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(w[e]);
      } else {
        const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z,
                               raw[u][0].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (sizeof(TX) == 2 && std::is_same<TX, __half>::value)
            f16x2_to_f32(w[e], v[2 * e], v[2 * e + 1]);
          else
            bf16x2_to_f32(w[e], v[2 * e], v[2 * e + 1]);
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int la = k_perm<PERM>(2 * e), lb = k_perm<PERM>(2 * e + 1);
        const float fa = __fmul_rn(v[la], sv[la]);
        const float fb = __fmul_rn(v[lb], sv[lb]);
        bad |= !(fabsf(fa) < 65520.f) || !(fabsf(fb) < 65520.f);
        o[e] = h2_bits(__floats2half2_rn(fa, fb));
      }
      *reinterpret_cast<uint4*>(Xs + (t0 + u) * K + c) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (bad) flag_error(err, TTQ_DEVERR_FP16_RANGE);
}

// U[t][rho] = fp16(sum_j X[t][j] A[rho][j]) for rho < r, 0 up to 64.
template <typename TX>
__global__ void __launch_bounds__(256)
    lowrank_u_kernel(const TX* __restrict__ X, int64_t T, int64_t K,
                     int64_t ldx, const TX* __restrict__ A, int r,
                     __half* __restrict__ U) {
  griddep_enter();
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

// 2D tensor [rows][inner] of `esize`-byte elements with a row pitch of
// `pitch_bytes`, copied in boxes of box_inner x box_rows; out-of-range
// elements read as zero.
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr,
               uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
               uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Maps {
  CUtensorMap x, u, c, d, z, y, w;
};

template <int BITS, int GMODE, int DQW, bool QDQ = false>
ttq_status launch_kernel(const Maps& m, const GemmArgs& a, dim3 grid,
                         int split, size_t smem, cudaStream_t st) {
  auto kern = lowbit_gemm_kernel<BITS, GMODE, DQW, QDQ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return TTQ_ERR_CUDA;
  LaunchShape ls;
  ls.grid = grid;
  ls.block = dim3(cta_threads(DQW), 1, 1);
  ls.smem = smem;
  ls.cluster_z = (unsigned)split;
  return launch(ls, st, kern, m.x, m.u, m.c, m.d, m.z, m.y, m.w, a);
}

template <int BITS, int GMODE>
ttq_status launch_persist(const Maps& m, const GemmArgs& a, unsigned ctas,
                          size_t smem, cudaStream_t st) {
  auto kern = lowbit_gemm_persist_kernel<BITS, GMODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return TTQ_ERR_CUDA;
  LaunchShape ls;
  ls.grid = dim3(ctas, 1, 1);
  ls.block = dim3(persist_threads(), 1, 1);
  ls.smem = smem;
  return launch(ls, st, kern, m.x, m.u, m.c, m.d, m.z, a);
}

template <int GMODE>
ttq_status dispatch_persist(int bits, const Maps& m, const GemmArgs& a,
                            unsigned ctas, size_t smem, cudaStream_t st) {
  switch (bits) {
#define TTQ_LP(B) \
  case B:         \
    return launch_persist<B, GMODE>(m, a, ctas, smem, st);
    TTQ_LP(2) TTQ_LP(3) TTQ_LP(4) TTQ_LP(5) TTQ_LP(6) TTQ_LP(7) TTQ_LP(8)
#undef TTQ_LP
  }
  return TTQ_ERR_INVALID_ARG;
}

template <int GMODE, int DQW, bool QDQ = false>
ttq_status dispatch_bits(int bits, const Maps& m, const GemmArgs& a, dim3 grid,
                         int split, size_t smem, cudaStream_t st) {
  switch (bits) {
#define TTQ_LK(B)                                                       \
  case B:                                                               \
    return launch_kernel<B, GMODE, DQW, QDQ>(m, a, grid, split, smem, st);
    TTQ_LK(2) TTQ_LK(3) TTQ_LK(4) TTQ_LK(5) TTQ_LK(6) TTQ_LK(7) TTQ_LK(8)
#undef TTQ_LK
  }
  return TTQ_ERR_INVALID_ARG;
}

template <typename TX>
ttq_status launch_pre(const void* X, int64_t T, int64_t K, int64_t ldx,
                      const float* inv_s, int bits, const void* A, int r,
                      __half* Xs, __half* U, cudaStream_t st) {
  const int64_t items = T * (K / 16);
  const int threads = 256;
  const unsigned grid = (unsigned)((items + threads - 1) / threads);
  const TX* x = static_cast<const TX*>(X);
  uint32_t* err = device_error_word();
  LaunchShape ls;
  ls.grid = dim3(grid);
  ls.block = dim3(threads);
  // 2-bit codes pair channels 8 apart: one thread per 16-channel span;
  // the other orders stay inside 8-channel halves (prescale8_kernel)
  LaunchShape l8;
  l8.grid = dim3((unsigned)((K / 8 + threads - 1) / threads),
                 (unsigned)((T + kPreRows - 1) / kPreRows));
  l8.block = dim3(threads);
  ttq_status e;
  switch (bits) {
    case 2: e = launch(ls, st, prescale_kernel<TX, 2>, x, T, K, ldx, inv_s, Xs, err); break;
    case 4: e = launch(l8, st, prescale8_kernel<TX, 4>, x, T, K, ldx, inv_s, Xs, err); break;
    case 8: e = launch(l8, st, prescale8_kernel<TX, 8>, x, T, K, ldx, inv_s, Xs, err); break;
    default: e = launch(l8, st, prescale8_kernel<TX, 0>, x, T, K, ldx, inv_s, Xs, err); break;
  }
  if (e != TTQ_OK || r == 0) return e;
  LaunchShape lu;
  lu.grid = dim3((unsigned)T);
  lu.block = dim3(256);
  return launch(lu, st, lowrank_u_kernel<TX>, x, T, K, ldx,
                static_cast<const TX*>(A), r, U);
}

}  // namespace

// Partial statistic rows per token tile: one per column part of the
// epilogue (two halves with eight or more dequantisers and 32+ tokens).
int stats_parts_of(int dqw, int bn) { return (dqw >= 8 && bn >= 32) ? 2 : 1; }

bool make_tensor_map_2d(CUtensorMap* m, CUtensorMapDataType dt,
                        const void* ptr, uint64_t inner, uint64_t rows,
                        uint64_t pitch_bytes, uint32_t box_inner,
                        uint32_t box_rows, CUtensorMapSwizzle swz) {
  return make_tmap(m, dt, ptr, inner, rows, pitch_bytes, box_inner, box_rows,
                   swz);
}

size_t gemm_workspace_bytes(int64_t T, int64_t K, int r) {
  size_t b = align_up((size_t)T * (size_t)K * 2, 1024);
  if (r > 0) b += align_up((size_t)T * 64 * 2, 1024);
  return b;
}

ttq_status launch_prepare(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                          int64_t ldx, const float* inv_s, int bits,
                          const void* A, int r, void* Xs, void* U,
                          cudaStream_t st) {
  __half* xs = static_cast<__half*>(Xs);
  __half* u = static_cast<__half*>(U);
  switch (xt) {
    case TTQ_F32:
      return launch_pre<float>(X, T, K, ldx, inv_s, bits, A, r, xs, u, st);
    case TTQ_BF16:
      return launch_pre<__nv_bfloat16>(X, T, K, ldx, inv_s, bits, A, r, xs, u,
                                       st);
    case TTQ_F16:
      return launch_pre<__half>(X, T, K, ldx, inv_s, bits, A, r, xs, u, st);
  }
  return TTQ_ERR_INVALID_ARG;
}

// Tile shape of the tensor-core projection: token tile bn, shared-memory
// ring depth S, TMEM weight ring depth SA, TMEM columns (S < 2: no shape).
void plan_tiles(int64_t T, int64_t N, int64_t K, int bits, int& bn, int& S,
                int& SA, int& tmem_cols, int& acc_cols, bool qdq = false) {
  const int sms = sm_count();
  const int64_t tiles_m = (N + kBM - 1) / kBM;
  const int k_stages = (int)((K + kSK - 1) / kSK);
  S = 0;
  auto fits = [&](int bn_, int S_, bool sp, size_t lim) {
    return (size_t)make_layout(bits, bn_, S_, sp, qdq).total + 1024 <= lim;
  };
  if (T <= 32) {
    bn = T <= 16 ? 16 : 32;
    acc_cols = 32;
    tmem_cols = 256;
    SA = (tmem_cols - acc_cols) / kSCols;
    // the shared-memory ring runs deeper than the TMEM weight ring so that
    // loads are issued well ahead of the dequantisers
    S = 8;
    while (S > SA && !fits(bn, S, true, 110 * 1024)) --S;
  } else {
    bn = 64;
    double best = 1e30;
    for (int c : {256, 192, 128, 64}) {
      int s_ = std::min(6, (512 - c) / kSCols);
      while (s_ > 1 && !fits(c, s_, false, kMaxSmem)) --s_;
      if (s_ < 2) continue;
      const int64_t ctas = tiles_m * ((T + c - 1) / c);
      const int64_t waves = (ctas + sms - 1) / sms;
      const double stage = std::max(8.0 * std::max(45.0, c / 2.0), 600.0);
      // shallow pipelines expose the load latency
      const double depth_penalty = s_ < 3 ? 1.25 : 1.0;
      const double t = (double)waves * (4000.0 + k_stages * stage * depth_penalty);
      if (t < best) {
        best = t;
        bn = c;
      }
    }
    acc_cols = bn;
    tmem_cols = 512;
    S = std::min(6, (tmem_cols - acc_cols) / kSCols);
    while (S > 1 && !fits(bn, S, false, kMaxSmem)) --S;
    SA = S;
  }
}

// Partial statistic rows of the fused output statistic for a prefill
// projection of T x N x K (0 when there is none: T <= 32 or no shape).
int64_t gemm_stats_rows(int64_t T, int64_t N, int64_t K, int bits) {
  if (T <= 32) return 0;
  int bn, S, SA, tmem_cols, acc_cols;
  plan_tiles(T, N, K, bits, bn, S, SA, tmem_cols, acc_cols);
  if (S < 2) return 0;
  return ((T + bn - 1) / bn) * stats_parts_of(kPrefillDequantWarps, bn);
}

// The fused (QDQ) form's extra inputs and outputs.
struct QdqInputs {
  const void* W;  // bf16 [N, K], row pitch ldw elements
  int64_t ldw;
  const float* s;
  uint32_t* codes;  // outputs (null: not stored)
  float* delta;
  uint8_t* zero;
};

ttq_status launch_gemm_impl(const void* Xs, const void* U, int64_t T,
                            int64_t K, const uint32_t* codes,
                            const float* delta, const uint8_t* zero,
                            int64_t N, int bits, int group, const void* B,
                            ttq_dtype bt, int r, void* Y, ttq_dtype yt,
                            int64_t ldy, cudaStream_t st, float* stats,
                            float stats_p, const QdqInputs* q) {
  // one or two tokens: the CUDA-core matrix-vector product (gemv.cu)
  if (!q && gemv_applies(T, K)) {
    if (stats) return TTQ_ERR_UNSUPPORTED;
    return launch_gemv(Xs, U, T, K, codes, delta, zero, N, bits, group, B, bt,
                       r, Y, yt, ldy, st);
  }
  if ((stats || q) && T <= 32) return TTQ_ERR_UNSUPPORTED;
  // Tile shape. A stage is 128 channels: a codes chunk, two 64-channel
  // activation boxes, one 64-column fp16 weight stage in TMEM.
  // Decode (T <= 32): 256 TMEM columns per CTA (two CTAs per SM), K split
  // over a cluster so that about one wave covers the GPU.
  // Prefill: all 512 TMEM columns; the token tile is picked by a model of
  // waves x (fixed cost + stages x max(MMA, dequant)), an MMA of N tokens
  // costing about max(45, N/2) cycles (eight per stage) and a stage about
  // 600 cycles of dequantisation. (Costing every MMA at least 128 cycles,
  // which moves every large layer to N = 256, measured slower: 390 against
  // 346 us on the Llama up layer, with one shared-memory stage less.)
  const int sms = sm_count();
  const int64_t tiles_m = (N + kBM - 1) / kBM;
  const int k_stages = (int)((K + kSK - 1) / kSK);
  int bn, S, SA, tmem_cols, acc_cols, split = 1;
  // dual: two CTAs per SM, four dequantiser warps and 256 TMEM columns each
  const bool dual = T <= 32;
  plan_tiles(T, N, K, bits, bn, S, SA, tmem_cols, acc_cols, q != nullptr);
  if (S < 2) return TTQ_ERR_UNSUPPORTED;
  if (T <= 32) {
    const size_t sm1 = make_layout(bits, bn, S, true).total + 1024;
    const int per_sm = sm1 <= 113 * 1024 ? 2 : 1;
    split = (int)std::min<int64_t>(
        8, std::max<int64_t>(1, per_sm * sms / tiles_m));
    split = std::min(split, k_stages);
  } else if (q && !stats && T <= bn && 2 * tiles_m <= sms) {
    // The fused form with one token tile: each CTA would quantize a whole
    // 128-row slab of the weight alone, on a few dozen SMs. Splitting K
    // over a cluster spreads the quantization over about one wave; the
    // ranks' partial tiles are reduced in rank order as in decode.
    int s_ = S;
    while (s_ > 1 && make_layout(bits, bn, s_, true, true).total + 1024 >
                         (size_t)kMaxSmem)
      --s_;
    if (s_ >= 2) {
      split = (int)std::min<int64_t>(8, sms / tiles_m);
      split = std::min(split, k_stages);
      if (split > 1) {
        S = s_;
        SA = std::min(SA, S);
      }
    }
  }
  // The persistent form (four or more output tiles per SM, plain codes, no
  // fused statistic): two accumulator buffers of bn columns and SA weight
  // stages share the 512 TMEM columns. The token tile minimises the tiles
  // per SM times the stage cost of the same model as above. (With fewer
  // tiles per SM the one-tile-per-CTA grid measured faster: 32.1 against
  // 38.9 us on 1024 x 6912 x 1152, 13.2 against 24.6 us on 2048 x 2304 x
  // 768. On the Llama-7B up layer the token tiles 192, 160 and 128
  // measured 322, 356 and 418 us: a stage costs nearly the same whatever
  // the tile, so the widest tile that leaves two weight stages wins.)
  bool persist = false;
  if (!dual && !q && !stats) {
    double best = 1e30;
    int pbn = 0, pS = 0, pSA = 0;
    for (int c : {192, 160, 128}) {
      const int sa = std::min(4, (512 - 2 * c) / kSCols);
      int s_ = 5;
      while (s_ > 1 && make_layout(bits, c, s_, false, false, kPersistBars)
                               .total + 1024 > (size_t)kMaxSmem)
        --s_;
      if (s_ < 2 || sa < 2) continue;
      const int64_t tiles = tiles_m * ((T + c - 1) / c);
      if (tiles < 4 * (int64_t)sms) continue;
      const int64_t per_sm = (tiles + sms - 1) / sms;
      const double stage = std::max(8.0 * std::max(45.0, c / 2.0), 600.0);
      const double t = (double)per_sm * k_stages * stage;
      if (t < best) {
        best = t;
        pbn = c;
        pS = s_;
        pSA = std::min(sa, s_);
      }
    }
    if (pbn > 0) {
      persist = true;
      bn = pbn;
      S = pS;
      SA = pSA;
      acc_cols = 2 * bn;
      tmem_cols = 512;
    }
  }
  const int per = (k_stages + split - 1) / split;
  split = (k_stages + per - 1) / per;  // every rank gets at least one stage
  const Layout L = persist ? make_layout(bits, bn, S, false, false, kPersistBars)
                           : make_layout(bits, bn, S, split > 1, q != nullptr);
  const size_t smem = L.total + 1024;
  const int64_t tiles_t = (T + bn - 1) / bn;

  Maps m;
  const int64_t G = K / group;
  bool ok =
      make_tmap(&m.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xs, K, T, K * 2, 64,
                bn, CU_TENSOR_MAP_SWIZZLE_128B) &&
      (r == 0 || make_tmap(&m.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, U, 64, T,
                           128, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B));
  if (q) {
    // bf16 weight tiles of 64 channels x 128 rows, 128-byte swizzled; the
    // codes maps are not read
    ok = ok && make_tmap(&m.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q->W, K, N,
                         (uint64_t)q->ldw * 2, 64, kBM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    m.c = m.d = m.z = m.x;
  } else {
    ok = ok &&
         make_tmap(&m.c, CU_TENSOR_MAP_DATA_TYPE_UINT32, codes, K * bits / 32,
                   N, codes_ld(K, bits) * 4, 4 * bits, kBM,
                   CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_tmap(&m.d, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, delta, G, N,
                   groups_ld(K, group) * 4, kParamGroups, kBM,
                   CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_tmap(&m.z, CU_TENSOR_MAP_DATA_TYPE_UINT8, zero, G, N,
                   groups_ld(K, group), kParamGroups, kBM,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    m.w = m.x;
  }
  if (!ok) return TTQ_ERR_CUDA;
  if (r == 0) m.u = m.x;  // never read without a low-rank stage
  // Y is stored by the tensor memory accelerator in boxes of 128 rows x the
  // tokens one group of four dequantiser warps drains (half the tile with
  // eight dequantisers); the split-K form reduces through the cluster
  // instead and never reads this map
  const int dqw = dual ? 4 : kPrefillDequantWarps;
  const int box_t = (dqw >= 8 && bn >= 32) ? bn / 2 : bn;
  int y_mode = 0;
  if (!persist && split == 1 && ((uint64_t)ldy * dtype_bytes(yt)) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(Y) % 16 == 0)
    y_mode = (yt != TTQ_F32 && box_t % 32 == 0) ? 2 : 1;
  if (y_mode > 0) {
    const CUtensorMapDataType ydt =
        yt == TTQ_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
        : yt == TTQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const bool ok_y =
        y_mode == 2
            ? make_tmap(&m.y, ydt, Y, N, T, (uint64_t)ldy * dtype_bytes(yt),
                        64, box_t, CU_TENSOR_MAP_SWIZZLE_128B)
            : make_tmap(&m.y, ydt, Y, N, T, (uint64_t)ldy * dtype_bytes(yt),
                        kBM, box_t, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok_y) return TTQ_ERR_CUDA;
  } else {
    m.y = m.x;
  }

  GemmArgs a;
  a.Blr = B;
  a.blr_t = (int)bt;
  a.r = r;
  a.N = (int)N;
  a.K = (int)K;
  a.T = (int)T;
  a.Y = Y;
  a.yt = (int)yt;
  a.ldy = ldy;
  a.bn = bn;
  a.S = S;
  a.SA = SA;
  a.tmem_cols = tmem_cols;
  a.acc_cols = acc_cols;
  a.group = group;
  a.k_stages = k_stages;
  a.per = per;
  a.y_mode = y_mode;
  a.qs = q ? q->s : nullptr;
  a.q_codes = q ? q->codes : nullptr;
  a.q_delta = q ? q->delta : nullptr;
  a.q_zero = q ? q->zero : nullptr;
  a.q_ldc = codes_ld(K, bits);
  a.q_ldg = groups_ld(K, group);
  a.stats = stats;
  a.stats_p = stats_p;
  a.stats_parts = stats_parts_of(dqw, bn);
  a.err = device_error_word();
  if (persist) {
    const unsigned ctas =
        (unsigned)std::min<int64_t>(tiles_m * tiles_t, (int64_t)sms);
    return group == 16 ? dispatch_persist<0>(bits, m, a, ctas, smem, st)
                       : dispatch_persist<1>(bits, m, a, ctas, smem, st);
  }
  const dim3 grid((unsigned)tiles_m, (unsigned)tiles_t, (unsigned)split);
  // decode packs two CTAs per SM with four dequant warps each; prefill runs
  // one CTA per SM with sixteen

  if (dual) {
    if (group == 16)
      return dispatch_bits<0, 4>(bits, m, a, grid, split, smem, st);
    return dispatch_bits<1, 4>(bits, m, a, grid, split, smem, st);
  }
  if (q)
    return group == 16
               ? dispatch_bits<0, kPrefillDequantWarps, true>(
                     bits, m, a, grid, split, smem, st)
               : dispatch_bits<1, kPrefillDequantWarps, true>(
                     bits, m, a, grid, split, smem, st);
  if (group == 16)
    return dispatch_bits<0, kPrefillDequantWarps>(bits, m, a, grid, split,
                                                     smem, st);
  return dispatch_bits<1, kPrefillDequantWarps>(bits, m, a, grid, split,
                                                   smem, st);
}

ttq_status launch_gemm_prepared(const void* Xs, const void* U, int64_t T,
                                int64_t K, const uint32_t* codes,
                                const float* delta, const uint8_t* zero,
                                int64_t N, int bits, int group, const void* B,
                                ttq_dtype bt, int r, void* Y, ttq_dtype yt,
                                int64_t ldy, cudaStream_t st, float* stats,
                                float stats_p) {
  return launch_gemm_impl(Xs, U, T, K, codes, delta, zero, N, bits, group, B,
                          bt, r, Y, yt, ldy, st, stats, stats_p, nullptr);
}

ttq_status launch_quantize_gemm_prepared(
    const void* W, int64_t ldw, const float* s, const void* Xs, const void* U,
    int64_t T, int64_t K, int64_t N, int bits, int group, const void* B,
    ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy, uint32_t* codes,
    float* delta, uint8_t* zero, cudaStream_t st) {
  const QdqInputs q = {W, ldw, s, codes, delta, zero};
  return launch_gemm_impl(Xs, U, T, K, nullptr, nullptr, nullptr, N, bits,
                          group, B, bt, r, Y, yt, ldy, st, nullptr, 2.f, &q);
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
  ttq_status e =
      launch_prepare(X, xt, T, K, ldx, inv_s, bits, A, r, Xs, U, st);
  if (e != TTQ_OK) return e;
  return launch_gemm_prepared(Xs, U, T, K, codes, delta, zero, N, bits, group,
                              B, xt, r, Y, yt, ldy, st);
}

}  // namespace ttq
