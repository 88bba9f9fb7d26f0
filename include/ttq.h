/*
 * ttq.h — C ABI of libttq, the sm_100a hot path of TTQ (activation-aware
 * test-time quantization).
 *
 * Source of the method: "TTQ: Activation-Aware Test-Time Quantization to
 * Accelerate LLM Inference On The Fly" (Koike-Akino, Liu, Wang; arXiv
 * 2603.19296), as summarised by the nubint.ai review of that paper (cited
 * below as "TTQ review"), section "Proposed method" (제안 방법), bullets 1-7:
 *   1  weights are quantized on the fly with group-wise RTN and QDQ;
 *   2  AWQ with a closed form built on a diagonal approximation of the input
 *      covariance;
 *   3  activation statistics are estimated online per prompt, the covariance
 *      is shrunk (C_lambda), the target is L = E_X ||(W - W_hat) X||^2;
 *   4  alpha, lambda, p are fixed (no search at test time);
 *   5  optional low-rank factors: W = W_q + B A;
 *   6  the overhead vanishes as d' and T grow;
 *   7  a CUDA GEMM kernel runs the quantized projection.
 *
 * Per prompt and per linear layer the hot path is four calls on one stream:
 *   ttq_act_stats -> ttq_awq_scales -> ttq_quantize_rtn_grouped
 *   -> ttq_w_lowbit_gemm (optionally with the low-rank term).
 *
 * Notation. X is [T, K] (tokens x input channels, row-major, row pitch ldx
 * elements). W is [N, K] (output x input, the PyTorch Linear layout, row
 * pitch ldw). Y = X diag(1/s) W_hat^T is [T, N] (row pitch ldy). A group is
 * g consecutive input channels of one weight row.
 *
 * Conventions shared by every call.
 *   - Pointers named X, W, Y, sum, s, inv_s, codes, delta, zero, A, B,
 *     workspace are DEVICE pointers owned by the caller. The library
 *     allocates nothing, frees nothing and keeps no pointer after a call
 *     returns.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call only enqueues work; none synchronises the host.
 *   - Argument checks happen before any launch. A bad argument returns
 *     TTQ_ERR_INVALID_ARG (or TTQ_ERR_UNSUPPORTED for a valid but
 *     unimplemented combination) and enqueues nothing. A failed launch
 *     returns TTQ_ERR_CUDA. The library never aborts the process.
 *   - Faults found on the device (a bounded wait that gave up, an fp16 range
 *     overflow) set a sticky device error word; ttq_device_error() reads it.
 *   - Alignment. X, W, Xs, U and A, and the s, inv_s, codes, delta and
 *     zero that the quantizer and the projection read, must start on a
 *     16-byte boundary, and ldx, ldw must keep every row of X and W 16-byte
 *     aligned (the kernels read them with 16-byte or tensor-memory-
 *     accelerator loads); the pitches of ttq_codes_ld and ttq_groups_ld
 *     keep the rows of codes, delta and zero aligned. Y, B, the sums, the
 *     s and inv_s written by the statistics calls, and the counter need
 *     only their element's alignment; rows of Y that are not 16-byte
 *     aligned are written by a per-row path. A pointer that breaks these
 *     rules returns TTQ_ERR_INVALID_ARG.
 */
#ifndef TTQ_H_
#define TTQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTQ_OK = 0,
  TTQ_ERR_INVALID_ARG = 1, /* bad pointer, size, pitch, alignment or enum  */
  TTQ_ERR_UNSUPPORTED = 2, /* valid request this build does not implement */
  TTQ_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed         */
  TTQ_ERR_TIMEOUT = 4,     /* a device-side bounded wait gave up           */
  TTQ_ERR_RANGE = 5        /* an fp16 operand overflowed on the device     */
} ttq_status;

typedef enum { TTQ_F32 = 0, TTQ_BF16 = 1, TTQ_F16 = 2 } ttq_dtype;

/* Fixed hyperparameters of one layer (TTQ review, Proposed method, bullet 4:
 * alpha, lambda, p are fixed; bullet 1: b bits, group g). */
typedef struct {
  int bits;     /* b, 2..8                                     */
  int group;    /* g, one of 16, 32, 64, 128                   */
  float alpha;  /* AWQ exponent, >= 0                          */
  float lambda; /* shrinkage weight, in [0, 1]                 */
  float p;      /* moment order of the channel statistic, > 0  */
} ttq_params;

/* Sticky device error bits (read with ttq_device_error). */
#define TTQ_DEVERR_TIMEOUT 0x1u    /* a bounded wait inside a kernel gave up */
#define TTQ_DEVERR_FP16_RANGE 0x2u /* |x / s| exceeded the fp16 range        */

/* ---------------------------------------------------------------------
 * Packed code layout (TTQ review, Proposed method, bullet 1: group-wise
 * RTN; the pages fix no storage format, this one is ours).
 *
 * Row n of the codes array holds K/32 blocks; block k holds the codes of
 * input channels 32k .. 32k+31 in `bits` consecutive uint32 words. Inside a
 * block the codes form a little-endian bit stream: the code of channel
 * 32k + c occupies bits [c*bits, c*bits + bits) of the block, where bit i of
 * the block is bit (i % 32) of word (i / 32). A row holds K*bits/32 words
 * followed by zero padding up to its pitch ttq_codes_ld(K, bits) (a multiple
 * of 4 words), so the array is [N][ttq_codes_ld(K, bits)] uint32.
 *
 * delta is [N][ttq_groups_ld(K, g)] float32 and zero is
 * [N][ttq_groups_ld(K, g)] uint8: entry [n][G] for the K/g groups of row n,
 * then zero padding up to the pitch (a multiple of 16 entries). The pitches
 * keep every row 16-byte aligned, which tensor-memory-accelerator copies
 * need. The scaled-domain weight of channel j in row n is
 *     W_hat_s[n][j] = (q[n][j] - zero[n][j/g]) * delta[n][j/g]
 * and the effective weight is W_hat_s[n][j] / s[j].
 * ------------------------------------------------------------------- */

/* Row pitches of the packed layout: words per codes row, entries per
 * delta/zero row. Both return 0 for invalid arguments. */
int64_t ttq_codes_ld(int64_t K, int bits);
int64_t ttq_groups_ld(int64_t K, int group);

/* Step 1, online activation statistics (TTQ review, Proposed method,
 * bullets 2-3: the diagonal of the input covariance, estimated per prompt).
 *
 * sum_out[j] (+)= sum_t |X[t][j]|^p, accumulated in fp32, for j < K.
 *   X      [T, K] of dtype xt (F32, BF16 or F16), row pitch ldx elements.
 *   p      > 0. p == 2 gives the diagonal of the uncentred X^T X.
 *   accumulate  0: overwrite sum_out; 1: add to it (chunked long prompts).
 * Requires K % 8 == 0 and T >= 1. The reduction order is fixed, so the
 * result is bit-reproducible run to run. */
ttq_status ttq_act_stats(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                         int64_t ldx, float p, int accumulate, float* sum_out,
                         void* stream);

/* Step 2, AWQ scales from the shrunk diagonal covariance (TTQ review,
 * Proposed method, bullets 2-4).
 *   m_j   = sum[j] / T_total
 *   mbar  = (1/K) sum_j m_j
 *   c_j   = (1 - lambda) m_j + lambda mbar        (shrink toward the mean)
 *   s_j   = c_j^(alpha/p); s_j = 1 when alpha == 0 or c_j <= 0 or not finite
 *   inv_s_j = 1 / s_j
 * Computed in fp64 on the device and stored as fp32. Only prm->alpha,
 * prm->lambda and prm->p are read. */
ttq_status ttq_awq_scales(const float* sum, int64_t T_total, int64_t K,
                          const ttq_params* prm, float* s, float* inv_s,
                          void* stream);

/* Step 2 for a layer whose input channels are split over several GPUs
 * (row-parallel tensor parallelism; the pages describe one GPU, the split
 * is ours). The channel mean mbar of the shrinkage (TTQ review, Proposed
 * method, bullet 3) runs over ALL input channels, so it needs one scalar
 * from every shard:
 *   ttq_channel_moment_total: *total = sum_j sum[j] / T_total over this
 *     shard's K channels, in fp64 and a fixed order (device double, 8-byte
 *     aligned).
 *   The caller adds the shards' totals (one all-reduce of one double).
 *   ttq_awq_scales_sharded: the scales of this shard's K channels as in
 *     ttq_awq_scales, but with mbar = *total / K_total, where *total (device
 *     double) is the added total and K_total the layer's channel count.
 * Invalid pointers, sizes or K_total < K return TTQ_ERR_INVALID_ARG. With
 * one shard (K_total = K) the scales equal ttq_awq_scales' to the rounding
 * of the fp64 mean. */
ttq_status ttq_channel_moment_total(const float* sum, int64_t T_total,
                                    int64_t K, double* total, void* stream);
ttq_status ttq_awq_scales_sharded(const float* sum, int64_t T_total, int64_t K,
                                  int64_t K_total, const ttq_params* prm,
                                  const double* total, float* s, float* inv_s,
                                  void* stream);

/* Steps 1 and 2 in one launch: ttq_act_stats on X followed by
 * ttq_awq_scales on the resulting sums, with the same arithmetic (TTQ
 * review, Proposed method, bullets 2-4). The CTAs that finish the
 * statistics last compute the scales, so nothing waits and no second launch
 * is needed.
 *   X, T, K, ldx, accumulate, sum_out   as for ttq_act_stats (p = prm->p).
 *   T_total  token count behind sum_out (T, or the running total when
 *            accumulate == 1); the scales divide by it.
 *   prm      alpha, lambda and p as for ttq_awq_scales.
 *   s, inv_s [K] float32 outputs as for ttq_awq_scales.
 *   counter  one uint32 of device memory that is zero before the first call;
 *            every call leaves it zero again. Calls that may run at the same
 *            time (different streams) need different counters. After a
 *            call that failed on the device, zero it again.
 * sum_out, s, inv_s and counter must not overlap (s holds partial results
 * during the launch); overlapping arguments return TTQ_ERR_INVALID_ARG.
 * sum_out is bit-identical to ttq_act_stats; s and inv_s agree with
 * ttq_awq_scales to the last few bits of the fp64 mean (the mean is summed
 * in a different fixed order). */
ttq_status ttq_act_stats_scales(const void* X, ttq_dtype xt, int64_t T,
                                int64_t K, int64_t ldx, int accumulate,
                                int64_t T_total, const ttq_params* prm,
                                float* sum_out, float* s, float* inv_s,
                                uint32_t* counter, void* stream);

/* Step 3, group-wise RTN of the scaled weights (TTQ review, Proposed
 * method, bullet 1). For row n and group G, in fp32 with IEEE round-to-
 * nearest-even for every operation and no fused multiply-add:
 *   w_j  = float(W[n][j]) * s_j                  (s == NULL means s_j = 1)
 *   mn   = min(0, min_G w_j),  mx = max(0, max_G w_j)
 *   D    = (mx - mn) / (2^b - 1);  D = 1 when it is 0
 *   z    = clamp(rint(-mn / D), 0, 2^b - 1)
 *   q_j  = clamp(rint(w_j / D) + z, 0, 2^b - 1)
 * where rint rounds half to even. Outputs codes (layout above), delta = D,
 * zero = z; padding is zeroed.
 *   W      [N, K] of dtype wt, row pitch ldw.
 * D and z are exactly these values. For the codes the kernel rounds the
 * exact product w_j * RN(1/D) to an integer (one rounded reciprocal per
 * group); that product lies within 2^-24 |w_j / D| of the quotient, so a
 * code can differ from the formula only where the IEEE quotient w_j / D is
 * within one fp32 step of a half-integer (a near-tie, about one weight in
 * 10^5 to 10^6 at 8 bits, fewer at fewer).
 * Requires 2 <= bits <= 8, group in {16,32,64,128}, K % 32 == 0,
 * K % group == 0. Deterministic. */
ttq_status ttq_quantize_rtn_grouped(const void* W, ttq_dtype wt, int64_t N,
                                    int64_t K, int64_t ldw, const float* s,
                                    int bits, int group, uint32_t* codes,
                                    float* delta, uint8_t* zero, void* stream);

/* Bytes of workspace ttq_w_lowbit_gemm needs for a T x K input. */
size_t ttq_w_lowbit_gemm_workspace_size(int64_t T, int64_t K, int r);

/* Step 4, the quantized projection with dequantisation inside the GEMM
 * (TTQ review, Proposed method, bullets 1 and 7; bullet 5 for the optional
 * low-rank term):
 *   Y[t][n] = sum_j (X[t][j] * inv_s[j]) * (q[n][j] - z) * D
 *             + sum_rho (sum_j X[t][j] A[rho][j]) * B[n][rho]   (if r > 0)
 *   X      [T, K] of dtype xt, row pitch ldx.
 *   inv_s  [K] float32 (from ttq_awq_scales).
 *   codes, delta, zero: from ttq_quantize_rtn_grouped for an [N, K] weight.
 *   A      [r, K], B [N, r], dtype xt, dense; NULL with r == 0 for none.
 *   Y      [T, N] of dtype yt (F32, BF16 or F16), row pitch ldy.
 *   workspace  device buffer of at least
 *              ttq_w_lowbit_gemm_workspace_size(T, K, r) bytes; its contents
 *              are scratch and are overwritten.
 * The tensor cores take fp16 operands: X / s is rounded once to fp16 and
 * each weight (q - z) * D once to fp16; products accumulate in fp32.
 * |X / s| must stay below 65504 (else TTQ_DEVERR_FP16_RANGE is raised).
 * Which kernel runs depends on T: T <= 2 a CUDA-core matrix-vector product
 * (the weight (q - z) D is applied in fp32, the activations are the fp16
 * X / s) when its staged activations (about 4.75 T K bytes) fit its shared
 * memory, otherwise and up to T = 32 the tensor-core decode configuration
 * (K split across a cluster), larger T the prefill one. The results agree to the tolerances
 * of the parity tests, not bit for bit across these regimes.
 * Requires K % 32 == 0, K % group == 0, 0 <= r <= 64. */
ttq_status ttq_w_lowbit_gemm(const void* X, ttq_dtype xt, int64_t T,
                             int64_t K, int64_t ldx, const float* inv_s,
                             const uint32_t* codes, const float* delta,
                             const uint8_t* zero, int64_t N, int bits,
                             int group, const void* A, const void* B, int r,
                             void* Y, ttq_dtype yt, int64_t ldy,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/* The two halves of ttq_w_lowbit_gemm, for callers that reuse one prepared
 * input across several projections of the same X (q, k, v share X and s)
 * or time the tensor-core kernel alone.
 *
 * ttq_prepare_activations: the activation side of step 4.
 *   Xs[t][P(j)] = fp16(X[t][j] * inv_s[j])     Xs [T, K] fp16, dense
 * where P permutes channels inside each aligned span of 16 to match the
 * order in which the kernel unpacks `bits`-bit codes: for bits = 2, 4, 8
 * position p of a span holds channel (p>>1) + 8(p&1), 8(p>>3) + ((p&7)>>1)
 * + 4(p&1), or 4(p>>2) + ((p&3)>>1) + 2(p&1) of that span; for other widths
 * P is the identity. Xs is therefore only valid for codes of that width.
 *   U[t][rho] = fp16(sum_j X[t][j] A[rho][j])  U [T, 64] fp16, dense, zero
 *                                               for rho >= r (r > 0 only)
 * A is [r, K] of dtype xt; pass A = U = NULL with r = 0.
 * Raises TTQ_DEVERR_FP16_RANGE if |X * inv_s| reaches the fp16 range. */
ttq_status ttq_prepare_activations(const void* X, ttq_dtype xt, int64_t T,
                                   int64_t K, int64_t ldx, const float* inv_s,
                                   int bits, const void* A, int r, void* Xs,
                                   void* U, void* stream);

/* ttq_w_lowbit_gemm_prepared: the projection on prepared operands, one
 * kernel launch (T <= 2: CUDA cores, otherwise tensor cores, as above):
 *   Y[t][n] = sum_j Xs[t][j] (q[n][j] - z) D + sum_rho U[t][rho] B[n][rho].
 * Xs, U as written by ttq_prepare_activations for the same bits; B [N, r]
 * of dtype bt. */
ttq_status ttq_w_lowbit_gemm_prepared(const void* Xs, const void* U,
                                      int64_t T, int64_t K,
                                      const uint32_t* codes,
                                      const float* delta, const uint8_t* zero,
                                      int64_t N, int bits, int group,
                                      const void* B, ttq_dtype bt, int r,
                                      void* Y, ttq_dtype yt, int64_t ldy,
                                      void* stream);

/* Steps 3 and 4 in one launch: the projection quantizes the weights
 * itself (TTQ review, Proposed method, bullet 1: group-wise RTN with QDQ,
 * quantize then dequantize inside the projection). The tensor-core
 * producer loads bf16 tiles of W; the dequantiser warps quantize each
 * 128-channel stage exactly as ttq_quantize_rtn_grouped does (same codes,
 * delta and zero, the same near-tie behaviour), dequantise as the codes
 * path does and feed the tensor cores; Y equals ttq_w_lowbit_gemm_prepared
 * on ttq_quantize_rtn_grouped's output bit for bit.
 *   W        [N, K] bf16, row pitch ldw (16-byte aligned rows); s [K]
 *            float32 scales (ttq_awq_scales), 16-byte aligned.
 *   Xs, U, B, r, Y, yt, ldy   as for ttq_w_lowbit_gemm_prepared.
 *   codes, delta, zero   where to store the quantized weights for later
 *            (decode) use, in the layout above, written once by the CTAs of
 *            the first token tile; all three NULL to skip. Row padding is
 *            left untouched.
 * Every token tile quantizes its weight tiles again, so the form pays off
 * where the prompt spans few token tiles. Only the prefill tile (T > 32)
 * runs it, and W must be bf16: otherwise TTQ_ERR_UNSUPPORTED. */
ttq_status ttq_quantize_gemm_prepared(
    const void* W, ttq_dtype wt, int64_t ldw, const float* s, const void* Xs,
    const void* U, int64_t T, int64_t K, int64_t N, int bits, int group,
    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
    uint32_t* codes, float* delta, uint8_t* zero, void* stream);

/* The projection on prepared operands that also emits the statistic of
 * its own output for the layer that takes that output as input (TTQ
 * review, Proposed method, bullets 2-3: the next layer's per-channel
 * statistic, here computed in the projection's epilogue instead of by a
 * separate pass over Y). Same arguments and Y as
 * ttq_w_lowbit_gemm_prepared, plus:
 *   p        moment order (> 0) of the statistic;
 *   stats    [stats_rows][N] float32 device buffer of partial sums:
 *            row i holds, for every output channel n, the sum of
 *            |Y[t][n]|^p over one range of tokens, Y[t][n] being the value
 *            stored in Y (after rounding to yt); ranges are disjoint and
 *            cover all T tokens;
 *   stats_rows  must equal ttq_projection_stats_rows(T, N, K, bits).
 * ttq_stats_reduce then gives sum_out[n] = sum_t |Y[t][n]|^p, the input
 * of ttq_awq_scales for that layer. Only the tensor-core prefill form
 * (T > 32) computes it: for T <= 32 ttq_projection_stats_rows returns 0 and
 * the call returns TTQ_ERR_UNSUPPORTED. A wrong stats_rows or a bad p
 * returns TTQ_ERR_INVALID_ARG. */
int64_t ttq_projection_stats_rows(int64_t T, int64_t N, int64_t K, int bits);
ttq_status ttq_w_lowbit_gemm_prepared_stats(
    const void* Xs, const void* U, int64_t T, int64_t K, const uint32_t* codes,
    const float* delta, const uint8_t* zero, int64_t N, int bits, int group,
    const void* B, ttq_dtype bt, int r, void* Y, ttq_dtype yt, int64_t ldy,
    float p, float* stats, int64_t stats_rows, void* stream);

/* sum_out[n] (+)= sum_i partials[i][n] over the P rows in order (fp32,
 * deterministic). partials [P][N], sum_out [N], device; accumulate 0 or 1.
 * Invalid arguments return TTQ_ERR_INVALID_ARG. */
ttq_status ttq_stats_reduce(const float* partials, int64_t P, int64_t N,
                            int accumulate, float* sum_out, void* stream);

/* ttq_w_lowbit_gemm without a workspace argument, for callers that cannot
 * allocate device memory where they run the projection (a plugin called by
 * an inference engine after the engine fixed its memory plan, or host code
 * that only receives device pointers and has no allocator). The pages have
 * no counterpart to this call; it is a deployment convenience.
 *
 * Same arguments and results as ttq_w_lowbit_gemm. The scratch it needs
 * comes from an array built into the library, TTQ_NOALLOC_SCRATCH_BYTES on
 * every GPU that loads the library, kept until the process exits. It calls
 * no allocator.
 *   - Inputs whose workspace (ttq_w_lowbit_gemm_workspace_size(T, K, r))
 *     exceeds TTQ_NOALLOC_SCRATCH_BYTES return TTQ_ERR_UNSUPPORTED and
 *     enqueue nothing; use ttq_w_lowbit_gemm for them.
 *   - The first call on a device looks up the array's address on that
 *     device (set-up done once per device); make that first call before
 *     any stream capture.
 *   - All calls share the one array and it keeps the last call's contents,
 *     so calls whose execution overlaps on the GPU (other streams or host
 *     threads) race; serialise them. */
#define TTQ_NOALLOC_SCRATCH_BYTES (16u << 20)
ttq_status ttq_w_lowbit_gemm_noalloc(const void* X, ttq_dtype xt, int64_t T,
                                     int64_t K, int64_t ldx,
                                     const float* inv_s,
                                     const uint32_t* codes,
                                     const float* delta, const uint8_t* zero,
                                     int64_t N, int bits, int group,
                                     const void* A, const void* B, int r,
                                     void* Y, ttq_dtype yt, int64_t ldy,
                                     void* stream);

/* The low-rank term alone (TTQ review, Proposed method, bullet 5; Main
 * results, bullet 4): Y[t][n] += sum_rho (sum_j X[t][j] A[rho][j]) B[n][rho].
 * X [T, K], A [r, K], B [N, r] of dtype xt; Y [T, N] of dtype yt, pitch ldy.
 * Accumulates in fp32; 1 <= r <= 64. */
ttq_status ttq_lowrank_add(const void* X, ttq_dtype xt, int64_t T, int64_t K,
                           int64_t ldx, const void* A, const void* B, int r,
                           int64_t N, void* Y, ttq_dtype yt, int64_t ldy,
                           void* stream);

/* Per-prompt ("dynamic") low-rank factors (TTQ review, Proposed method,
 * bullet 5: W = W_q + B A with dynamic B, A and W_q quantized on the fly;
 * Main results, bullet 4: TTQ quantizes the residual). With TTQ's scales s
 * of the prompt, the factors span the dominant r-dimensional column space
 * of W_s = W diag(s), found by randomized subspace iteration (Halko,
 * Martinsson and Tropp 2011, Algorithm 4.4) from r probe vectors omega:
 *   Q = orth(W_s omega^T);  iters times: Z = orth(W_s^T Q), Q = orth(W_s Z)
 *   B = bf16(Q) [N, r],  A = bf16(Q^T W) [r, K]     (B A = Q Q^T W)
 * orth() orthonormalises the columns in order (Gram-Schmidt's order) and
 * drops a column whose part orthogonal to the kept ones has a norm of at
 * most 2^-10 of the input's largest column (that column of B is zero).
 *   W      bf16 [N, K], row pitch ldw (ldw >= K, ldw % 8 == 0), 16-byte
 *          aligned (read by TMA).
 *   s      fp32 [K] scales of step 2 (positive).
 *   omega  fp32 [r, K] probe vectors the caller draws (standard Gaussian);
 *          the call is deterministic given them.
 *   B, A   bf16 outputs, dense [N, r] and [r, K], 2-byte aligned; the
 *          layout ttq_w_lowbit_gemm takes for its low-rank term.
 *   1 <= r <= 64, 0 <= iters <= 16.
 * workspace: ttq_lowrank_factors_workspace_size(N, K, r) bytes, 256-byte
 * aligned, caller-owned, not used concurrently by another call. The
 * products with W run on the tensor cores with fp16 operands (W and the
 * basis rounded to fp16), fp32 accumulation; the orthonormalisation runs a
 * Cholesky factorisation in fp64. Argument errors return
 * TTQ_ERR_INVALID_ARG before anything is enqueued; a weight beyond fp16's
 * range raises TTQ_DEVERR_FP16_RANGE. */
size_t ttq_lowrank_factors_workspace_size(int64_t N, int64_t K, int r);
ttq_status ttq_lowrank_factors(const void* W, int64_t N, int64_t K,
                               int64_t ldw, const float* s, const float* omega,
                               int r, int iters, void* B, void* A,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* The residual TTQ quantizes when W = W_q + B A (TTQ review, Main results,
 * bullet 4): R = bf16(W - B A), each element accumulated from W in fp32 by
 * fused multiply-adds in the order j = 0 .. r-1 and rounded to bf16 once.
 * W, R bf16 [N, K] with pitches ldw, ldr (multiples of 8, rows 16-byte
 * aligned); B bf16 [N, r], A bf16 [r, K] dense; 1 <= r <= 64. R may be W
 * itself (ldr == ldw) but must not overlap it otherwise, nor B or A. */
ttq_status ttq_lowrank_residual(const void* W, int64_t N, int64_t K,
                                int64_t ldw, const void* B, const void* A,
                                int r, void* R, int64_t ldr, void* stream);

/* Expand packed codes to one uint8 per weight: q_out [N][K] (device).
 * Inverse of the packing in ttq_quantize_rtn_grouped. */
ttq_status ttq_unpack_codes(const uint32_t* codes, int64_t N, int64_t K,
                            int bits, uint8_t* q_out, void* stream);

/* Human-readable name of a status. Never NULL. */
const char* ttq_status_string(ttq_status status);

/* Reads the sticky device error word of the current device (a
 * synchronising copy; call it outside the hot loop). Clears it when clear
 * is non-zero. Returns the TTQ_DEVERR_* bits, or -1 if the copy failed. */
int ttq_device_error(int clear);

/* Self-test of the failure path shared by every kernel's waits: one
 * device thread initialises an mbarrier and waits for its first phase with
 * the same bounded wait the kernels use. With arrive != 0 the thread
 * arrives first and the wait completes (*out = 1). With arrive == 0
 * nothing ever arrives: after about 1.5 s of SM clocks the wait gives up,
 * raises TTQ_DEVERR_TIMEOUT in the sticky error word and the kernel returns
 * normally (*out = 0), leaving the context usable. out: one device uint32,
 * 4-byte aligned, written asynchronously on `stream`. Returns
 * TTQ_ERR_INVALID_ARG for a NULL or misaligned out, TTQ_ERR_CUDA if the
 * launch fails. Not part of the method; for tests of error handling. */
ttq_status ttq_selftest_bounded_wait(int arrive, uint32_t* out, void* stream);

/* ABI version of this header (3: ttq_act_stats_scales added; 4:
 * ttq_selftest_bounded_wait added; 5: ttq_channel_moment_total and
 * ttq_awq_scales_sharded added; 6: ttq_projection_stats_rows,
 * ttq_w_lowbit_gemm_prepared_stats and ttq_stats_reduce added; 7:
 * ttq_quantize_gemm_prepared added; 8: ttq_lowrank_factors,
 * ttq_lowrank_factors_workspace_size and ttq_lowrank_residual added). */
int ttq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTQ_H_ */
