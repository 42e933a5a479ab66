/*
 * hifa4.h -- C ABI of the B200 (sm_100a) 4-bit FlashAttention forward with
 * Smooth-QK and P-Reordering.
 *
 * Method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for
 * LLM Inference" (arXiv 2607.04302), Abstract paragraphs 1-2: both QK^T and PV
 * run as 4-bit GEMMs with an online softmax state (running max m, normalizer
 * l); Smooth-QK rescales post-RoPE Q by s and K by 1/s with calibration-static
 * per-channel scales; P-Reordering accumulates l from the same quantized
 * weights P-hat that feed the PV GEMM, fused into that GEMM.  The paper's HIF4
 * format is replaced by Blackwell's block-scaled E2M1: NVFP4 (one UE4M3 scale
 * per 16 elements) or MXFP4 (one UE8M0 scale per 32 elements, OCP MX v1.0).
 *
 * Conventions for every entry point:
 *  - All pointers named as device pointers must point to device memory of the
 *    current CUDA device; the caller owns and allocates all memory.  The
 *    library never allocates, frees or synchronizes.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Outputs are valid once the stream reaches the call.
 *  - Argument validation is synchronous and returns HIFA4_ERR_INVALID_ARG or
 *    HIFA4_ERR_UNSUPPORTED without launching anything; a failed launch
 *    returns HIFA4_ERR_CUDA.  hifa4_last_error() gives a thread-local detail
 *    string for the last failing call on the calling thread.
 *  - Kernels bound every internal wait.  A wait that runs out (a protocol
 *    error, never expected) ends the kernel early and sets a device error
 *    word; hifa4_device_error() returns and clears it (it synchronizes the
 *    device).  No call traps or asserts on the device.
 *  - Element layouts (N padded to Np = ceil(N/128)*128; pad rows/tokens hold
 *    zero codes and zero scales):
 *      Q-hat codes   [B][Hq][Np][d/2]   bytes, element 2i in the low nibble
 *      K-hat codes   [B][Hkv][Np][d/2]
 *      V-hat^T codes [B][Hkv][d][Np/2]  channel-major (tokens contiguous)
 *    Scale layouts are "tiled" per head: for a matrix of R rows (padded to
 *    128) and nb blocks per row (padded to a multiple of 4), 512-byte chunks
 *    ordered (row/128, block/4); inside a chunk, the scale of (row r, block b)
 *    is at byte (r%32)*16 + ((r%128)/32)*4 + (b%4).  hifa4_scale_bytes()
 *    gives the size of one head's scale matrix; the per-head matrices of a
 *    tensor are stored back to back in [B][H] order.
 *  - All pointers must be 16-byte aligned.
 */
#ifndef HIFA4_H_
#define HIFA4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HIFA4_OK = 0,
  HIFA4_ERR_INVALID_ARG = 1,
  HIFA4_ERR_UNSUPPORTED = 2,
  HIFA4_ERR_CUDA = 3,
  HIFA4_ERR_TIMEOUT = 4
} hifa4_status;

typedef enum { HIFA4_NVFP4 = 0, HIFA4_MXFP4 = 1 } hifa4_format;

/* P-Reordering (normalizer from P-hat, fused into the PV MMA) or the
 * inconsistent higher-precision normalizer (from unquantized P). */
typedef enum { HIFA4_NORM_PREORDER = 0, HIFA4_NORM_INCONSISTENT = 1 } hifa4_norm_mode;

typedef enum { HIFA4_BF16 = 0, HIFA4_FP16 = 1 } hifa4_dtype;

/* P-hat of NVFP4 uses a two-level scale: UE4M3 block scale times the global
 * prescale 2^HIFA4_NVFP4_P_PRESCALE_LOG2 (a reading: the paper does not define
 * the HIF4 P-hat scale).  MXFP4 P-hat uses the plain OCP rule. */
#define HIFA4_NVFP4_P_PRESCALE_LOG2 (-8)

typedef void* hifa4_stream_t; /* a cudaStream_t */

#if defined(__GNUC__)
#define HIFA4_API __attribute__((visibility("default")))
#else
#define HIFA4_API
#endif

/* ---------------------------------------------------------------- sizes --- */

/* Bytes of one head's codes for `rows` rows of `k` elements (rows padded to
 * 128): pad128(rows) * k / 2. */
HIFA4_API size_t hifa4_codes_bytes(int64_t rows, int k);

/* Bytes of one head's tiled scale matrix for `rows` rows of `k` elements
 * (rows padded to 128, blocks per row padded to a multiple of 4). */
HIFA4_API size_t hifa4_scale_bytes(int64_t rows, int k, hifa4_format fmt);

/* ------------------------------------------------------- calibration --- */

/* Smooth-QK calibration (paper Abstract para 2: "computed once from a small
 * offline calibration set"; the formula is a reading).  For kv head h and
 * channel c: aK = max|K[b,h,t,c]|, aQ = max|Q[b,hq,t,c]| over batches b,
 * tokens t < n_cal and the G = Hq/Hkv query heads hq of group h;
 *   s = clamp(aK^alpha / aQ^(1-alpha), 2^-16, 2^16) in fp64 -> fp32,
 *   inv_s = fl32(1/s); s = inv_s = 1 where enable == 0 or an amax is 0.
 * enable == 2 applies an applicability gate per kv head (the paper's Abstract
 * para 3 names a gate without a rule; this rule is a reading): smoothing is
 * on for head h iff max_c aK[h][c] > 8 * median_c aK[h][c] (the median of the
 * d channels is the mean of the two middle order statistics), decided in
 * fp64; otherwise s = inv_s = 1 for that head.
 * q: device [B][Hq][ld_tok][d], k: device [B][Hkv][ld_tok][d] of `dt`;
 * s_out, inv_s_out: device float [Hkv][d].  Requires 0 < n_cal <= ld_tok,
 * Hq % Hkv == 0, d in {64, 128, 256}.  Issues two small kernels. */
HIFA4_API hifa4_status hifa4_calibrate_smooth_qk(const void* q, const void* k, hifa4_dtype dt, int B, int Hq,
                                       int Hkv, int n_cal, int ld_tok, int d, float alpha,
                                       int enable, float* s_out, float* inv_s_out,
                                       hifa4_stream_t stream);

/* -------------------------------------------------- scale + quantize --- */

/* Fused Smooth-QK scale and block quantization (paper Abstract para 2: "only
 * a fusible element-wise scaling").  q' = fl32(q*s[h(hq),c]) and
 * k' = fl32(k*inv_s[h,c]) are quantized in blocks along d; V (unscaled) is
 * quantized in blocks along tokens and written transposed.  Block rule:
 * NVFP4 amax/6 -> UE4M3 (RNE, saturating) and codes E2M1(x * fl32(1/scale));
 * MXFP4 E = floor(log2 amax) - 2 and codes E2M1(x * 2^-E).
 * Inputs (device): q [B][Hq][N][d], k, v [B][Hkv][N][d] of `dt`; s, inv_s
 * device float [Hkv][d] or NULL (= 1).  Outputs (device): the code and tiled
 * scale layouts described at the top of this file (q_scales: B*Hq heads of
 * hifa4_scale_bytes(N, d), k_scales: B*Hkv of hifa4_scale_bytes(N, d),
 * vt_scales: B*Hkv of hifa4_scale_bytes(d, Np)).  Requires N >= 1,
 * d in {64, 128, 256}, Hq % Hkv == 0. */
HIFA4_API hifa4_status hifa4_quantize_qkv(const void* q, const void* k, const void* v, hifa4_dtype dt, int B,
                                int Hq, int Hkv, int N, int d, const float* s, const float* inv_s,
                                hifa4_format fmt, uint8_t* q_codes, uint8_t* q_scales,
                                uint8_t* k_codes, uint8_t* k_scales, uint8_t* vt_codes,
                                uint8_t* vt_scales, hifa4_stream_t stream);

/* The K / V half of hifa4_quantize_qkv, for building a 4-bit KV cache (the
 * decode path): k' = fl32(k*inv_s[h,c]) quantized along d and V quantized
 * along tokens into V-hat^T, with exactly the rules and layouts above.
 * k, v: device [B][Hkv][N][d] of `dt`; inv_s device float [Hkv][d] or NULL.
 * Same requirements as hifa4_quantize_qkv. */
HIFA4_API hifa4_status hifa4_quantize_kv(const void* k, const void* v, hifa4_dtype dt, int B, int Hkv, int N,
                                         int d, const float* inv_s, hifa4_format fmt, uint8_t* k_codes,
                                         uint8_t* k_scales, uint8_t* vt_codes, uint8_t* vt_scales,
                                         hifa4_stream_t stream);

/* ------------------------------------------------- Q-Mean auxiliary --- */

/* The pages name "the adopted Q-Mean auxiliary" (paper Abstract para 3) and
 * nothing more; the reading built here (off unless these entry points are
 * used): the per-channel calibration mean mu of the smoothed query is
 * subtracted before Q is quantized, and every score gets back the rank-one
 * term mu . K-hat of its key, so that without quantization the scores are
 * unchanged ((q - mu) . k + mu . k = q . k).  Use: hifa4_calibrate_q_mean ->
 * hifa4_quantize_qkv_qmean -> hifa4_q_mean_bias -> hifa4_attn_fwd_qmean. */

/* mu[hq][c] = fl32( sum_{b, t < n_cal} fl32(q[b][hq][t][c] * s[hq/G][c]) /
 * (B * n_cal) ), the sum in fp64 in the order b, then t (reproducible bit for
 * bit).  q: device [B][Hq][ld_tok][d] of `dt`; s: device float [Hkv][d] (the
 * Smooth-QK scales of hifa4_calibrate_smooth_qk) or NULL for 1; mu_out:
 * device float [Hq][d], caller-owned.  Requires 0 < n_cal <= ld_tok,
 * Hq % Hkv == 0, d in {64, 128, 256}. */
HIFA4_API hifa4_status hifa4_calibrate_q_mean(const void* q, hifa4_dtype dt, int B, int Hq, int Hkv, int n_cal,
                                              int ld_tok, int d, const float* s, float* mu_out,
                                              hifa4_stream_t stream);

/* hifa4_quantize_qkv with the Q-Mean auxiliary: rows t < N of Q quantize
 * fl32(fl32(q*s) - mu[hq]) (padding rows stay zero); K and V exactly as in
 * hifa4_quantize_qkv.  q_mu: device float [Hq][d], 16-byte aligned.  Other
 * arguments, layouts and requirements as hifa4_quantize_qkv. */
HIFA4_API hifa4_status hifa4_quantize_qkv_qmean(const void* q, const void* k, const void* v, hifa4_dtype dt,
                                                int B, int Hq, int Hkv, int N, int d, const float* s,
                                                const float* inv_s, const float* q_mu, hifa4_format fmt,
                                                uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes,
                                                uint8_t* k_scales, uint8_t* vt_codes, uint8_t* vt_scales,
                                                hifa4_stream_t stream);

/* The rank-one score term of the Q-Mean auxiliary: bias_out[b][hq][key] =
 * mu[hq] . K-hat[b][hq/G][key] (fp32) for every key of the padded rows
 * (Np = N rounded up to 128; padding keys give 0).  k_codes / k_scales: the
 * K-hat layouts of hifa4_quantize_qkv(_qmean) with the same fmt; q_mu:
 * device float [Hq][d]; bias_out: device float [B][Hq][Np], caller-owned.
 * Requires Hq / Hkv <= 8. */
HIFA4_API hifa4_status hifa4_q_mean_bias(const uint8_t* k_codes, const uint8_t* k_scales, const float* q_mu,
                                         int B, int Hq, int Hkv, int N, int d, hifa4_format fmt,
                                         float* bias_out, hifa4_stream_t stream);

/* ------------------------------------------------ attention forward --- */

/* 4-bit FlashAttention forward (paper Abstract paras 1-2).  For each (b, hq)
 * and 128-row query tile, key tiles of block_n keys are visited in ascending
 * order: S = Q-hat K-hat^T (block-scaled FP4 MMA, fp32 accumulate), online
 * softmax in fp32 with P = 2^(S*c - m) (c = softmax_scale*log2 e), P-hat =
 * per-block quantization of P (NVFP4 with the 2^-8 prescale, or MXFP4),
 * O += P-hat V-hat (FP4 MMA).  mode PREORDER accumulates l from P-hat inside
 * the PV MMA (a ones column); mode INCONSISTENT accumulates l from P in fp32.
 * Output O = acc / l in o_dt, [B][Hq][N][d]; lse (optional, [B][Hq][N]
 * float) = m + log2(l) in base 2.  dbg_l_phat / dbg_l_p (optional, [B][Hq][N]
 * float) receive the final normalizers from P-hat and from P (their ratio
 * minus one is the per-row normalizer error epsilon of Theorem 1).
 * Inputs are the layouts written by hifa4_quantize_qkv with the same fmt.
 * causal: top-left aligned (key <= query).  block_n: 0 (default 128), 64 or
 * 128.  Requires d in {64, 128, 256}, Hq % Hkv == 0, N >= 1. */
HIFA4_API hifa4_status hifa4_attn_fwd(const uint8_t* q_codes, const uint8_t* q_scales,
                            const uint8_t* k_codes, const uint8_t* k_scales,
                            const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                            int Hkv, int N, int d, hifa4_format fmt, float softmax_scale,
                            int causal, hifa4_norm_mode mode, int block_n, void* o,
                            hifa4_dtype o_dt, float* lse, float* dbg_l_phat, float* dbg_l_p,
                            hifa4_stream_t stream);

/* hifa4_attn_fwd with a lazily updated running max (the conditional rescaling
 * of FlashAttention-4; the paper states the exact online recurrence, which is
 * rescale_threshold = 0, i.e. hifa4_attn_fwd).  Per query row and key tile,
 * with x_t the tile's largest scaled score fl32(S*c):
 *   if x_t > fl32(m + rescale_threshold):  m_new = x_t, alpha = 2^(m - m_new)
 *   else:                                   m_new = m,   alpha = 1
 * (in fp32; m = -inf always moves).  P = 2^(x - m_new) may then reach
 * 2^rescale_threshold; P-hat is that P block-quantized by the same rules, and
 * O, l and lse follow the same recurrence, so without quantization the result
 * is exact attention for any threshold.  Tiles where no row of a warp moves
 * its max skip the O rescale and its wait for the previous PV product.
 * rescale_threshold in log2 units: [0, 3] for NVFP4 (P up to 2^3 keeps the
 * P-hat scale, fl32(amax/6)/2^-8, below UE4M3's 448), [0, 8] for MXFP4;
 * otherwise HIFA4_ERR_INVALID_ARG (NaN included). */
HIFA4_API hifa4_status hifa4_attn_fwd_ex(const uint8_t* q_codes, const uint8_t* q_scales,
                                         const uint8_t* k_codes, const uint8_t* k_scales,
                                         const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                                         int Hkv, int N, int d, hifa4_format fmt, float softmax_scale,
                                         int causal, hifa4_norm_mode mode, int block_n, void* o,
                                         hifa4_dtype o_dt, float* lse, float* dbg_l_phat, float* dbg_l_p,
                                         float rescale_threshold, hifa4_stream_t stream);

/* Debug view of hifa4_attn_fwd_ex: the same forward (o written as there),
 * plus the quantized attention weights P-hat exactly as the kernel feeds them
 * to the PV MMA (paper Abstract para 2: P-Reordering normalizes by "the same
 * quantized attention weights P-hat used in the PV GEMM"), for checking them
 * against a reference.  With nkt = ceil(N / block_n) key tiles per row and
 * beta = 16 (NVFP4) or 32 (MXFP4), for query row r of (b, hq) and key tile j:
 *   phat_codes  [B][Hq][N][nkt][block_n/2]    E2M1 codes of the tile's keys,
 *               key 2i in the low nibble (device, 16-byte aligned)
 *   phat_scales [B][Hq][N][nkt][block_n/beta] block scale codes (UE4M3 of
 *               the 2^-8-prescaled scale for NVFP4, UE8M0 for MXFP4)
 *   tile_m      [B][Hq][N][nkt] float: running max after tile j (log2 units
 *               of the scaled scores)
 *   tile_sum_p  [B][Hq][N][nkt] float, or NULL: sum of the unquantized P of
 *               tile j against that max (must be zero-filled by the caller)
 * Tiles past the end of a row's 128-row query tile under causal masking are
 * not visited and not written: the caller initializes the buffers.  With
 * tile_sum_p == NULL the kernel runs the variant hifa4_attn_fwd_ex runs
 * without debug sums (under P-Reordering part of each tile's codes are then
 * decided from the log2-domain argument without forming P); a non-NULL
 * tile_sum_p selects the variant that forms and sums P, as dbg_l_p does.
 * Other arguments, requirements and errors as hifa4_attn_fwd_ex; the dump
 * pointers must be non-NULL except tile_sum_p. */
HIFA4_API hifa4_status hifa4_attn_fwd_dump(const uint8_t* q_codes, const uint8_t* q_scales,
                                           const uint8_t* k_codes, const uint8_t* k_scales,
                                           const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                                           int Hkv, int N, int d, hifa4_format fmt, float softmax_scale,
                                           int causal, hifa4_norm_mode mode, int block_n, void* o,
                                           hifa4_dtype o_dt, float rescale_threshold, uint8_t* phat_codes,
                                           uint8_t* phat_scales, float* tile_m, float* tile_sum_p,
                                           hifa4_stream_t stream);

/* hifa4_attn_fwd_ex with the Q-Mean auxiliary: every score S of key k gets
 * qk_bias[b][hq][k] added before the softmax scaling (fl32(S + bias), then
 * as in hifa4_attn_fwd_ex).  Inputs: Q-hat from hifa4_quantize_qkv_qmean,
 * qk_bias from hifa4_q_mean_bias (device float [B][Hq][Np], 16-byte
 * aligned).  Runs in the kernel instantiation that carries the optional
 * extras.  Requires d in {64, 128} (the score terms ride on the key tile's
 * single K/V barrier, which the two-stage d = 256 pipeline does not use);
 * other arguments and requirements as hifa4_attn_fwd_ex (no debug sums). */
HIFA4_API hifa4_status hifa4_attn_fwd_qmean(const uint8_t* q_codes, const uint8_t* q_scales,
                                            const uint8_t* k_codes, const uint8_t* k_scales,
                                            const uint8_t* vt_codes, const uint8_t* vt_scales,
                                            const float* qk_bias, int B, int Hq, int Hkv, int N, int d,
                                            hifa4_format fmt, float softmax_scale, int causal,
                                            hifa4_norm_mode mode, int block_n, void* o, hifa4_dtype o_dt,
                                            float* lse, float rescale_threshold, hifa4_stream_t stream);

/* The prefill forward with Smooth-QK and the Q quantization fused into the
 * attention kernel (the paper's Abstract para 2: Smooth-QK needs "only a
 * fusible element-wise scaling"): q [B][Hq][N][d] in q_dt, unscaled and
 * unquantized (device); s the Smooth-QK scales [Hkv][d] fp32 (device) or
 * NULL for 1.  Each CTA scales and quantizes its 128-row query tile itself,
 * by exactly the rules of hifa4_quantize_qkv (q' = fl32(q * s[h]), blocks
 * along d), so the result equals hifa4_quantize_qkv + hifa4_attn_fwd_ex
 * bit for bit, without the round trip of Q-hat through memory.  K and V come
 * quantized (hifa4_quantize_kv with inv_s = 1/s).  Other arguments,
 * requirements and errors as hifa4_attn_fwd_ex. */
HIFA4_API hifa4_status hifa4_attn_fwd_fused(const void* q, hifa4_dtype q_dt, const float* s,
                                            const uint8_t* k_codes, const uint8_t* k_scales,
                                            const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                                            int Hkv, int N, int d, hifa4_format fmt, float softmax_scale,
                                            int causal, hifa4_norm_mode mode, int block_n, void* o,
                                            hifa4_dtype o_dt, float* lse, float* dbg_l_phat, float* dbg_l_p,
                                            float rescale_threshold, hifa4_stream_t stream);

/* ----------------------------------------------------- split-KV decode --- */

/* Workspace bytes for hifa4_attn_decode with `num_splits` splits (per split
 * and query row: d accumulators plus m and l, fp32). */
HIFA4_API size_t hifa4_decode_workspace_size(int B, int Hq, int d, int num_splits);

/* Split count chosen by hifa4_attn_decode when num_splits == 0. */
HIFA4_API int hifa4_decode_default_splits(int B, int Hkv, int kv_len, int block_n);

/* One decode step over a 4-bit KV cache: the split-KV decode workload of the
 * 4-bit path (B = 64 sequences, one query each, 32768 cached tokens, GQA
 * 32 / 8, d = 128), the prefill recurrence of the paper's Abstract paras 1-2
 * over a cache quantized once.  The cache layouts are those of
 * hifa4_quantize_qkv with N = kv_len.  q: device [B][Hq][d] of q_dt,
 * unscaled; s: device float [Hkv][d] Smooth-QK scales or NULL.  Inside the
 * kernel each query row is scaled (fl32(q*s)) and quantized by the Q rule.
 * Keys split into chunks of L = ceil(kv_len/num_splits) rounded up to
 * block_n; each split runs the prefill recurrence without a mask and writes
 * (acc, m, l) to `workspace`; a combine kernel merges them:
 * O = sum 2^(m_s-M) acc_s / sum 2^(m_s-M) l_s.  o: device [B][Hq][d] of o_dt.
 * num_splits 0 = hifa4_decode_default_splits; *num_splits_used (optional,
 * host) receives the count of non-empty splits.  Requires d == 128,
 * Hq/Hkv in {1, 2, 4, 8}, block_n == 0 or 128. */
HIFA4_API hifa4_status hifa4_attn_decode(const void* q, hifa4_dtype q_dt, const float* s,
                               const uint8_t* k_codes, const uint8_t* k_scales,
                               const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                               int Hkv, int kv_len, int d, hifa4_format fmt, float softmax_scale,
                               hifa4_norm_mode mode, int block_n, int num_splits,
                               int* num_splits_used, void* workspace, size_t ws_bytes, void* o,
                               hifa4_dtype o_dt, hifa4_stream_t stream);

/* ------------------------------------------------- appendable cache --- */

/* A KV cache that grows by appends, for decode loops.  Its buffers have the
 * hifa4_quantize_kv layouts for a fixed `capacity` tokens (Np =
 * pad128(capacity): k_codes [B][Hkv][Np][d/2], k_scales
 * hifa4_scale_bytes(capacity, d) per head, vt_codes [B][Hkv][d][Np/2],
 * vt_scales hifa4_scale_bytes(d, Np) per head), all zero before the first
 * append, plus v_tail [B][Hkv][beta][d] (dt): the raw V values of the
 * partially filled last block of beta tokens (beta = 16 NVFP4, 32 MXFP4),
 * owned by the caller and passed unchanged between appends.
 *
 * Appends tokens [pos, pos + T) from k_new, v_new [B][Hkv][T][d] (dt, device):
 * K rows scaled by inv_s ([Hkv][d] fp32, or NULL for 1) and block-quantized;
 * every V block the new tokens touch is quantized again from its raw values
 * (older tokens of the block from v_tail, tokens not yet written as 0); v_tail
 * is updated.  After appends covering [0, L), the cache equals
 * hifa4_quantize_kv of the L tokens laid out at this capacity, bit for bit.
 * Requires 0 <= pos, T >= 1, pos + T <= capacity, d in {64, 128, 256}.  One
 * kernel launch on `stream`; no host synchronization. */
HIFA4_API hifa4_status hifa4_kv_cache_append(const void* k_new, const void* v_new, hifa4_dtype dt, int B, int Hkv,
                                             int T, int d, const float* inv_s, hifa4_format fmt, int pos,
                                             int capacity, uint8_t* k_codes, uint8_t* k_scales, uint8_t* vt_codes,
                                             uint8_t* vt_scales, void* v_tail, hifa4_stream_t stream);

/* hifa4_attn_decode over the first kv_len tokens of an appendable cache laid
 * out for kv_capacity tokens (kv_len <= kv_capacity), with each split's
 * running max updated lazily by rescale_threshold under the rule of
 * hifa4_attn_fwd_ex (0 = the exact recurrence; same bounds); same arguments
 * and results otherwise.  hifa4_attn_decode is the case kv_capacity = kv_len,
 * rescale_threshold = 0. */
HIFA4_API hifa4_status hifa4_attn_decode_cache(const void* q, hifa4_dtype q_dt, const float* s,
                                               const uint8_t* k_codes, const uint8_t* k_scales,
                                               const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                                               int Hkv, int kv_len, int kv_capacity, int d, hifa4_format fmt,
                                               float softmax_scale, hifa4_norm_mode mode, int block_n,
                                               int num_splits, int* num_splits_used, void* workspace,
                                               size_t ws_bytes, void* o, hifa4_dtype o_dt,
                                               float rescale_threshold, hifa4_stream_t stream);

/* Decode for callers that cannot allocate device memory.  (The paper has no
 * counterpart; this is a deployment convenience of this library.)  Callers
 * such as an inference-server plugin or a framework custom operator that is
 * handed only its input and output buffers (the host framework's allocator
 * owns all device memory), or a latency-critical serving loop where a device
 * allocation may block or synchronize, cannot provide the workspace that
 * hifa4_attn_decode needs.  This entry point takes the same arguments minus
 * the workspace and keeps the split partials in a library-owned scratch array
 * in device global memory of hifa4_decode_noalloc_max_bytes() (16 MiB), which
 * every GPU that loads the library holds until the process exits.  It calls
 * no allocation routine.  A call needing more scratch than that (B * Hq *
 * splits_used * (d + 2) * 4 bytes) returns HIFA4_ERR_INVALID_ARG with the
 * sizes in hifa4_last_error().  The first call on a device looks up the
 * scratch's device address for that device (a CUDA runtime query), so make
 * that first call before any stream capture; the lookup is repeated when the
 * device's context has changed (after cudaDeviceReset, for instance).  All
 * calls on a device share the one scratch array: calls that overlap on the GPU
 * (concurrent streams) race on it and must be serialized by the caller.  The
 * scratch keeps the last call's contents; nothing in it needs to start at
 * zero: every split writes its partials before the combine reads them, and a
 * split whose bounded wait gave up writes NaN markers, so its output turns NaN
 * (with the device error word set) rather than reusing an earlier call's. */
HIFA4_API size_t hifa4_decode_noalloc_max_bytes(void);
HIFA4_API hifa4_status hifa4_attn_decode_noalloc(const void* q, hifa4_dtype q_dt, const float* s,
                                                 const uint8_t* k_codes, const uint8_t* k_scales,
                                                 const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq,
                                                 int Hkv, int kv_len, int d, hifa4_format fmt, float softmax_scale,
                                                 hifa4_norm_mode mode, int block_n, int num_splits,
                                                 int* num_splits_used, void* o, hifa4_dtype o_dt,
                                                 hifa4_stream_t stream);

/* -------------------------------------------------------- measurement --- */

/* One 128 x n block-scaled FP4 product D = A B^T (K-major A [128][k], B [n][k]
 * in the code/tiled-scale layouts above; d_out device float [128][n]),
 * repeated `repeats` times into the same accumulator (D = repeats * A B^T)
 * on each of `ctas` CTAs (CTA 0 writes d_out).  With repeats >> 1 and ctas a
 * multiple of the SM count this measures the dense FP4 tensor peak.
 * Requires n in {64, 128, 256}, k a multiple of 128 up to 512. */
HIFA4_API hifa4_status hifa4_fp4_mma_probe(const uint8_t* a_codes, const uint8_t* a_scales,
                                 const uint8_t* b_codes, const uint8_t* b_scales, int n, int k,
                                 hifa4_format fmt, int repeats, int ctas, float* d_out,
                                 hifa4_stream_t stream);

/* E2M1 / UE4M3 hardware conversion of `count` fp32 values (device): e2m1_out
 * [count] codes (1 per byte) and e4m3_out [count] saturating E4M3 codes.  Used
 * to check the written rounding rules against the conversion instructions. */
HIFA4_API hifa4_status hifa4_convert_probe(const float* x, int64_t count, uint8_t* e2m1_out,
                                 uint8_t* e4m3_out, hifa4_stream_t stream);

/* Conformance of the kernels' fast fl32(a/6) (reciprocal plus one exact
 * residual correction) with IEEE division, and of its variant with 2^8 folded
 * into the constants with 2^8 * fl32(a/6), for every float bit pattern in
 * [lo_bits, hi_bits): adds the number of patterns where either differs to *mismatches
 * and lowers *first_bad (both device; caller initializes 0 / 0xFFFFFFFF). */
HIFA4_API hifa4_status hifa4_div6_probe(uint32_t lo_bits, uint32_t hi_bits, unsigned long long* mismatches,
                                        uint32_t* first_bad, hifa4_stream_t stream);

/* ------------------------------------------------- BF16 reference --- */

/* Plain BF16 FlashAttention forward, the unquantized baseline the 4-bit path
 * is measured against (no Smooth-QK, no quantization; P rounded to bf16 for
 * the PV MMA, l summed in fp32 over the unrounded P).  All device pointers:
 *   q  [B, Hq, N, d] bf16, k [B, Hkv, N, d] bf16,
 *   vt [B, Hkv, d, N] bf16 (V transposed, see hifa4_bf16_transpose_v),
 *   o  [B, Hq, N, d] bf16 (written), lse [B, Hq, N] f32 base-2 log-sum-exp
 *   (m + log2 l of the scores times softmax_scale * log2 e) or NULL.
 * d in {64, 128, 256}; N a multiple of 8; Hq a multiple of Hkv (GQA); causal is
 * top-left aligned.  Pointers 16-byte aligned.  Asynchronous on `stream`. */
HIFA4_API hifa4_status hifa4_bf16_attn_fwd(const void* q, const void* k, const void* vt, int B, int Hq, int Hkv,
                                           int N, int d, float softmax_scale, int causal, void* o, float* lse,
                                           hifa4_stream_t stream);

/* V [B, Hkv, N, d] bf16 -> vt [B, Hkv, d, N] bf16 (device, no overlap). */
HIFA4_API hifa4_status hifa4_bf16_transpose_v(const void* v, int B, int Hkv, int N, int d, void* vt,
                                              hifa4_stream_t stream);

/* The FMA-pipe 2^y the prefill kernel uses for part of each P tile (range
 * reduction to the nearest integer plus a degree-4 polynomial, see ptx.cuh),
 * applied to `count` fp32 values y <= 0 (device in, device out).  Lets a test
 * hold its relative error to the fitted bound and check the y <= -127 -> 0
 * and y = 0 -> 1 edges. */
HIFA4_API hifa4_status hifa4_exp2_poly_probe(const float* y, int64_t count, float* out, hifa4_stream_t stream);

/* The exponential-free P-hat code decision the prefill kernel uses for its
 * FMA-pipe share of elements when only codes are needed (a cubic that equals
 * 2^f at the three E2M1 rounding edges it can meet, see ptx.cuh), applied to
 * `count` fp32 log2-domain values y <= 3.5: codes_map[i] = E2M1 code (RNE,
 * saturating) of that argument, codes_ex2[i] = the code of the MUFU 2^y,
 * one code per byte (device in, device out).  Lets a test compare both with
 * the written encoder of fl32(2^y). */
HIFA4_API hifa4_status hifa4_e2m1_map_probe(const float* y, int64_t count, uint8_t* codes_map, uint8_t* codes_ex2,
                                            hifa4_stream_t stream);

/* The kernels' failure path, exercised: one warp waits on an mbarrier that
 * nothing arrives at.  The bounded wait gives up after its limit (2 s), sets
 * its CTA's abort flag and the timeout bit 8 of the device error word, and the
 * kernel returns.  status (device, 2 words): [0] = 1 if the wait succeeded
 * (it must not), [1] = the abort flag.  The context stays usable; read and
 * clear the error word with hifa4_device_error(). */
HIFA4_API hifa4_status hifa4_wait_timeout_probe(unsigned int* status, hifa4_stream_t stream);

/* ----------------------------------------------------------- errors --- */

HIFA4_API const char* hifa4_status_string(hifa4_status st);
HIFA4_API const char* hifa4_last_error(void);
/* Synchronizes the device, returns the device error word and clears it
 * (0 = no kernel gave up a wait). */
HIFA4_API unsigned int hifa4_device_error(void);

#ifdef __cplusplus
}
#endif
#endif /* HIFA4_H_ */
