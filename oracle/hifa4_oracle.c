/*
 * hifa4_oracle.c -- plain, slow CPU oracle for the 4-bit FlashAttention forward
 * with Smooth-QK and P-Reordering.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA library under
 * bit_quantized_flashattention_smooth_b200/csrc, and the CUDA library never
 * calls it.
 *
 * Sources followed (page titles and sections):
 *   [HiFA4] "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for
 *           LLM Inference" (arXiv 2607.04302), Abstract paragraphs 1-3 and
 *           Section 1 (Introduction).
 *   [HiFA4-announce] the arXiv announcement abstract of the same paper
 *           (sign of the normalizer error: "net probability-mass loss").
 *   [MX]    OCP Microscaling Formats (MX) v1.0: E2M1 element, E8M0 scale,
 *           shared exponent = floor(log2(amax)) - emax_elem.
 *   [NVFP4] NVIDIA NVFP4: 16 E2M1 elements share one unsigned E4M3 scale.
 *
 * The pages never define HIF4, the Smooth-QK scale formula, the P-hat scale,
 * or epsilon; the reading taken for each is stated in the comment of the
 * function that implements it.  Attention and decode also take an optional
 * lazy running-max threshold tau (the conditional rescaling of
 * FlashAttention-4, which the pages do not describe); tau = 0 is the pages'
 * exact online recurrence.
 *
 * Arithmetic: everything that is not a 4-bit/8-bit format decision is done in
 * double precision.  Format decisions (block amax, scale, element rounding)
 * are made in IEEE single precision, as the written specification fixes them,
 * so that the CUDA path and the oracle take each integer decision in the same
 * precision.  Compile with -O2 -ffp-contract=off (no fused multiply-add, no
 * fast-math).
 *
 * Parity pins live in tests/test_oracle_*.py.  One item is "parity unpinned":
 * the magnitude of epsilon (the pages' -0.064 belongs to a real model trace).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_NVFP4 0
#define OR_MXFP4 1
#define OR_PREORDER 0
#define OR_INCONSISTENT 1

/* ------------------------------------------------------------------------ */
/* 1. Element and scale formats                                              */
/* ------------------------------------------------------------------------ */

/* E2M1 magnitudes by 3-bit code [MX, Table "FP4 E2M1"]. */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

int or_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double or_e2m1_decode(uint8_t code) {
  double mag = E2M1_GRID[code & 7];
  return (code & 8) ? -mag : mag;
}

/* Round-to-nearest-even onto the E2M1 grid, saturating at 6; the sign bit is
 * kept for negative inputs, including those that round to zero. */
uint8_t or_e2m1_encode(float y) {
  uint8_t sign = signbit(y) ? 8 : 0;
  double a = fabs((double)y);
  if (a >= 6.0) return sign | 7;
  for (int i = 0; i < 7; ++i) {
    double lo = E2M1_GRID[i], hi = E2M1_GRID[i + 1];
    if (a <= hi) {
      double mid = 0.5 * (lo + hi);  /* exact: the grid is dyadic */
      int pick;
      if (a < mid) pick = i;
      else if (a > mid) pick = i + 1;
      else pick = (i % 2 == 0) ? i : i + 1;  /* tie: even code */
      return sign | (uint8_t)pick;
    }
  }
  return sign | 7;
}

/* Unsigned E4M3 (E4M3FN with the sign bit forced to 0): bias 7, three
 * mantissa bits, subnormals m * 2^-9, 0x7F is NaN and never produced. */
double or_ue4m3_decode(uint8_t code) {
  int e = (code >> 3) & 15, m = code & 7;
  if (code >= 0x7F) return NAN;
  if (e == 0) return ldexp((double)m, -9);
  return ldexp(8.0 + m, e - 10);
}

/* RNE onto the UE4M3 grid for t >= 0, saturating at 448 (code 0x7E). */
uint8_t or_ue4m3_encode(float t) {
  double a = (double)t;
  if (!(a > 0.0)) return 0;
  if (a >= 448.0) return 0x7E;
  /* binary search for the largest code c with value(c) <= a */
  int lo = 0, hi = 0x7E;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (or_ue4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
  }
  int c = lo;
  double v0 = or_ue4m3_decode((uint8_t)c), v1 = or_ue4m3_decode((uint8_t)(c + 1));
  if (a == v0) return (uint8_t)c;
  double mid = 0.5 * (v0 + v1);
  if (a < mid) return (uint8_t)c;
  if (a > mid) return (uint8_t)(c + 1);
  return (uint8_t)((c % 2 == 0) ? c : c + 1);
}

/* UE8M0: 2^(code-127); 0xFF is NaN and never produced. */
double or_ue8m0_decode(uint8_t code) {
  if (code == 0xFF) return NAN;
  return ldexp(1.0, (int)code - 127);
}

/* Element-wise encoders over an array (for comparing with hardware
 * conversions): e2m1[i] = E2M1(x[i]); e4m3[i] = UE4M3(|x[i]|). */
void or_encode_array(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3) {
  #pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    e2m1[i] = or_e2m1_encode(x[i]);
    e4m3[i] = or_ue4m3_encode(fabsf(x[i]));
  }
}

/* ------------------------------------------------------------------------ */
/* 2. Block quantizers                                                       */
/* ------------------------------------------------------------------------ */

/* NVFP4 block of n=16 values with a power-of-two global prescale g:
 *   amax = max|x|;  t = fl32(fl32(amax/6)/g);  sc = UE4M3(t);
 *   sd = fl32(decode(sc)*g);  sd == 0 -> all codes 0;
 *   otherwise code_i = E2M1(fl32(x_i * fl32(1/sd))).
 * Returns sc; writes one code per element (low 4 bits). */
uint8_t or_quant_block_nvfp4(const float* x, int n, float g, uint8_t* codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  float t = (amax / 6.0f) / g;
  uint8_t sc = or_ue4m3_encode(t);
  float sd = (float)or_ue4m3_decode(sc) * g;
  if (sd == 0.0f) {
    for (int i = 0; i < n; ++i) codes[i] = 0;
    return sc;
  }
  float inv = 1.0f / sd;
  for (int i = 0; i < n; ++i) codes[i] = or_e2m1_encode(x[i] * inv);
  return sc;
}

/* Dequantized value of an NVFP4 element (with the same global prescale g). */
double or_dequant_nvfp4(uint8_t code, uint8_t sc, float g) {
  float sd = (float)or_ue4m3_decode(sc) * g;
  return or_e2m1_decode(code) * (double)sd;
}

/* MXFP4 shared exponent [MX]: E = clamp(floor(log2 amax) - 2, -127, 127),
 * with E = -127 for amax = 0. */
int or_mx_exponent(float amax) {
  if (amax == 0.0f) return -127;
  int e2;
  frexp((double)amax, &e2);      /* amax = f * 2^e2, f in [0.5, 1) */
  int E = (e2 - 1) - 2;
  if (E < -127) E = -127;
  if (E > 127) E = 127;
  return E;
}

/* MXFP4 block of n=32 values: code_i = E2M1(fl32(x_i * 2^-E)), scale code
 * E+127.  Values that land in [6, 8) after the shift clip to 6. */
uint8_t or_quant_block_mxfp4(const float* x, int n, uint8_t* codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  int E = or_mx_exponent(amax);
  for (int i = 0; i < n; ++i) {
    float y = (float)ldexp((double)x[i], -E);   /* one IEEE rounding */
    codes[i] = or_e2m1_encode(y);
  }
  return (uint8_t)(E + 127);
}

double or_dequant_mxfp4(uint8_t code, uint8_t sc) {
  return or_e2m1_decode(code) * or_ue8m0_decode(sc);
}

/* Quantize `rows` rows of K values along K in blocks of beta (16 NVFP4, 32
 * MXFP4).  codes: rows*K/2 bytes, element 2i in the low nibble of byte i and
 * element 2i+1 in the high nibble.  scales: plain row-major rows*(K/beta). */
void or_quantize_rows(const float* x, int64_t rows, int K, int fmt, float g,
                      uint8_t* codes, uint8_t* scales) {
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  int nb = K / beta;
  #pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    uint8_t c[32];
    for (int b = 0; b < nb; ++b) {
      const float* xb = x + r * K + (int64_t)b * beta;
      uint8_t sc = (fmt == OR_NVFP4) ? or_quant_block_nvfp4(xb, beta, g, c)
                                     : or_quant_block_mxfp4(xb, beta, c);
      scales[r * nb + b] = sc;
      for (int i = 0; i < beta; i += 2)
        codes[r * (K / 2) + (b * beta + i) / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
    }
  }
}

double or_dequant(uint8_t code, uint8_t sc, int fmt, float g) {
  return (fmt == OR_NVFP4) ? or_dequant_nvfp4(code, sc, g) : or_dequant_mxfp4(code, sc);
}

/* Byte offset of the scale of (row, k-block) in the tiled scale layout:
 * 128-row groups x 4-block groups form 512-byte chunks, chunks ordered by
 * row group then block group; inside a chunk, (row % 32) selects a 16-byte
 * line, (row % 128) / 32 a 4-byte word in it and (block % 4) the byte. */
int64_t or_sf_tiled_offset(int64_t row, int kb, int n_kchunks) {
  return ((row / 128) * n_kchunks + kb / 4) * 512 + (row % 32) * 16 +
         ((row % 128) / 32) * 4 + (kb % 4);
}

/* plain [rows][nb] -> tiled layout (rows padded to 128, blocks to 4). */
void or_sf_tile(const uint8_t* plain, int64_t rows, int nb, uint8_t* tiled,
                int64_t rows_padded) {
  int nkc = (nb + 3) / 4;
  memset(tiled, 0, (size_t)(rows_padded / 128) * nkc * 512);
  for (int64_t r = 0; r < rows; ++r)
    for (int b = 0; b < nb; ++b)
      tiled[or_sf_tiled_offset(r, b, nkc)] = plain[r * nb + b];
}

/* ------------------------------------------------------------------------ */
/* 3. Smooth-QK calibration and the fused scale + quantize                   */
/* ------------------------------------------------------------------------ */

/* [HiFA4, Abstract para 2]: a calibration-static per-channel equivalent
 * rescaling Q' = Q*s, K' = K/s after RoPE, computed once from a small
 * calibration set, moving quantization difficulty from K to Q.
 * Reading (formula not on the pages): per kv-head h and channel c,
 *   aK = max |K[b,h,t,c]|, aQ = max |Q[b,hq,t,c]| over b, the G query heads
 *   of group h and t < n_cal;  s = clamp(aK^alpha / aQ^(1-alpha), 2^-16, 2^16)
 *   in fp64, rounded to fp32; s = 1 when disabled or either amax is 0;
 *   inv_s = fl32(1/s).
 * q, k: [B][H][ld_tok][d] as float (exact copies of the bf16/fp16 inputs). */
static int or_cmp_double(const void* a, const void* b) {
  const double x = *(const double*)a, y = *(const double*)b;
  return (x > y) - (x < y);
}

void or_calibrate(const float* q, const float* k, int B, int Hq, int Hkv,
                  int n_cal, int ld_tok, int d, double alpha, int enable,
                  float* s, float* inv_s) {
  int G = Hq / Hkv;
  double* akv = (double*)malloc(sizeof(double) * d);
  double* sorted = (double*)malloc(sizeof(double) * d);
  for (int h = 0; h < Hkv; ++h) {
    /* applicability gate [reading of HiFA4, Abstract para 3, which names the
     * gate but not its rule]: enable == 2 turns smoothing on for head h only
     * if its largest channel amax of K exceeds 8 times the median over the d
     * channels (mean of the two middle order statistics). */
    int on = enable != 0;
    if (enable == 2) {
      double mx = 0.0;
      for (int c = 0; c < d; ++c) {
        double aK = 0.0;
        for (int b = 0; b < B; ++b)
          for (int t = 0; t < n_cal; ++t) {
            double vk = fabs((double)k[(((int64_t)b * Hkv + h) * ld_tok + t) * d + c]);
            if (vk > aK) aK = vk;
          }
        akv[c] = aK;
        sorted[c] = aK;
        if (aK > mx) mx = aK;
      }
      qsort(sorted, (size_t)d, sizeof(double), or_cmp_double);
      const double median = 0.5 * (sorted[d / 2 - 1] + sorted[d / 2]);
      on = mx > 8.0 * median;
    }
    for (int c = 0; c < d; ++c) {
      double aK = 0.0, aQ = 0.0;
      for (int b = 0; b < B; ++b) {
        for (int t = 0; t < n_cal; ++t) {
          double vk = fabs((double)k[(((int64_t)b * Hkv + h) * ld_tok + t) * d + c]);
          if (vk > aK) aK = vk;
          for (int gq = 0; gq < G; ++gq) {
            int hq = h * G + gq;
            double vq = fabs((double)q[(((int64_t)b * Hq + hq) * ld_tok + t) * d + c]);
            if (vq > aQ) aQ = vq;
          }
        }
      }
      float sv = 1.0f;
      if (on && aK > 0.0 && aQ > 0.0) {
        double v = pow(aK, alpha) / pow(aQ, 1.0 - alpha);
        if (v < ldexp(1.0, -16)) v = ldexp(1.0, -16);
        if (v > ldexp(1.0, 16)) v = ldexp(1.0, 16);
        sv = (float)v;
      }
      s[h * d + c] = sv;
      inv_s[h * d + c] = 1.0f / sv;
    }
  }
  free(akv);
  free(sorted);
}

/* Q-Mean auxiliary [a reading of HiFA4, Abstract para 3, which names "the
 * adopted Q-Mean auxiliary" and nothing more]: the per-channel mean of the
 * smoothed query over the calibration tokens,
 *   mu[hq][c] = fl32( sum_{b, t < n_cal} fl32(q * s[h(hq)][c]) / (B * n_cal) ),
 * the sum in fp64 in the order b, then t.  The quantized query is then
 * q' - mu (or_quantize_qkv), and each score gets back the rank-one term
 * mu . K-hat of its key (or_attention), so that without quantization the
 * scores are unchanged: (q' - mu) . k + mu . k = q' . k.
 * q [B][Hq][ld_tok][d]; s [Hkv][d] or NULL (= 1); mu out [Hq][d]. */
void or_calibrate_q_mean(const float* q, int B, int Hq, int Hkv, int n_cal,
                         int ld_tok, int d, const float* s, float* mu) {
  int G = Hq / Hkv;
  for (int hq = 0; hq < Hq; ++hq) {
    int h = hq / G;
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int b = 0; b < B; ++b)
        for (int t = 0; t < n_cal; ++t) {
          float x = q[(((int64_t)b * Hq + hq) * ld_tok + t) * d + c];
          float xs = s ? x * s[h * d + c] : x;
          acc += (double)xs;
        }
      mu[hq * d + c] = (float)(acc / (double)((int64_t)B * n_cal));
    }
  }
}

/* Fused scale + quantize of Q, K, V [HiFA4, Abstract para 2: "only a fusible
 * element-wise scaling"].  q' = fl32(q*s[c]), k' = fl32(k*inv_s[c]) on the
 * kv-head of the row, then blocks along d.  V is not scaled; it is blocked
 * along tokens and written transposed ([d][Np] codes, tokens contiguous).
 * Rows/tokens from N up to Np (N rounded up to 128) are zero padding.
 * s/inv_s may be NULL (treated as 1).  q_mu [Hq][d] (the Q-Mean auxiliary,
 * or NULL): rows t < N of Q quantize fl32(fl32(q*s) - mu) instead.
 * Outputs: q_codes [B][Hq][Np][d/2], q_sc plain [B][Hq][Np][d/beta];
 *          k likewise with Hkv; vt_codes [B][Hkv][d][Np/2],
 *          vt_sc plain [B][Hkv][d][Np/beta]. */
void or_quantize_qkv(const float* q, const float* k, const float* v, int B,
                     int Hq, int Hkv, int N, int d, const float* s,
                     const float* inv_s, int fmt, uint8_t* q_codes,
                     uint8_t* q_sc, uint8_t* k_codes, uint8_t* k_sc,
                     uint8_t* vt_codes, uint8_t* vt_sc, const float* q_mu) {
  int G = Hq / Hkv;
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  int64_t Np = ((int64_t)N + 127) / 128 * 128;
  int nb = d / beta;
  /* Q */
  for (int b = 0; b < B; ++b)
    for (int hq = 0; hq < Hq; ++hq) {
      int h = hq / G;
      float* buf = (float*)calloc((size_t)Np * d, sizeof(float));
      for (int t = 0; t < N; ++t)
        for (int c = 0; c < d; ++c) {
          float x = q[(((int64_t)b * Hq + hq) * N + t) * d + c];
          float xs = s ? x * s[h * d + c] : x;
          if (q_mu) xs = xs - q_mu[hq * d + c];
          buf[(int64_t)t * d + c] = xs;
        }
      int64_t base = ((int64_t)b * Hq + hq) * Np;
      or_quantize_rows(buf, Np, d, fmt, 1.0f, q_codes + base * (d / 2), q_sc + base * nb);
      free(buf);
    }
  /* K */
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      float* buf = (float*)calloc((size_t)Np * d, sizeof(float));
      for (int t = 0; t < N; ++t)
        for (int c = 0; c < d; ++c) {
          float x = k[(((int64_t)b * Hkv + h) * N + t) * d + c];
          buf[(int64_t)t * d + c] = inv_s ? x * inv_s[h * d + c] : x;
        }
      int64_t base = ((int64_t)b * Hkv + h) * Np;
      or_quantize_rows(buf, Np, d, fmt, 1.0f, k_codes + base * (d / 2), k_sc + base * nb);
      free(buf);
    }
  /* V, transposed: row = channel, K dimension = tokens */
  int nbt = (int)(Np / beta);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      float* buf = (float*)calloc((size_t)Np * d, sizeof(float));
      for (int t = 0; t < N; ++t)
        for (int c = 0; c < d; ++c)
          buf[(int64_t)c * Np + t] = v[(((int64_t)b * Hkv + h) * N + t) * d + c];
      int64_t base = ((int64_t)b * Hkv + h) * d;
      or_quantize_rows(buf, d, (int)Np, fmt, 1.0f, vt_codes + base * (Np / 2), vt_sc + base * nbt);
      free(buf);
    }
}

/* ------------------------------------------------------------------------ */
/* 4. Attention forward (prefill)                                            */
/* ------------------------------------------------------------------------ */

static inline uint8_t nib(const uint8_t* codes, int64_t i) {
  uint8_t byte = codes[i / 2];
  return (i % 2 == 0) ? (byte & 15) : (byte >> 4);
}

/* Softmax probability of one score, as the written specification fixes it:
 * P = fl32(2^(x - m)) computed in fp64, with results below 2^-126 set to 0. */
static double prob_of(double x, double m, int exact) {
  double p = exp2(x - m);
  if (exact) return p;
  float pf = (float)p;
  if (pf < 0x1p-126f) pf = 0.0f;
  return (double)pf;
}

/* Test knobs of the oracle (never used by the product):
 *   OR_VAR_NO_PQUANT  P-hat = P (the P quantizer replaced by the identity);
 *   OR_VAR_EXACT      scores and probabilities kept in fp64 (no fl32 steps).
 * With both set the recurrence is exact softmax attention in fp64. */
#define OR_VAR_NO_PQUANT 1
#define OR_VAR_EXACT 2

/* Process one key tile for one query row: the online-softmax update of
 * [HiFA4, Abstract para 1] with P-hat quantized per beta-block of the tile
 * [HiFA4, Abstract para 2].  x[k] holds fl32(S*c) for the tile's BN keys, with
 * masked keys marked by vis[k] = 0.  State: m, l_phat, l_p, acc[d].
 * vdq: dequantized V̂ of this kv head, [d][Np] (fp64), key offset k0.
 * tau: the running max moves to the tile's max x_t only when
 * x_t > fl32(m + tau) (fp32, as the kernels decide it; fp64 in the exact
 * variant); tau = 0 is the exact recurrence m' = max(m, x_t).  With a stale
 * m the probabilities P = 2^(x - m) may exceed 1.  (The lazy rescaling of
 * FlashAttention-4; the paper states the exact recurrence.) */
typedef struct {
  double m;        /* running max, in the log2 domain of scaled scores */
  double l_phat;   /* sum of P-hat under the same recurrence */
  double l_p;      /* sum of unquantized P under the same recurrence */
  double* acc;     /* [d] running P-hat . V-hat */
} or_row_state;

static void tile_update(or_row_state* st, const double* x, const int* vis, int BN,
                        int fmt, float gP, const double* vdq, int64_t Np,
                        int64_t k0, int d, int variant, float tau, uint8_t* phat_dump,
                        uint8_t* phat_sc_dump, double* tsum) {
  int exact = (variant & OR_VAR_EXACT) != 0;
  double mt = -INFINITY;
  for (int k = 0; k < BN; ++k)
    if (vis[k] && x[k] > mt) mt = x[k];
  double m_old = st->m;
  double thr = exact ? m_old + tau : (double)((float)m_old + tau);
  double m_new = (mt > thr) ? mt : m_old;
  double alpha = (m_old == -INFINITY) ? 0.0 : exp2(m_old - m_new);
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  double P[256], Phat[256];
  float P32[256];
  for (int k = 0; k < BN; ++k) {
    P[k] = vis[k] ? prob_of(x[k], m_new, exact) : 0.0;
    P32[k] = (float)P[k];
  }
  for (int b0 = 0; b0 < BN; b0 += beta) {
    uint8_t c[32];
    uint8_t sc = (fmt == OR_NVFP4) ? or_quant_block_nvfp4(P32 + b0, beta, gP, c)
                                   : or_quant_block_mxfp4(P32 + b0, beta, c);
    for (int i = 0; i < beta; ++i) {
      Phat[b0 + i] = (variant & OR_VAR_NO_PQUANT) ? P[b0 + i] : or_dequant(c[i], sc, fmt, gP);
      if (phat_dump) phat_dump[b0 + i] = c[i];
    }
    if (phat_sc_dump) phat_sc_dump[b0 / beta] = sc;
  }
  double sp = 0.0, sph = 0.0;
  for (int k = 0; k < BN; ++k) { sp += P[k]; sph += Phat[k]; }
  if (tsum) { tsum[0] = sph; tsum[1] = sp; }
  st->l_p = alpha * st->l_p + sp;
  st->l_phat = alpha * st->l_phat + sph;
  for (int c = 0; c < d; ++c) {
    double a = 0.0;
    for (int k = 0; k < BN; ++k)
      if (Phat[k] != 0.0) a += Phat[k] * vdq[(int64_t)c * Np + k0 + k];
    st->acc[c] = alpha * st->acc[c] + a;
  }
  st->m = m_new;
}

/* Dequantize the tiles of one head once, for clarity of the main loop.  All
 * scale arrays are plain row-major [rows][nb]. */
static void dequant_rows(const uint8_t* codes, const uint8_t* sc, int64_t rows,
                         int K, int fmt, double* out) {
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  int nb = K / beta;
  for (int64_t r = 0; r < rows; ++r)
    for (int i = 0; i < K; ++i)
      out[r * K + i] = or_dequant(nib(codes + r * (K / 2), i), sc[r * nb + i / beta], fmt, 1.0f);
}

/* The P-hat global prescale g_P: 2^pexp for NVFP4, unused for MXFP4. */
static float p_prescale(int fmt, int pexp) {
  return (fmt == OR_NVFP4) ? (float)ldexp(1.0, pexp) : 1.0f;
}

/* Attention forward over quantized inputs (layouts of or_quantize_qkv).
 * For each (b, hq, query row i) and key tiles j = 0, 1, ... of BN keys in
 * ascending order (causal: top-left aligned, key <= i), run tile_update;
 * then O = acc / l with l = l_phat under P-Reordering and l = l_p under the
 * inconsistent normalizer [HiFA4, Abstract para 2]; lse = m + log2(l).
 * Outputs (any may be NULL except O): O [B][Hq][N][d] fp64, lse [B][Hq][N],
 * l_phat / l_p [B][Hq][N], phat_dump [B][Hq][N][Nkt*BN] codes (1 per byte),
 * phat_sc_dump [B][Hq][N][Nkt*BN/beta], m_dump [B][Hq][N][Nkt] (running max
 * after each tile), tsum_dump [B][Hq][N][Nkt][2] (sum of P-hat and sum of P
 * over the tile's keys, both relative to that tile's running max: the
 * per-tile terms whose ratio minus one is the tile's normalizer error).
 * Test-only ablations: q_raw [B][Hq][N][d], k_raw [B][Hkv][N][d] and v_raw
 * [B][Hkv][N][d] (fp32, each may be NULL) replace the dequantized Q-hat,
 * K-hat or V-hat of the scores and the PV product by the given values.
 * q_mu [Hq][d] (the Q-Mean auxiliary of or_calibrate_q_mean, or NULL): every
 * score gets back mu . K-hat of its key, computed in fp64 from the
 * dequantized K-hat (or k_raw), before the scaling: x = fl32((q.k + mu.k) * c). */
void or_attention(const uint8_t* q_codes, const uint8_t* q_sc,
                  const uint8_t* k_codes, const uint8_t* k_sc,
                  const uint8_t* vt_codes, const uint8_t* vt_sc, int B, int Hq,
                  int Hkv, int N, int d, int fmt, double softmax_scale,
                  int causal, int mode, int BN, int pexp, double* O,
                  double* lse, double* l_phat_out, double* l_p_out,
                  uint8_t* phat_dump, uint8_t* phat_sc_dump, double* m_dump,
                  double* tsum_dump, const float* q_raw, const float* k_raw,
                  const float* v_raw, int row_begin, int row_end, int variant,
                  float tau, const float* q_mu) {
  int G = Hq / Hkv;
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  int64_t Np = ((int64_t)N + 127) / 128 * 128;
  int nb = d / beta;
  int ntiles = (N + BN - 1) / BN;
  float gP = p_prescale(fmt, pexp);
  double c_log2 = softmax_scale * 1.4426950408889634074;  /* log2(e) */
  if (row_end <= 0 || row_end > N) row_end = N;
  #pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int hq = 0; hq < Hq; ++hq) {
      int h = hq / G;
      double* qd = (double*)malloc(sizeof(double) * Np * d);
      double* kd = (double*)malloc(sizeof(double) * Np * d);
      double* vd = (double*)malloc(sizeof(double) * Np * d);
      int64_t qb = ((int64_t)b * Hq + hq) * Np, kb = ((int64_t)b * Hkv + h) * Np;
      int64_t vb = ((int64_t)b * Hkv + h) * d;
      dequant_rows(q_codes + qb * (d / 2), q_sc + qb * nb, Np, d, fmt, qd);
      dequant_rows(k_codes + kb * (d / 2), k_sc + kb * nb, Np, d, fmt, kd);
      dequant_rows(vt_codes + vb * (Np / 2), vt_sc + vb * (Np / beta), d, (int)Np, fmt, vd);
      if (q_raw || k_raw || v_raw) {
        int64_t qr = ((int64_t)b * Hq + hq) * N, kr = ((int64_t)b * Hkv + h) * N;
        for (int64_t t = 0; t < Np; ++t)
          for (int c = 0; c < d; ++c) {
            if (q_raw) qd[t * d + c] = t < N ? (double)q_raw[(qr + t) * d + c] : 0.0;
            if (k_raw) kd[t * d + c] = t < N ? (double)k_raw[(kr + t) * d + c] : 0.0;
            if (v_raw) vd[(int64_t)c * Np + t] = t < N ? (double)v_raw[(kr + t) * d + c] : 0.0;
          }
      }
      /* the Q-Mean term of every key: bias[key] = mu . k */
      double* bias = (double*)calloc((size_t)Np, sizeof(double));
      if (q_mu)
        for (int64_t key = 0; key < Np; ++key) {
          double sb = 0.0;
          for (int c = 0; c < d; ++c) sb += (double)q_mu[hq * d + c] * kd[key * d + c];
          bias[key] = sb;
        }
      double* acc = (double*)malloc(sizeof(double) * d);
      double* x = (double*)malloc(sizeof(double) * BN);
      int* vis = (int*)malloc(sizeof(int) * BN);
      for (int i = row_begin; i < row_end; ++i) {
        or_row_state st = {-INFINITY, 0.0, 0.0, acc};
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        int kv_end = causal ? i + 1 : N;
        int jt_end = (kv_end + BN - 1) / BN;
        int64_t row_id = ((int64_t)b * Hq + hq) * N + i;
        for (int j = 0; j < jt_end; ++j) {
          for (int kk = 0; kk < BN; ++kk) {
            int key = j * BN + kk;
            vis[kk] = key < kv_end;
            x[kk] = -INFINITY;
            if (vis[kk]) {
              double sdot = 0.0;
              for (int c = 0; c < d; ++c)
                sdot += qd[(int64_t)i * d + c] * kd[(int64_t)key * d + c];
              sdot += bias[key];
              x[kk] = (variant & OR_VAR_EXACT) ? sdot * c_log2 : (double)(float)(sdot * c_log2);
            }
          }
          uint8_t* pd = phat_dump ? phat_dump + row_id * (int64_t)ntiles * BN + (int64_t)j * BN : NULL;
          uint8_t* psd = phat_sc_dump ? phat_sc_dump + row_id * (int64_t)ntiles * (BN / beta) + (int64_t)j * (BN / beta) : NULL;
          double* ts = tsum_dump ? tsum_dump + (row_id * (int64_t)ntiles + j) * 2 : NULL;
          tile_update(&st, x, vis, BN, fmt, gP, vd, Np, (int64_t)j * BN, d, variant, tau, pd, psd, ts);
          if (m_dump) m_dump[row_id * (int64_t)ntiles + j] = st.m;
        }
        double l = (mode == OR_PREORDER) ? st.l_phat : st.l_p;
        for (int c = 0; c < d; ++c) O[row_id * d + c] = acc[c] / l;
        if (lse) lse[row_id] = st.m + log2(l);
        if (l_phat_out) l_phat_out[row_id] = st.l_phat;
        if (l_p_out) l_p_out[row_id] = st.l_p;
      }
      free(qd); free(kd); free(vd); free(bias); free(acc); free(x); free(vis);
    }
}

/* ------------------------------------------------------------------------ */
/* 5. Split-KV decode over a 4-bit KV cache                                  */
/* ------------------------------------------------------------------------ */

/* Length of one split: ceil(kv_len / num_splits) rounded up to BN. */
int or_split_len(int kv_len, int num_splits, int BN) {
  int L = (kv_len + num_splits - 1) / num_splits;
  return (L + BN - 1) / BN * BN;
}

/* One decode step.  q: [B][Hq][d] float (unscaled); the query is scaled by s
 * of its kv head and quantized in blocks along d exactly as or_quantize_qkv
 * quantizes Q.  The cache is in the layouts of or_quantize_qkv with N=kv_len.
 * Each split runs the prefill recurrence (non-causal) over its BN tiles;
 * partials (acc_s, m_s, l_s) merge in fp64:
 *   M = max m_s, O = sum 2^(m_s-M) acc_s / sum 2^(m_s-M) l_s,
 * with l_s = l_phat (P-Reordering) or l_p (inconsistent). */
void or_decode(const float* q, const float* s, const uint8_t* k_codes,
               const uint8_t* k_sc, const uint8_t* vt_codes,
               const uint8_t* vt_sc, int B, int Hq, int Hkv, int kv_len, int d,
               int fmt, double softmax_scale, int mode, int BN, int num_splits,
               int pexp, double* O, double* lse, int variant, float tau) {
  int G = Hq / Hkv;
  int beta = (fmt == OR_NVFP4) ? 16 : 32;
  int64_t Np = ((int64_t)kv_len + 127) / 128 * 128;
  int nb = d / beta;
  float gP = p_prescale(fmt, pexp);
  double c_log2 = softmax_scale * 1.4426950408889634074;
  int L = or_split_len(kv_len, num_splits, BN);
  #pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int hq = 0; hq < Hq; ++hq) {
      int h = hq / G;
      int64_t kb = ((int64_t)b * Hkv + h) * Np;
      int64_t vb = ((int64_t)b * Hkv + h) * d;
      double* kd = (double*)malloc(sizeof(double) * Np * d);
      double* vd = (double*)malloc(sizeof(double) * Np * d);
      dequant_rows(k_codes + kb * (d / 2), k_sc + kb * nb, Np, d, fmt, kd);
      dequant_rows(vt_codes + vb * (Np / 2), vt_sc + vb * (Np / beta), d, (int)Np, fmt, vd);
      /* quantize the query row: fl32(q*s) then blocks along d */
      float* qs = (float*)malloc(sizeof(float) * d);
      uint8_t* qc = (uint8_t*)malloc(d / 2);
      uint8_t* qsc = (uint8_t*)malloc(nb);
      double* qd = (double*)malloc(sizeof(double) * d);
      for (int c = 0; c < d; ++c) {
        float x = q[((int64_t)b * Hq + hq) * d + c];
        qs[c] = s ? x * s[h * d + c] : x;
      }
      or_quantize_rows(qs, 1, d, fmt, 1.0f, qc, qsc);
      dequant_rows(qc, qsc, 1, d, fmt, qd);
      double* acc = (double*)malloc(sizeof(double) * d);
      double* accsum = (double*)calloc(d, sizeof(double));
      double* x = (double*)malloc(sizeof(double) * BN);
      int* vis = (int*)malloc(sizeof(int) * BN);
      int nsplit_used = (kv_len + L - 1) / L;
      double* ms = (double*)malloc(sizeof(double) * nsplit_used);
      double* ls = (double*)malloc(sizeof(double) * nsplit_used);
      double* accs = (double*)malloc(sizeof(double) * nsplit_used * d);
      for (int sp = 0; sp < nsplit_used; ++sp) {
        int k_begin = sp * L, k_end = (sp + 1) * L < kv_len ? (sp + 1) * L : kv_len;
        or_row_state st = {-INFINITY, 0.0, 0.0, acc};
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (int j0 = k_begin; j0 < k_end; j0 += BN) {
          for (int kk = 0; kk < BN; ++kk) {
            int key = j0 + kk;
            vis[kk] = key < k_end;
            x[kk] = -INFINITY;
            if (vis[kk]) {
              double sdot = 0.0;
              for (int c = 0; c < d; ++c) sdot += qd[c] * kd[(int64_t)key * d + c];
              x[kk] = (variant & OR_VAR_EXACT) ? sdot * c_log2 : (double)(float)(sdot * c_log2);
            }
          }
          tile_update(&st, x, vis, BN, fmt, gP, vd, Np, j0, d, variant, tau, NULL, NULL, NULL);
        }
        ms[sp] = st.m;
        ls[sp] = (mode == OR_PREORDER) ? st.l_phat : st.l_p;
        for (int c = 0; c < d; ++c) accs[(int64_t)sp * d + c] = acc[c];
      }
      double M = -INFINITY;
      for (int sp = 0; sp < nsplit_used; ++sp) if (ms[sp] > M) M = ms[sp];
      double den = 0.0;
      for (int sp = 0; sp < nsplit_used; ++sp) {
        double w = exp2(ms[sp] - M);
        den += w * ls[sp];
        for (int c = 0; c < d; ++c) accsum[c] += w * accs[(int64_t)sp * d + c];
      }
      int64_t row_id = (int64_t)b * Hq + hq;
      for (int c = 0; c < d; ++c) O[row_id * d + c] = accsum[c] / den;
      if (lse) lse[row_id] = M + log2(den);
      free(kd); free(vd); free(qs); free(qc); free(qsc); free(qd); free(acc);
      free(accsum); free(x); free(vis); free(ms); free(ls); free(accs);
    }
}
