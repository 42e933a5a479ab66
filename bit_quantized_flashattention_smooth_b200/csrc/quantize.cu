// quantize.cu -- Smooth-QK calibration (amax reduction + scale formula) and
// the fused scale + block-quantize kernels for Q, K (blocks along d) and V
// (blocks along tokens, written channel-major).
//
// Method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for
// LLM Inference", Abstract para 2 (Smooth-QK is a calibration-static
// per-channel rescale applied as a fusible element-wise scaling).  Block
// rules: NVFP4 (UE4M3 scale per 16) and MXFP4 (OCP MX v1.0, UE8M0 per 32).
// All format decisions are made in IEEE fp32: scaled value fl32(x*s), block
// amax, fl32(amax/6), RNE to UE4M3, fl32(1/scale), fl32(x*inv), RNE to E2M1.
// These kernels are bound by HBM bandwidth: each input element is read once
// with 16-byte loads, each code / scale byte written once.
#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Quantize one block of BETA fp32 values in place into packed codes
// (BETA/2 bytes, element 2i in the low nibble) and return the scale code.
// inv_tab[c] = fl32(1 / UE4M3(c)) (0 for c = 0), in shared memory.
template <int FMT, int BETA>
__device__ __forceinline__ uint32_t quant_block(const float (&v)[BETA], uint32_t (&packed)[BETA / 8],
                                                const float* inv_tab) {
  float amax = fmaxf(fabsf(v[0]), fabsf(v[1]));
#pragma unroll
  for (int i = 2; i + 1 < BETA; i += 2) amax = fmax3(amax, fabsf(v[i]), fabsf(v[i + 1]));
  float mult;
  uint32_t sc;
  uint32_t keep = 0xFFFFFFFFu;
  if constexpr (FMT == HIFA4_NVFP4) {
    // fl32(amax/6): the reciprocal-and-residual form is IEEE-exact on
    // [2^-122, 2^20] (checked on the GPU); below, both give scale code 0
    const float t = amax <= 1048576.0f ? div6_rn(amax) : __fdiv_rn(amax, 6.0f);
    sc = cvt_e4m3(t);
    mult = inv_tab[sc];
    if (sc == 0) keep = 0u;                             // scale 0: every code 0 (no -0 codes)
  } else {
    const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
    sc = ef >= 2u ? ef - 2u : 0u;                       // E + 127, E = floor(log2 amax) - 2
    mult = __uint_as_float((254u - sc) << 23);          // 2^-E
  }
  const float2 m2 = make_float2(mult, mult);
#pragma unroll
  for (int w = 0; w < BETA / 8; ++w) {
    const float* e = v + 8 * w;
    packed[w] = keep & cvt_e2m1x8(fmul2(make_float2(e[0], e[1]), m2), fmul2(make_float2(e[2], e[3]), m2),
                                  fmul2(make_float2(e[4], e[5]), m2), fmul2(make_float2(e[6], e[7]), m2));
  }
  return sc;
}

// Rows of Q or K, one lane per block: D/BETA lanes cover a row, so each
// 16-byte load instruction of a warp touches a few whole 128-byte lines
// instead of one line per lane, and the code bytes of a row are written by
// consecutive lanes.  kLpbUnroll row groups per lane are loaded before any is
// quantized.  Rows are flattened (head, token); tokens N..Np-1 are zero
// padding; head bh uses smoothing row (bh % H) / G of `scale`.
template <int FMT>
struct LpbCfg {
  static constexpr int kUnroll = FMT == HIFA4_NVFP4 ? 2 : 1;
};

template <int FMT, int D>
struct RowTile {
  static constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  static constexpr int U = LpbCfg<FMT>::kUnroll;
  static constexpr int LPR = D / BETA;     // lanes (= blocks) per row
  static constexpr int RPW = 32 / LPR;     // rows per warp and row group
  static constexpr int ROWS = 8 * U * RPW; // rows per 256-thread CTA; divides 128
  static_assert(128 % ROWS == 0, "a CTA's rows stay inside one head");
};

// CTA `cta` of a tensor with `heads` heads of Np (padded) rows: head
// cta / (Np / ROWS), rows [chunk * ROWS, +ROWS).  Index arithmetic per CTA,
// none per lane beyond shifts.
template <int FMT, typename T, int D>
__device__ __forceinline__ void quantize_rows_lpb(const T* __restrict__ x, int H, int G, int N, int Np,
                                                  const float* __restrict__ scale, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, int64_t sf_head_bytes, int cta,
                                                  const float* inv_tab) {
  using R = RowTile<FMT, D>;
  constexpr int BETA = R::BETA, U = R::U, LPR = R::LPR, RPW = R::RPW;
  constexpr int WPR = (LPR + 3) / 4;       // scale words per row
  const int cpt = Np / R::ROWS;
  const int bh = cta / cpt;
  const int chunk = cta - bh * cpt;
  const int kvh = (bh % H) / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lb = lane % LPR;
  const T* xh = x + static_cast<int64_t>(bh) * N * D + lb * BETA;
  const float* srow = scale != nullptr ? scale + kvh * D + lb * BETA : nullptr;
  float v[U][BETA];
  int tok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    tok[u] = chunk * R::ROWS + (warp * U + u) * RPW + lane / LPR;
    if (tok[u] < N) {
      const T* src = xh + static_cast<int64_t>(tok[u]) * D;
#pragma unroll
      for (int i = 0; i < BETA / 8; ++i) {
        float f[8];
        load8<T>(src + 8 * i, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[u][8 * i + j] = f[j];
      }
    } else {
#pragma unroll
      for (int i = 0; i < BETA; ++i) v[u][i] = 0.0f;
    }
  }
  uint8_t* ch = codes + (static_cast<int64_t>(bh) * Np) * (D / 2) + lb * (BETA / 2);
  uint8_t* sh = sf + static_cast<int64_t>(bh) * sf_head_bytes;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int t = tok[u];
    if (srow != nullptr && t < N) {
      const float4* s4 = reinterpret_cast<const float4*>(srow);
#pragma unroll
      for (int i = 0; i < BETA / 4; ++i) {
        const float4 sv = s4[i];
        const float2 p0 = fmul2(make_float2(v[u][4 * i + 0], v[u][4 * i + 1]), make_float2(sv.x, sv.y));
        const float2 p1 = fmul2(make_float2(v[u][4 * i + 2], v[u][4 * i + 3]), make_float2(sv.z, sv.w));
        v[u][4 * i + 0] = p0.x;
        v[u][4 * i + 1] = p0.y;
        v[u][4 * i + 2] = p1.x;
        v[u][4 * i + 3] = p1.y;
      }
    }
    uint32_t packed[BETA / 8];
    const uint32_t sc = quant_block<FMT, BETA>(v[u], packed, inv_tab);
    uint8_t* dst = ch + static_cast<int64_t>(t) * (D / 2);
    if constexpr (BETA == 16) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    uint8_t* sfw = sh + sf_word_offset(t, lb / 4, WPR);
    sfw[lb % 4] = static_cast<uint8_t>(sc);
    if constexpr (LPR < 4) {
      // the rest of the row's only scale word holds no block: zero it
      if (lb == LPR - 1)
#pragma unroll
        for (int bb = LPR; bb < 4; ++bb) sfw[bb] = 0;   // lb / 4 == 0: the same word
    }
  }
}

// V: one CTA per (128-token tile, head, 64-channel group).  The tile is staged
// in shared memory with coalesced 16-byte loads; then one thread per (channel,
// scale word) quantizes 4 blocks of tokens and writes 4*BETA/2 contiguous code
// bytes of the channel-major V^T row plus one scale word.
constexpr int kVCh = 64;   // channels per V CTA
template <int FMT, typename T>
__device__ __forceinline__ void quantize_v_tile(const T* __restrict__ v, int N, int Np, int d,
                                                uint8_t* __restrict__ vt_codes, uint8_t* __restrict__ vt_sf,
                                                int64_t sf_head_bytes, int tile, T* tile_smem, const float* inv_tab) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  const int ncg = d / kVCh;
  const int cg = tile % ncg;
  const int64_t bhx = tile / ncg;          // head * (Np / 128) + token tile
  const int ntt = Np / 128;
  const int t0 = static_cast<int>(bhx % ntt) * 128;
  const int64_t head = bhx / ntt;
  const int c_base = cg * kVCh;
  constexpr int VEC = kVCh / 8;   // 16-byte vectors per token row
  for (int i = threadIdx.x; i < 128 * VEC; i += blockDim.x) {
    const int r = i / VEC, cv = i % VEC;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (t0 + r < N)
      u = *reinterpret_cast<const uint4*>(v + (head * N + t0 + r) * static_cast<int64_t>(d) + c_base + cv * 8);
    *reinterpret_cast<uint4*>(tile_smem + r * kVCh + cv * 8) = u;
  }
  __syncthreads();
  const int words_per_ch = 128 / (4 * BETA);
  const int nkc = Np / (4 * BETA);
  if (cg == 0 && d < 128) {
    // rows d..127 of the 128-row scale group are padding (d = 64): zero them
    for (int task = threadIdx.x; task < (128 - d) * words_per_ch; task += blockDim.x) {
      const int c = d + task % (128 - d), w = task / (128 - d);
      *reinterpret_cast<uint32_t*>(vt_sf + head * sf_head_bytes + sf_word_offset(c, t0 / (4 * BETA) + w, nkc)) = 0u;
    }
  }
  // one task per (channel, token block): all threads busy, codes and the
  // scale byte written per block
  for (int task = threadIdx.x; task < kVCh * (128 / BETA); task += blockDim.x) {
    const int cl = task % kVCh, blk = task / kVCh;
    const int c = c_base + cl;
    float val[BETA];
#pragma unroll
    for (int i = 0; i < BETA; ++i) {
      const int tt = blk * BETA + i;
      if constexpr (std::is_same<T, __nv_bfloat16>::value)
        val[i] = __bfloat162float(tile_smem[tt * kVCh + cl]);
      else
        val[i] = __half2float(tile_smem[tt * kVCh + cl]);
    }
    uint32_t packed[BETA / 8];
    const uint32_t sc = quant_block<FMT, BETA>(val, packed, inv_tab);
    uint8_t* dst = vt_codes + (head * d + c) * static_cast<int64_t>(Np / 2) + (t0 + blk * BETA) / 2;
    if constexpr (BETA == 16) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    const int gb = t0 / BETA + blk;                   // block index along the row
    vt_sf[head * sf_head_bytes + sf_word_offset(c, gb / 4, nkc) + (gb % 4)] = static_cast<uint8_t>(sc);
  }
}

// One launch for the whole step: CTAs [0, nv) quantize V tiles, the next nq
// Q rows, the rest K rows.
struct QuantArgs {
  const void *q, *k, *v;
  const float *s, *inv_s;
  uint8_t *qc, *qs, *kc, *ks, *vc, *vs;
  int B, Hq, Hkv, N, Np, d;
  int64_t sf_qk_head, sf_v_head, q_rows, k_rows;
  int nq_ctas, nk_ctas, nv_ctas;
};

template <int FMT, typename T, int D>
__global__ void __launch_bounds__(256, 4) quantize_qkv_kernel(const QuantArgs a) {
  __shared__ __align__(16) T tile_smem[128 * kVCh];
  __shared__ float inv_tab[128];
  if (FMT == HIFA4_NVFP4 && threadIdx.x < 128)
    inv_tab[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __fdiv_rn(1.0f, ue4m3_to_f32(threadIdx.x));
  __syncthreads();
  // V tiles first (the longest CTAs start early), then Q rows, then K rows
  const int bid = static_cast<int>(blockIdx.x) - a.nv_ctas;
  if (bid < 0) {
    quantize_v_tile<FMT, T>(static_cast<const T*>(a.v), a.N, a.Np, a.d, a.vc, a.vs, a.sf_v_head,
                            static_cast<int>(blockIdx.x), tile_smem, inv_tab);
  } else if (bid < a.nq_ctas) {
    quantize_rows_lpb<FMT, T, D>(static_cast<const T*>(a.q), a.Hq, a.Hq / a.Hkv, a.N, a.Np, a.s, a.qc, a.qs,
                                 a.sf_qk_head, bid, inv_tab);
  } else if (bid < a.nq_ctas + a.nk_ctas) {
    quantize_rows_lpb<FMT, T, D>(static_cast<const T*>(a.k), a.Hkv, 1, a.N, a.Np, a.inv_s, a.kc, a.ks,
                                 a.sf_qk_head, bid - a.nq_ctas, inv_tab);
  }
}

// ------------------------------------------------------------ calibration ---
// amax over (batch, tokens < n_cal) per (head, channel) into the fp32 bit
// patterns of out[kv head][d] (non-negative floats order like unsigned ints).
template <typename T>
__global__ void calib_amax_kernel(const T* __restrict__ x, int B, int H, int ld_tok, int n_cal, int d,
                                  int heads_per_group, int rows_per_cta, unsigned int* __restrict__ out) {
  const int h = blockIdx.y;
  const int kvh = h / heads_per_group;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
  const int64_t rows = static_cast<int64_t>(B) * n_cal;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float m = 0.0f;
    for (int64_t r = r0; r < min(rows, r0 + rows_per_cta); ++r) {
      const int b = static_cast<int>(r / n_cal), t = static_cast<int>(r % n_cal);
      float val;
      const T* p = x + ((static_cast<int64_t>(b) * H + h) * ld_tok + t) * d + c;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) val = __bfloat162float(*p);
      else val = __half2float(*p);
      m = fmaxf(m, fabsf(val));
    }
    atomicMax(out + static_cast<int64_t>(kvh) * d + c, __float_as_uint(m));
  }
}

// s = clamp(aK^alpha / aQ^(1-alpha), 2^-16, 2^16) in fp64 -> fp32, inv = 1/s.
// On entry s holds the bits of aQ and inv_s the bits of aK.  One CTA per kv
// head, one thread per channel.  enable: 0 = off (s = 1), 1 = on, 2 = the
// applicability gate: on for a head iff max_c aK > kGateTau * median_c aK
// (median of the d channels: the mean of the two middle order statistics),
// decided in fp64.
constexpr double kGateTau = 8.0;
__global__ void calib_finalize_kernel(float* s, float* inv_s, int d, double alpha, int enable) {
  __shared__ float ak_sh[256];
  __shared__ double mid[2];
  __shared__ int gate_on;
  const int h = blockIdx.x, c = threadIdx.x;
  const int i = h * d + c;
  const double aq = static_cast<double>(__uint_as_float(reinterpret_cast<unsigned int*>(s)[i]));
  const float akf = __uint_as_float(reinterpret_cast<unsigned int*>(inv_s)[i]);
  const double ak = static_cast<double>(akf);
  int on = enable != 0;
  if (enable == 2) {
    ak_sh[c] = akf;
    if (c == 0) gate_on = 0;
    __syncthreads();
    // rank of this channel (ties broken by index): the two middle ranks give the median
    int rank = 0;
    for (int c2 = 0; c2 < d; ++c2) {
      const float x = ak_sh[c2];
      rank += (x < akf || (x == akf && c2 < c)) ? 1 : 0;
    }
    if (rank == d / 2 - 1) mid[0] = ak;
    if (rank == d / 2) mid[1] = ak;
    __syncthreads();
    const double median = 0.5 * (mid[0] + mid[1]);
    if (ak > kGateTau * median) atomicOr(&gate_on, 1);   // some channel exceeds tau * median
    __syncthreads();
    on = gate_on;
  }
  float sv = 1.0f;
  if (on && ak > 0.0 && aq > 0.0) {
    double val = pow(ak, alpha) / pow(aq, 1.0 - alpha);
    val = fmin(fmax(val, 1.52587890625e-05), 65536.0);
    sv = static_cast<float>(val);
  }
  s[i] = sv;
  inv_s[i] = __fdiv_rn(1.0f, sv);
}

// ---------------------------------------------------------- host launchers ---
template <typename T, int D>
static void launch_quant_d(const QuantArgs& a, int fmt, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(a.nq_ctas + a.nk_ctas + a.nv_ctas);
  if (fmt == HIFA4_NVFP4) quantize_qkv_kernel<HIFA4_NVFP4, T, D><<<grid, 256, 0, st>>>(a);
  else quantize_qkv_kernel<HIFA4_MXFP4, T, D><<<grid, 256, 0, st>>>(a);
}
template <typename T>
static void launch_quant(const QuantArgs& a, int fmt, cudaStream_t st) {
  if (a.d == 64) launch_quant_d<T, 64>(a, fmt, st);
  else if (a.d == 128) launch_quant_d<T, 128>(a, fmt, st);
  else launch_quant_d<T, 256>(a, fmt, st);
}

// q == nullptr quantizes only K and V (a KV cache).
hifa4_status quantize_qkv_launch(const void* q, const void* k, const void* v, int dt, int B, int Hq, int Hkv, int N,
                                 int d, const float* s, const float* inv_s, int fmt, uint8_t* qc, uint8_t* qs,
                                 uint8_t* kc, uint8_t* ks, uint8_t* vc, uint8_t* vs, cudaStream_t st) {
  QuantArgs a;
  a.q = q; a.k = k; a.v = v; a.s = s; a.inv_s = inv_s;
  a.qc = qc; a.qs = qs; a.kc = kc; a.ks = ks; a.vc = vc; a.vs = vs;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.N = N; a.Np = static_cast<int>(pad128(N)); a.d = d;
  a.sf_qk_head = static_cast<int64_t>(hifa4_scale_bytes(N, d, static_cast<hifa4_format>(fmt)));
  a.sf_v_head = static_cast<int64_t>(hifa4_scale_bytes(d, a.Np, static_cast<hifa4_format>(fmt)));
  a.q_rows = q ? static_cast<int64_t>(B) * Hq * a.Np : 0;
  a.k_rows = static_cast<int64_t>(B) * Hkv * a.Np;
  // 8 warps per CTA, each kUnroll row groups of 32 / (d / BETA) rows
  const int lpr = d / beta_of(fmt);
  const int rows_per_cta = 8 * (32 / lpr) * (fmt == HIFA4_NVFP4 ? LpbCfg<HIFA4_NVFP4>::kUnroll
                                                                 : LpbCfg<HIFA4_MXFP4>::kUnroll);
  a.nq_ctas = static_cast<int>(a.q_rows / rows_per_cta);    // Np is a multiple of 128, rows_per_cta divides 128
  a.nk_ctas = static_cast<int>(a.k_rows / rows_per_cta);
  a.nv_ctas = (a.Np / 128) * (a.B * a.Hkv) * (a.d / kVCh);
  if (dt == HIFA4_BF16) launch_quant<__nv_bfloat16>(a, fmt, st);
  else launch_quant<__half>(a, fmt, st);
  return launch_status(q ? "quantize_qkv" : "quantize_kv");
}

template <typename T>
static void launch_calib_amax(const void* x, int B, int H, int ld_tok, int n_cal, int d, int hpg, unsigned int* out,
                              cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(B) * n_cal;
  const int rows_per_cta = 64;
  dim3 grid(static_cast<unsigned>((rows + rows_per_cta - 1) / rows_per_cta), H);
  calib_amax_kernel<T><<<grid, d, 0, st>>>(static_cast<const T*>(x), B, H, ld_tok, n_cal, d, hpg, rows_per_cta, out);
}

hifa4_status calibrate_launch(const void* q, const void* k, int dt, int B, int Hq, int Hkv, int n_cal, int ld_tok,
                              int d, float alpha, int enable, float* s_out, float* inv_s_out, cudaStream_t st) {
  const size_t bytes = static_cast<size_t>(Hkv) * d * sizeof(float);
  if (cudaMemsetAsync(s_out, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(inv_s_out, 0, bytes, st) != cudaSuccess)
    return launch_status("calibrate memset");
  unsigned int* aq = reinterpret_cast<unsigned int*>(s_out);
  unsigned int* ak = reinterpret_cast<unsigned int*>(inv_s_out);
  if (dt == HIFA4_BF16) {
    launch_calib_amax<__nv_bfloat16>(q, B, Hq, ld_tok, n_cal, d, Hq / Hkv, aq, st);
    launch_calib_amax<__nv_bfloat16>(k, B, Hkv, ld_tok, n_cal, d, 1, ak, st);
  } else {
    launch_calib_amax<__half>(q, B, Hq, ld_tok, n_cal, d, Hq / Hkv, aq, st);
    launch_calib_amax<__half>(k, B, Hkv, ld_tok, n_cal, d, 1, ak, st);
  }
  calib_finalize_kernel<<<Hkv, d, 0, st>>>(s_out, inv_s_out, d, static_cast<double>(alpha), enable);
  return launch_status("calibrate_smooth_qk");
}

}  // namespace hifa4
