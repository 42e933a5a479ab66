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
template <int FMT, int BETA>
__device__ __forceinline__ uint32_t quant_block(const float (&v)[BETA], uint32_t (&packed)[BETA / 8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < BETA; ++i) amax = fmaxf(amax, fabsf(v[i]));
  float mult;
  uint32_t sc;
  if constexpr (FMT == HIFA4_NVFP4) {
    float t = __fdiv_rn(amax, 6.0f);
    sc = cvt_e4m3(t);
    float sd = ue4m3_to_f32(sc);
    mult = (sc == 0) ? 0.0f : __fdiv_rn(1.0f, sd);
  } else {
    uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
    sc = ef >= 2u ? ef - 2u : 0u;                       // E + 127, E = floor(log2 amax) - 2
    mult = __uint_as_float((254u - sc) << 23);          // 2^-E
  }
#pragma unroll
  for (int w = 0; w < BETA / 8; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float lo = __fmul_rn(v[8 * w + 2 * j], mult);
      float hi = __fmul_rn(v[8 * w + 2 * j + 1], mult);
      uint32_t byte = cvt_e2m1x2(hi, lo);
      if (FMT == HIFA4_NVFP4 && sc == 0) byte = 0;
      word |= byte << (8 * j);
    }
    packed[w] = word;
  }
  return sc;
}

// One thread per (row, scale word): a word covers up to 4 consecutive blocks
// of a row.  x: [BH][N][d] rows of head bh; rows N..Np-1 are zero padding.
// Head bh uses smoothing scale row (bh % H) / G of `scale` ([Hkv][d]).
template <int FMT, typename T>
__device__ __forceinline__ void quantize_row_word(const T* __restrict__ x, int H, int G, int N, int Np, int d,
                                                  const float* __restrict__ scale, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, int64_t sf_head_bytes, int64_t idx) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  const int nb = d / BETA;
  const int wpr = (nb + 3) / 4;
  const int w = static_cast<int>(idx % wpr);
  const int64_t rowg = idx / wpr;
  const int t = static_cast<int>(rowg % Np);
  const int64_t bh = rowg / Np;
  const int kvh = static_cast<int>(bh % H) / G;
  const int nbw = min(4, nb - 4 * w);
  uint32_t sc_word = 0;
  for (int blk = 0; blk < nbw; ++blk) {
    const int c0 = (4 * w + blk) * BETA;
    float v[BETA];
    if (t < N) {
      const T* src = x + (bh * N + t) * static_cast<int64_t>(d) + c0;
#pragma unroll
      for (int i = 0; i < BETA / 8; ++i) {
        float f[8];
        load8<T>(src + 8 * i, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * i + j] = f[j];
      }
      if (scale != nullptr) {
        const float4* s4 = reinterpret_cast<const float4*>(scale + static_cast<int64_t>(kvh) * d + c0);
#pragma unroll
        for (int i = 0; i < BETA / 4; ++i) {
          float4 s = s4[i];
          v[4 * i + 0] = __fmul_rn(v[4 * i + 0], s.x);
          v[4 * i + 1] = __fmul_rn(v[4 * i + 1], s.y);
          v[4 * i + 2] = __fmul_rn(v[4 * i + 2], s.z);
          v[4 * i + 3] = __fmul_rn(v[4 * i + 3], s.w);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < BETA; ++i) v[i] = 0.0f;
    }
    uint32_t packed[BETA / 8];
    uint32_t sc = quant_block<FMT, BETA>(v, packed);
    uint8_t* dst = codes + (bh * Np + t) * static_cast<int64_t>(d / 2) + c0 / 2;
    if constexpr (BETA == 16) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    sc_word |= sc << (8 * blk);
  }
  *reinterpret_cast<uint32_t*>(sf + bh * sf_head_bytes + sf_word_offset(t, w, wpr)) = sc_word;
}

// V: one CTA per (128-token tile, head, 64-channel group).  The tile is staged
// in shared memory with coalesced 16-byte loads; then one thread per (channel,
// scale word) quantizes 4 blocks of tokens and writes 4*BETA/2 contiguous code
// bytes of the channel-major V^T row plus one scale word.
constexpr int kVCh = 64;   // channels per V CTA
template <int FMT, typename T>
__device__ __forceinline__ void quantize_v_tile(const T* __restrict__ v, int N, int Np, int d,
                                                uint8_t* __restrict__ vt_codes, uint8_t* __restrict__ vt_sf,
                                                int64_t sf_head_bytes, int tile, T* tile_smem) {
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
  for (int task = threadIdx.x; task < kVCh * words_per_ch; task += blockDim.x) {
    const int cl = task % kVCh, w = task / kVCh;
    const int c = c_base + cl;
    uint32_t sc_word = 0;
    uint32_t out[4 * BETA / 8];
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      float val[BETA];
#pragma unroll
      for (int i = 0; i < BETA; ++i) {
        const int tt = w * 4 * BETA + blk * BETA + i;
        if constexpr (std::is_same<T, __nv_bfloat16>::value)
          val[i] = __bfloat162float(tile_smem[tt * kVCh + cl]);
        else
          val[i] = __half2float(tile_smem[tt * kVCh + cl]);
      }
      uint32_t packed[BETA / 8];
      const uint32_t sc = quant_block<FMT, BETA>(val, packed);
#pragma unroll
      for (int j = 0; j < BETA / 8; ++j) out[blk * (BETA / 8) + j] = packed[j];
      sc_word |= sc << (8 * blk);
    }
    uint8_t* dst = vt_codes + (head * d + c) * static_cast<int64_t>(Np / 2) + (t0 + w * 4 * BETA) / 2;
#pragma unroll
    for (int j = 0; j < 4 * BETA / 8; j += 4)
      *reinterpret_cast<uint4*>(dst + 4 * j) = make_uint4(out[j], out[j + 1], out[j + 2], out[j + 3]);
    *reinterpret_cast<uint32_t*>(vt_sf + head * sf_head_bytes + sf_word_offset(c, t0 / (4 * BETA) + w, nkc)) =
        sc_word;
  }
}

// One launch for the whole step: CTAs [0, nq) quantize Q rows, [nq, nq+nk)
// K rows, the rest V tiles.
struct QuantArgs {
  const void *q, *k, *v;
  const float *s, *inv_s;
  uint8_t *qc, *qs, *kc, *ks, *vc, *vs;
  int B, Hq, Hkv, N, Np, d;
  int64_t sf_qk_head, sf_v_head, q_words, k_words;
  int nq_ctas, nk_ctas;
};

template <int FMT, typename T>
__global__ void __launch_bounds__(256) quantize_qkv_kernel(const QuantArgs a) {
  __shared__ __align__(16) T tile_smem[128 * kVCh];
  const int bid = blockIdx.x;
  if (bid < a.nq_ctas) {
    const int64_t idx = static_cast<int64_t>(bid) * blockDim.x + threadIdx.x;
    if (idx < a.q_words)
      quantize_row_word<FMT, T>(static_cast<const T*>(a.q), a.Hq, a.Hq / a.Hkv, a.N, a.Np, a.d, a.s, a.qc, a.qs,
                                a.sf_qk_head, idx);
  } else if (bid < a.nq_ctas + a.nk_ctas) {
    const int64_t idx = static_cast<int64_t>(bid - a.nq_ctas) * blockDim.x + threadIdx.x;
    if (idx < a.k_words)
      quantize_row_word<FMT, T>(static_cast<const T*>(a.k), a.Hkv, 1, a.N, a.Np, a.d, a.inv_s, a.kc, a.ks,
                                a.sf_qk_head, idx);
  } else {
    quantize_v_tile<FMT, T>(static_cast<const T*>(a.v), a.N, a.Np, a.d, a.vc, a.vs, a.sf_v_head,
                            bid - a.nq_ctas - a.nk_ctas, tile_smem);
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
// On entry s holds the bits of aQ and inv_s the bits of aK.
__global__ void calib_finalize_kernel(float* s, float* inv_s, int n, double alpha, int enable) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  double aq = static_cast<double>(__uint_as_float(reinterpret_cast<unsigned int*>(s)[i]));
  double ak = static_cast<double>(__uint_as_float(reinterpret_cast<unsigned int*>(inv_s)[i]));
  float sv = 1.0f;
  if (enable && ak > 0.0 && aq > 0.0) {
    double val = pow(ak, alpha) / pow(aq, 1.0 - alpha);
    val = fmin(fmax(val, 1.52587890625e-05), 65536.0);
    sv = static_cast<float>(val);
  }
  s[i] = sv;
  inv_s[i] = __fdiv_rn(1.0f, sv);
}

// ---------------------------------------------------------- host launchers ---
template <typename T>
static void launch_quant(const QuantArgs& a, int fmt, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(a.nq_ctas + a.nk_ctas + (a.Np / 128) * (a.B * a.Hkv) * (a.d / kVCh));
  if (fmt == HIFA4_NVFP4) quantize_qkv_kernel<HIFA4_NVFP4, T><<<grid, 256, 0, st>>>(a);
  else quantize_qkv_kernel<HIFA4_MXFP4, T><<<grid, 256, 0, st>>>(a);
}

// q == nullptr quantizes only K and V (a KV cache).
hifa4_status quantize_qkv_launch(const void* q, const void* k, const void* v, int dt, int B, int Hq, int Hkv, int N,
                                 int d, const float* s, const float* inv_s, int fmt, uint8_t* qc, uint8_t* qs,
                                 uint8_t* kc, uint8_t* ks, uint8_t* vc, uint8_t* vs, cudaStream_t st) {
  QuantArgs a;
  a.q = q; a.k = k; a.v = v; a.s = s; a.inv_s = inv_s;
  a.qc = qc; a.qs = qs; a.kc = kc; a.ks = ks; a.vc = vc; a.vs = vs;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.N = N; a.Np = static_cast<int>(pad128(N)); a.d = d;
  const int wpr = (d / beta_of(fmt) + 3) / 4;
  a.sf_qk_head = static_cast<int64_t>(hifa4_scale_bytes(N, d, static_cast<hifa4_format>(fmt)));
  a.sf_v_head = static_cast<int64_t>(hifa4_scale_bytes(d, a.Np, static_cast<hifa4_format>(fmt)));
  a.q_words = q ? static_cast<int64_t>(B) * Hq * a.Np * wpr : 0;
  a.k_words = static_cast<int64_t>(B) * Hkv * a.Np * wpr;
  a.nq_ctas = static_cast<int>((a.q_words + 255) / 256);
  a.nk_ctas = static_cast<int>((a.k_words + 255) / 256);
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
  const int n = Hkv * d;
  calib_finalize_kernel<<<(n + 255) / 256, 256, 0, st>>>(s_out, inv_s_out, n, static_cast<double>(alpha), enable);
  return launch_status("calibrate_smooth_qk");
}

}  // namespace hifa4
