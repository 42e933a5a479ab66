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
#include "quant_rules.cuh"

namespace hifa4 {

// Rows of Q or K with every load coalesced: lane l of a warp reads the l-th
// 16-byte chunk (8 values) of the warp's 512 contiguous input bytes (32 / (d/8)
// whole rows), so one load instruction covers four whole 128-byte lines.  The
// BETA/8 lanes that share a block combine their maxima by shuffles and each
// writes its own 4 code bytes (the warp's code writes are one contiguous
// 128-byte line); the first lane of a block writes the scale byte.  U row
// groups per lane are loaded before any is quantized.  Rows are flattened
// (head, token); tokens N..Np-1 are zero padding; head bh uses smoothing row
// (bh % H) / G of `scale`.
template <int FMT, int D>
struct RowTile {
  static constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  static constexpr int U = 4;              // row groups per lane
  static constexpr int CPR = D / 8;        // 16-byte chunks per row
  static constexpr int RPI = 32 / CPR;     // rows per warp and row group
  static constexpr int LPB = BETA / 8;     // lanes per block
  static constexpr int NB = D / BETA;      // blocks per row
  static constexpr int ROWS = 8 * U * RPI; // rows per 256-thread CTA; divides 128
  static_assert(128 % ROWS == 0, "a CTA's rows stay inside one head");
};

// One lane's 8 values of a BETA-block spread over LPB = BETA/8 adjacent lanes:
// the block's scale code (the same in every lane of the block) and this lane's
// 8 E2M1 codes packed in a word, by exactly the rules of quant_block.
template <int FMT, int BETA>
__device__ __forceinline__ uint32_t quant_part(const float (&v)[8], uint32_t& packed, const float* inv_tab) {
  float amax = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])), fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])),
                     fmaxf(fabsf(v[6]), fabsf(v[7])));
#pragma unroll
  for (int o = 1; o < BETA / 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float mult;
  uint32_t sc;
  uint32_t keep = 0xFFFFFFFFu;
  if constexpr (FMT == HIFA4_NVFP4) {
    const float t = amax <= 1048576.0f ? div6_rn(amax) : __fdiv_rn(amax, 6.0f);
    sc = cvt_e4m3(t);
    mult = inv_tab[sc];
    if (sc == 0) keep = 0u;
  } else {
    const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
    sc = ef >= 2u ? ef - 2u : 0u;
    mult = __uint_as_float((254u - sc) << 23);
  }
  const float2 m2 = make_float2(mult, mult);
  packed = keep & cvt_e2m1x8(qmul2(make_float2(v[0], v[1]), m2), qmul2(make_float2(v[2], v[3]), m2),
                             qmul2(make_float2(v[4], v[5]), m2), qmul2(make_float2(v[6], v[7]), m2));
  return sc;
}

// CTA `cta` of a tensor with `heads` heads of Np (padded) rows: head
// cta / (Np / ROWS), rows [chunk * ROWS, +ROWS).  Index arithmetic per CTA,
// none per lane beyond shifts.
template <int FMT, typename T, int D>
__device__ __forceinline__ void quantize_rows_lpb(const T* __restrict__ x, int H, int G, int N, int Np,
                                                  const float* __restrict__ scale, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, int64_t sf_head_bytes, int cta,
                                                  const float* inv_tab) {
  using R = RowTile<FMT, D>;
  constexpr int BETA = R::BETA, U = R::U, CPR = R::CPR, RPI = R::RPI, LPB = R::LPB, NB = R::NB;
  constexpr int WPR = (NB + 3) / 4;        // scale words per row
  const int cpt = Np / R::ROWS;
  const int bh = cta / cpt;
  const int chunk = cta - bh * cpt;
  const int kvh = (bh % H) / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ch = lane % CPR;               // 16-byte chunk of the row
  const int blk = ch / LPB;                // its block
  const T* xh = x + static_cast<int64_t>(bh) * N * D + ch * 8;
  float v[U][8];
  int tok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    tok[u] = chunk * R::ROWS + (warp * U + u) * RPI + lane / CPR;
    if (tok[u] < N) {
      load8<T>(xh + static_cast<int64_t>(tok[u]) * D, v[u]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[u][i] = 0.0f;
    }
  }
  float sv[8];
  if (scale != nullptr) {
    const float4* s4 = reinterpret_cast<const float4*>(scale + kvh * D + ch * 8);
    const float4 a = s4[0], b = s4[1];
    sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w; sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
  }
  uint8_t* cbase = codes + (static_cast<int64_t>(bh) * Np) * (D / 2) + ch * 4;
  uint8_t* sh = sf + static_cast<int64_t>(bh) * sf_head_bytes;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int t = tok[u];
    if (scale != nullptr && t < N) {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 p2 = qmul2(make_float2(v[u][i], v[u][i + 1]), make_float2(sv[i], sv[i + 1]));
        v[u][i] = p2.x;
        v[u][i + 1] = p2.y;
      }
    }
    uint32_t packed;
    const uint32_t sc = quant_part<FMT, BETA>(v[u], packed, inv_tab);
    *reinterpret_cast<uint32_t*>(cbase + static_cast<int64_t>(t) * (D / 2)) = packed;
    if (ch % LPB == 0) {
      uint8_t* sfw = sh + sf_word_offset(t, blk / 4, WPR);
      sfw[blk % 4] = static_cast<uint8_t>(sc);
      if constexpr (NB < 4) {
        // the rest of the row's only scale word holds no block: zero it
        if (blk == NB - 1)
#pragma unroll
          for (int bb = NB; bb < 4; ++bb) sfw[bb] = 0;   // blk / 4 == 0: the same word
      }
    }
  }
}

// V: one CTA per (128-token tile, head, 64-channel group).  The tile is staged
// in shared memory with coalesced 16-byte loads; then one thread per (channel,
// token block) quantizes the block (the 32 lanes of a warp read 32 adjacent
// channels of a token: one shared-memory wavefront) and writes the scale
// byte, and the codes go through a second staging buffer so that each
// channel-major V^T row's 64 code bytes of the tile are written by 16-byte
// stores of consecutive threads.
constexpr int kVCh = 64;   // channels per V CTA
template <int FMT, typename T>
__device__ __forceinline__ void quantize_v_tile(const T* __restrict__ v, int N, int Np, int d,
                                                uint8_t* __restrict__ vt_codes, uint8_t* __restrict__ vt_sf,
                                                int64_t sf_head_bytes, int tile, T* tile_smem,
                                                unsigned char* code_stage, const float* inv_tab) {
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
    // codes staged per channel row (64 bytes = 128 tokens), pieces swizzled
    // by the channel so that the 32 channels of a warp spread over the banks
    unsigned char* srow = code_stage + cl * 64;
    if constexpr (BETA == 16)
      *reinterpret_cast<uint2*>(srow + ((blk ^ (cl & 7)) * 8)) = make_uint2(packed[0], packed[1]);
    else
      *reinterpret_cast<uint4*>(srow + ((blk ^ (cl & 3)) * 16)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    const int gb = t0 / BETA + blk;                   // block index along the row
    vt_sf[head * sf_head_bytes + sf_word_offset(c, gb / 4, nkc) + (gb % 4)] = static_cast<uint8_t>(sc);
  }
  __syncthreads();
  // each V^T row's 64 code bytes of this tile leave as four 16-byte stores
  for (int i = threadIdx.x; i < kVCh * 4; i += blockDim.x) {
    const int cl = i / 4, q = i % 4;
    const unsigned char* srow = code_stage + cl * 64;
    uint4 u;
    if constexpr (BETA == 16) {
      const uint2 lo = *reinterpret_cast<const uint2*>(srow + (((2 * q) ^ (cl & 7)) * 8));
      const uint2 hi = *reinterpret_cast<const uint2*>(srow + (((2 * q + 1) ^ (cl & 7)) * 8));
      u = make_uint4(lo.x, lo.y, hi.x, hi.y);
    } else {
      u = *reinterpret_cast<const uint4*>(srow + ((q ^ (cl & 3)) * 16));
    }
    *reinterpret_cast<uint4*>(vt_codes + (head * d + c_base + cl) * static_cast<int64_t>(Np / 2) + t0 / 2 + q * 16) = u;
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
  __shared__ __align__(16) unsigned char code_stage[kVCh * 64];
  __shared__ float inv_tab[128];
  if (FMT == HIFA4_NVFP4 && threadIdx.x < 128)
    inv_tab[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __fdiv_rn(1.0f, ue4m3_to_f32(threadIdx.x));
  __syncthreads();
  // V tiles first (the longest CTAs start early), then Q rows, then K rows
  const int bid = static_cast<int>(blockIdx.x) - a.nv_ctas;
  if (bid < 0) {
    quantize_v_tile<FMT, T>(static_cast<const T*>(a.v), a.N, a.Np, a.d, a.vc, a.vs, a.sf_v_head,
                            static_cast<int>(blockIdx.x), tile_smem, code_stage, inv_tab);
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
  // 8 warps per CTA, each RowTile::U row groups of 32 / (d / 8) rows
  const int rows_per_cta = d == 64 ? RowTile<HIFA4_NVFP4, 64>::ROWS
                                   : (d == 128 ? RowTile<HIFA4_NVFP4, 128>::ROWS : RowTile<HIFA4_NVFP4, 256>::ROWS);
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
