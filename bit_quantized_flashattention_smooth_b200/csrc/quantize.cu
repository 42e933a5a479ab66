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

// Element ch (0: low half, 1: high half) of a packed pair of 16-bit floats,
// exactly in fp32.
template <typename T>
__device__ __forceinline__ float chan_of(uint32_t w, int ch);
template <>
__device__ __forceinline__ float chan_of<__nv_bfloat16>(uint32_t w, int ch) {
  return __uint_as_float(ch == 0 ? (w << 16) : (w & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ float chan_of<__half>(uint32_t w, int ch) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(ch == 0 ? (w & 0xFFFFu) : (w >> 16))));
}
// One lane's 8 values of a BETA-block spread over LPB = BETA/8 adjacent lanes:
// the block's scale code (the same in every lane of the block) and this lane's
// 8 E2M1 codes packed in a word, by exactly the rules of quant_block.
template <int FMT, int BETA>
__device__ __forceinline__ uint32_t quant_part(const float (&v)[8], uint32_t& packed, const float* inv_tab) {
  // two-input maxima with |x| as operand modifiers (measured faster here than
  // the three-input form)
  float amax = fmaxf(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))),
                     fmaxf(fmaxf(fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7]))));
#pragma unroll
  for (int o = 1; o < BETA / 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float mult;
  uint32_t keep;
  const uint32_t sc = block_scale<FMT>(amax, inv_tab, mult, keep);
  const float2 m2 = make_float2(mult, mult);
  packed = keep & cvt_e2m1x8(qmul2(make_float2(v[0], v[1]), m2), qmul2(make_float2(v[2], v[3]), m2),
                             qmul2(make_float2(v[4], v[5]), m2), qmul2(make_float2(v[6], v[7]), m2));
  return sc;
}

// CTA `cta` of a tensor with `heads` heads of Np (padded) rows: head
// cta / (Np / ROWS), rows [chunk * ROWS, +ROWS).  A lane's U row groups are
// RPI rows apart and all fall inside one 32-row band of one 128-row scale
// group (a warp's U * RPI rows start on a multiple of U * RPI, which divides
// 32, and a CTA's rows on a multiple of ROWS), so every per-group address is
// the lane's first one plus a constant: the scale byte moves by RPI * 16
// bytes per group, the codes by RPI * D/2, the input by RPI * D values.
template <int FMT, typename T, int D, bool QM>
__device__ __forceinline__ void quantize_rows_lpb(const T* __restrict__ x, int H, int G, int N, int Np,
                                                  const float* __restrict__ scale, const float* __restrict__ mu,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                  int64_t sf_head_bytes, int cta, const float* inv_tab) {
  using R = RowTile<FMT, D>;
  constexpr int BETA = R::BETA, U = R::U, CPR = R::CPR, RPI = R::RPI, LPB = R::LPB, NB = R::NB;
  constexpr int WPR = (NB + 3) / 4;        // scale words per row
  static_assert(32 % (U * RPI) == 0, "a warp's rows stay inside one 32-row band");
  const int cpt = Np / R::ROWS;
  const int bh = cta / cpt;
  const int chunk = cta - bh * cpt;
  const int kvh = (bh % H) / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ch = lane % CPR;               // 16-byte chunk of the row
  const int blk = ch / LPB;                // its block
  const int t0 = chunk * R::ROWS + warp * U * RPI + lane / CPR;   // the lane's first row
  const int nvalid = N - t0;               // groups u with u * RPI < nvalid hold real rows
  const T* src = x + (static_cast<int64_t>(bh) * N + t0) * D + ch * 8;
  // all U loads in flight at once, kept packed (4 registers each) until their
  // row group is quantized; rows past N are zeros
  uint4 raw[U];
  if (chunk * R::ROWS + R::ROWS <= N) {
    // every row of the CTA is real (all CTAs but the last of a head): plain
    // loads, no per-group selects
#pragma unroll
    for (int u = 0; u < U; ++u) raw[u] = *reinterpret_cast<const uint4*>(src + u * RPI * D);
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u)
      raw[u] = u * RPI < nvalid ? *reinterpret_cast<const uint4*>(src + u * RPI * D) : make_uint4(0u, 0u, 0u, 0u);
  }
  float sv[8];
  if (scale != nullptr) {
    const float4* s4 = reinterpret_cast<const float4*>(scale + kvh * D + ch * 8);
    const float4 a = s4[0], b = s4[1];
    sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w; sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
  }
  // Q-Mean auxiliary: the head's calibration mean of this lane's 8 channels,
  // subtracted after the smoothing multiply from real rows (re-read per row
  // group from L1 rather than held in registers across the loop)
  const float4* mu4 = QM ? reinterpret_cast<const float4*>(mu + static_cast<int64_t>(bh % H) * D + ch * 8) : nullptr;
  uint8_t* cdst = codes + (static_cast<int64_t>(bh) * Np + t0) * (D / 2) + ch * 4;
  uint8_t* sdst = sf + static_cast<int64_t>(bh) * sf_head_bytes + sf_word_offset(t0, blk / 4, WPR) + blk % 4;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float v[8];
    {
      const uint32_t wd[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = chan_of<T>(wd[i], 0);
        v[2 * i + 1] = chan_of<T>(wd[i], 1);
      }
    }
    if (scale != nullptr) {
      // padding rows are +0 and stay +0 (s is finite and positive)
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 p2 = qmul2(make_float2(v[i], v[i + 1]), make_float2(sv[i], sv[i + 1]));
        v[i] = p2.x;
        v[i + 1] = p2.y;
      }
    }
    if (QM && u * RPI < nvalid) {
      // x - mu = x + (-mu) exactly: one packed add per pair
      const float4 a = mu4[0], b = mu4[1];
      const float nmu[8] = {-a.x, -a.y, -a.z, -a.w, -b.x, -b.y, -b.z, -b.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 d2 = fadd2(make_float2(v[i], v[i + 1]), make_float2(nmu[i], nmu[i + 1]));
        v[i] = d2.x;
        v[i + 1] = d2.y;
      }
    }
    uint32_t packed;
    const uint32_t sc = quant_part<FMT, BETA>(v, packed, inv_tab);
    *reinterpret_cast<uint32_t*>(cdst + u * RPI * (D / 2)) = packed;
    if (ch % LPB == 0) {
      uint8_t* sb = sdst + u * RPI * 16;
      *sb = static_cast<uint8_t>(sc);
      if constexpr (NB < 4) {
        // the rest of the row's only scale word holds no block: zero it
        if (blk == NB - 1)
#pragma unroll
          for (int bb = NB; bb < 4; ++bb) sb[bb - blk] = 0;   // blk / 4 == 0: the same word
      }
    }
  }
}

// V: one warp per (head, 32-token chunk, 64-channel group), quantized along
// tokens in registers.  Lane l owns channels c = 64g + 2l and c + 1: for each
// of the chunk's 32 tokens it loads the two channels' values as one 32-bit
// word (the warp's 32 words of a token are one contiguous 128-byte line), then
// quantizes each channel's blocks of BETA tokens by the rules of quant_block
// and writes the channel's 16 code bytes of the chunk (one V^T row segment)
// and its block scale bytes directly.  Tokens N..Np-1 are zero padding.
constexpr int kVCh = 64;   // channels per V warp task
constexpr int kVTok = 32;  // tokens per V warp task
template <typename T>
__device__ __forceinline__ float2 unpack_pair(uint32_t w);
template <>
__device__ __forceinline__ float2 unpack_pair<__nv_bfloat16>(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}
template <>
__device__ __forceinline__ float2 unpack_pair<__half>(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
// Element-wise max of |x| over two packed 16-bit values: an exact selection,
// so the block amax of each channel can be taken before any conversion.
template <typename T>
__device__ __forceinline__ uint32_t absmax_pair(uint32_t a, uint32_t b);
template <>
__device__ __forceinline__ uint32_t absmax_pair<__nv_bfloat16>(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmax2(__habs2(*reinterpret_cast<const __nv_bfloat162*>(&a)),
                             __habs2(*reinterpret_cast<const __nv_bfloat162*>(&b)));
  return *reinterpret_cast<uint32_t*>(&r);
}
template <>
__device__ __forceinline__ uint32_t absmax_pair<__half>(uint32_t a, uint32_t b) {
  __half2 r = __hmax2(__habs2(*reinterpret_cast<const __half2*>(&a)), __habs2(*reinterpret_cast<const __half2*>(&b)));
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int FMT, typename T>
__device__ __forceinline__ void quantize_v_cols(const T* __restrict__ v, int N, int Np, int d,
                                                uint8_t* __restrict__ vt_codes, uint8_t* __restrict__ vt_sf,
                                                int64_t sf_head_bytes, int64_t task, const float* inv_tab) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  constexpr int NBLK = kVTok / BETA;             // blocks of the chunk per channel
  const int lane = threadIdx.x & 31;
  const int ncg = d / kVCh;
  const int nchunk = Np / kVTok;
  const int cg = static_cast<int>(task % ncg);
  const int64_t rest = task / ncg;
  const int t0 = static_cast<int>(rest % nchunk) * kVTok;
  const int64_t head = rest / nchunk;
  const int c = cg * kVCh + 2 * lane;
  const int nkc = Np / (4 * BETA);               // scale chunks per 128-row group of V^T
  uint32_t w[kVTok];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(v + (head * N + t0) * static_cast<int64_t>(d) + c);
  if (t0 + kVTok <= N) {
    // a chunk of real tokens (all but the last chunk of a head): plain loads
#pragma unroll
    for (int i = 0; i < kVTok; ++i) w[i] = src[static_cast<int64_t>(i) * (d / 2)];
  } else {
#pragma unroll
    for (int i = 0; i < kVTok; ++i) w[i] = (t0 + i < N) ? src[static_cast<int64_t>(i) * (d / 2)] : 0u;
  }
  uint32_t codes0[kVTok / 8], codes1[kVTok / 8];
  uint32_t scw0 = 0, scw1 = 0;
#pragma unroll
  for (int b = 0; b < NBLK; ++b) {
    // both channels' block amax at once (exact), then each channel's scale
    uint32_t am = absmax_pair<T>(w[b * BETA], w[b * BETA + 1]);
#pragma unroll
    for (int i = 2; i < BETA; ++i) am = absmax_pair<T>(am, w[b * BETA + i]);
    const float2 amf = unpack_pair<T>(am);
    float mult0, mult1;
    uint32_t keep0, keep1;
    scw0 |= block_scale<FMT>(amf.x, inv_tab, mult0, keep0) << (8 * b);
    scw1 |= block_scale<FMT>(amf.y, inv_tab, mult1, keep1) << (8 * b);
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      const float2 m2 = ch == 0 ? make_float2(mult0, mult0) : make_float2(mult1, mult1);
      const uint32_t keep = ch == 0 ? keep0 : keep1;
#pragma unroll
      for (int q = 0; q < BETA / 8; ++q) {
        const uint32_t* e = w + b * BETA + 8 * q;
        const uint32_t cw = keep & cvt_e2m1x8(qmul2(make_float2(chan_of<T>(e[0], ch), chan_of<T>(e[1], ch)), m2),
                                              qmul2(make_float2(chan_of<T>(e[2], ch), chan_of<T>(e[3], ch)), m2),
                                              qmul2(make_float2(chan_of<T>(e[4], ch), chan_of<T>(e[5], ch)), m2),
                                              qmul2(make_float2(chan_of<T>(e[6], ch), chan_of<T>(e[7], ch)), m2));
        if (ch == 0) codes0[b * (BETA / 8) + q] = cw;
        else codes1[b * (BETA / 8) + q] = cw;
      }
    }
  }
  const int gb = t0 / BETA;                      // the chunk's NBLK blocks: consecutive bytes of one word
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int cc = c + ch;
    const uint32_t* cw = ch == 0 ? codes0 : codes1;
    *reinterpret_cast<uint4*>(vt_codes + (head * d + cc) * static_cast<int64_t>(Np / 2) + t0 / 2) =
        make_uint4(cw[0], cw[1], cw[2], cw[3]);
    uint8_t* sfw = vt_sf + head * sf_head_bytes + sf_word_offset(cc, gb / 4, nkc) + (gb % 4);
    const uint32_t scw = ch == 0 ? scw0 : scw1;
    if constexpr (NBLK == 2) *reinterpret_cast<uint16_t*>(sfw) = static_cast<uint16_t>(scw);
    else *sfw = static_cast<uint8_t>(scw);
  }
  if (cg == 0 && d < 128) {
    // rows d..127 of the 128-row scale group are padding (d = 64): zero them
    for (int r = d + lane; r < 128; r += 32) {
      uint8_t* sfw = vt_sf + head * sf_head_bytes + sf_word_offset(r, gb / 4, nkc) + (gb % 4);
      if constexpr (NBLK == 2) *reinterpret_cast<uint16_t*>(sfw) = 0;
      else *sfw = 0;
    }
  }
}

// One launch for the whole step: CTAs [0, nv) quantize V (8 warp tasks each),
// the next nq Q rows, the rest K rows.
struct QuantArgs {
  const void *q, *k, *v;
  const float *s, *inv_s, *q_mu;
  uint8_t *qc, *qs, *kc, *ks, *vc, *vs;
  int B, Hq, Hkv, N, Np, d;
  int64_t sf_qk_head, sf_v_head, q_rows, k_rows, v_tasks;
  int nq_ctas, nk_ctas, nv_ctas;
};

// fl32(1 / UE4M3(c)) for c = 1..127 (0 for c = 0), the element multiplier of
// a block with scale code c: IEEE division evaluated by the compiler, the
// same correctly rounded quotient __fdiv_rn gives on the device, so the
// kernel only copies it into shared memory.
struct InvScaleTable {
  float v[128];
};
constexpr float ue4m3_value(int c) {
  // (1 + m/8) 2^(e-7) for e > 0, m 2^-9 for e = 0 (powers of two exact)
  const int e = (c >> 3) & 15, m = c & 7;
  float p = 1.0f;
  if (e == 0) {
    for (int i = 0; i < 9; ++i) p *= 0.5f;
    return static_cast<float>(m) * p;
  }
  for (int i = 0; i < 7 - e; ++i) p *= 0.5f;
  for (int i = 0; i < e - 7; ++i) p *= 2.0f;
  return (1.0f + static_cast<float>(m) / 8.0f) * p;
}
constexpr InvScaleTable make_inv_scale_table() {
  InvScaleTable t{};
  for (int c = 1; c < 128; ++c) t.v[c] = 1.0f / ue4m3_value(c);
  return t;
}
__device__ const InvScaleTable kInvScale = make_inv_scale_table();

// QM: the Q rows subtract the Q-Mean auxiliary (its own instantiation: the
// plain quantizer carries none of it).  Resident CTAs per SM: 4 for NVFP4
// (64 registers, no spills; 5 or 6 spill and run 9-35 % slower), 6 for MXFP4
// (its spills cost less than the extra warps gain: 6 % faster on the long
// context).
template <int FMT, typename T, int D, bool QM>
__global__ void __launch_bounds__(256, FMT == HIFA4_NVFP4 ? 4 : 6) quantize_qkv_kernel(const QuantArgs a) {
  __shared__ float inv_tab[128];
  if (FMT == HIFA4_NVFP4 && threadIdx.x < 128) inv_tab[threadIdx.x] = kInvScale.v[threadIdx.x];
  __syncthreads();
  // V tiles first (the longest CTAs start early), then Q rows, then K rows
  const int bid = static_cast<int>(blockIdx.x) - a.nv_ctas;
  if (bid < 0) {
    const int64_t task = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (task < a.v_tasks)
      quantize_v_cols<FMT, T>(static_cast<const T*>(a.v), a.N, a.Np, a.d, a.vc, a.vs, a.sf_v_head, task, inv_tab);
  } else if (bid < a.nq_ctas) {
    quantize_rows_lpb<FMT, T, D, QM>(static_cast<const T*>(a.q), a.Hq, a.Hq / a.Hkv, a.N, a.Np, a.s, a.q_mu, a.qc,
                                     a.qs, a.sf_qk_head, bid, inv_tab);
  } else if (bid < a.nq_ctas + a.nk_ctas) {
    quantize_rows_lpb<FMT, T, D, false>(static_cast<const T*>(a.k), a.Hkv, 1, a.N, a.Np, a.inv_s, nullptr, a.kc,
                                        a.ks, a.sf_qk_head, bid - a.nq_ctas, inv_tab);
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

// Q-Mean auxiliary (a reading: the pages name "the adopted Q-Mean auxiliary"
// and nothing more): mu[hq][c] = fl32(sum_{b, t < n_cal} fl32(q * s[h][c]) /
// (B * n_cal)), the sum in fp64 in the order b, then t -- one thread per
// (q head, channel), so the result is reproducible bit for bit.
template <typename T>
__global__ void calib_q_mean_kernel(const T* __restrict__ q, int B, int Hq, int G, int ld_tok, int n_cal, int d,
                                    const float* __restrict__ s, float* __restrict__ mu) {
  const int hq = blockIdx.x, c = threadIdx.x;
  if (c >= d) return;
  const float sc = s != nullptr ? s[(hq / G) * d + c] : 1.0f;
  double acc = 0.0;
  for (int b = 0; b < B; ++b) {
    const T* p = q + ((static_cast<int64_t>(b) * Hq + hq) * ld_tok) * d + c;
    for (int t = 0; t < n_cal; ++t) {
      float x;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) x = __bfloat162float(p[static_cast<int64_t>(t) * d]);
      else x = __half2float(p[static_cast<int64_t>(t) * d]);
      acc += static_cast<double>(s != nullptr ? __fmul_rn(x, sc) : x);
    }
  }
  mu[hq * d + c] = static_cast<float>(acc / static_cast<double>(static_cast<int64_t>(B) * n_cal));
}

// The rank-one score term of the Q-Mean auxiliary: bias[b][hq][key] =
// mu[hq] . K-hat[b][h(hq)][key] for every key of the padded rows (padding
// keys have zero codes: bias 0), accumulated in fp64 (each product of an fp32
// mu and an exact K-hat element is exact there; four interleaved partial sums)
// and rounded once to fp32.  One thread per (b, q head, key), block by block:
// the block's scale byte of the tiled layout, its codes as 32-bit words,
// decoded in registers (E2M1 x block scale, exact in fp32); mu is staged in
// shared memory already widened to fp64.
template <int FMT, int D>
__global__ void __launch_bounds__(128) q_mean_bias_kernel(const uint8_t* __restrict__ kc,
                                                          const uint8_t* __restrict__ ks,
                                                          const float* __restrict__ mu, int Hq, int Hkv, int Np,
                                                          int64_t sf_head_bytes, float* __restrict__ bias) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  constexpr int NB = D / BETA;                     // blocks per row
  constexpr int NKC = (NB + 3) / 4;                // scale words per row
  __shared__ double mu_sh[D];
  const int bhq = blockIdx.y;                      // b * Hq + q head
  const int hq = bhq % Hq, b = bhq / Hq;
  const int bh = b * Hkv + hq / (Hq / Hkv);        // its kv head's K-hat
  for (int i = threadIdx.x; i < D; i += blockDim.x) mu_sh[i] = static_cast<double>(mu[hq * D + i]);
  __syncthreads();
  const int key = blockIdx.x * blockDim.x + threadIdx.x;
  if (key >= Np) return;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(kc + (static_cast<int64_t>(bh) * Np + key) * (D / 2));
  const uint8_t* sfh = ks + static_cast<int64_t>(bh) * sf_head_bytes;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 1
  for (int blk = 0; blk < NB; ++blk) {
    const uint32_t sc = sfh[sf_word_offset(key, blk / 4, NKC) + blk % 4];
    // UE4M3 value, or 2^(sc - 127) (code 0 is 2^-127, a subnormal)
    const float scale = FMT == HIFA4_NVFP4 ? ue4m3_to_f32(sc) : __uint_as_float(sc == 0 ? 0x00400000u : sc << 23);
#pragma unroll
    for (int wi = 0; wi < BETA / 8; ++wi) {
      const uint32_t wd = row[blk * (BETA / 8) + wi];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int c = blk * BETA + 8 * wi + n;
        const uint32_t code = (wd >> (4 * n)) & 15u;
        // E2M1 magnitude: exponent field e, mantissa bit m: 0.5 m for e = 0,
        // else 2^(e-1) (1 + m/2)
        const uint32_t e = (code >> 1) & 3u, m = code & 1u;
        const float mag = e == 0 ? 0.5f * static_cast<float>(m) : __uint_as_float(((e + 126u) << 23) | (m << 22));
        const float kv = __fmul_rn((code & 8u) ? -mag : mag, scale);
        acc[n & 3] = __fma_rn(mu_sh[c], static_cast<double>(kv), acc[n & 3]);
      }
    }
  }
  bias[static_cast<int64_t>(bhq) * Np + key] = static_cast<float>((acc[0] + acc[1]) + (acc[2] + acc[3]));
}

// ---------------------------------------------------------- host launchers ---
template <typename T, int D>
static void launch_quant_d(const QuantArgs& a, int fmt, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(a.nq_ctas + a.nk_ctas + a.nv_ctas);
  const bool qm = a.q_mu != nullptr;
  if (fmt == HIFA4_NVFP4) {
    if (qm) quantize_qkv_kernel<HIFA4_NVFP4, T, D, true><<<grid, 256, 0, st>>>(a);
    else quantize_qkv_kernel<HIFA4_NVFP4, T, D, false><<<grid, 256, 0, st>>>(a);
  } else {
    if (qm) quantize_qkv_kernel<HIFA4_MXFP4, T, D, true><<<grid, 256, 0, st>>>(a);
    else quantize_qkv_kernel<HIFA4_MXFP4, T, D, false><<<grid, 256, 0, st>>>(a);
  }
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
                                 uint8_t* kc, uint8_t* ks, uint8_t* vc, uint8_t* vs, const float* q_mu,
                                 cudaStream_t st) {
  QuantArgs a;
  a.q = q; a.k = k; a.v = v; a.s = s; a.inv_s = inv_s; a.q_mu = q_mu;
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
  a.v_tasks = static_cast<int64_t>(a.Np / kVTok) * (a.B * a.Hkv) * (a.d / kVCh);   // one warp each
  a.nv_ctas = static_cast<int>((a.v_tasks + 7) / 8);
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

hifa4_status calib_q_mean_launch(const void* q, int dt, int B, int Hq, int Hkv, int n_cal, int ld_tok, int d,
                                 const float* s, float* mu, cudaStream_t st) {
  if (dt == HIFA4_BF16)
    calib_q_mean_kernel<__nv_bfloat16><<<Hq, d, 0, st>>>(static_cast<const __nv_bfloat16*>(q), B, Hq, Hq / Hkv,
                                                         ld_tok, n_cal, d, s, mu);
  else
    calib_q_mean_kernel<__half><<<Hq, d, 0, st>>>(static_cast<const __half*>(q), B, Hq, Hq / Hkv, ld_tok, n_cal,
                                                  d, s, mu);
  return launch_status("calibrate_q_mean");
}

hifa4_status q_mean_bias_launch(const uint8_t* kc, const uint8_t* ks, const float* mu, int B, int Hq, int Hkv, int N,
                                int d, int fmt, float* bias, cudaStream_t st) {
  const int Np = static_cast<int>(pad128(N));
  const int64_t sf_head = static_cast<int64_t>(hifa4_scale_bytes(N, d, static_cast<hifa4_format>(fmt)));
  const dim3 grid(static_cast<unsigned>(Np / 128), static_cast<unsigned>(B * Hq));
  auto go = [&](auto fmt_tag, auto d_tag) {
    constexpr int F = decltype(fmt_tag)::value, DD = decltype(d_tag)::value;
    q_mean_bias_kernel<F, DD><<<grid, 128, 0, st>>>(kc, ks, mu, Hq, Hkv, Np, sf_head, bias);
  };
  using NV = std::integral_constant<int, HIFA4_NVFP4>;
  using MX = std::integral_constant<int, HIFA4_MXFP4>;
  if (fmt == HIFA4_NVFP4) {
    if (d == 64) go(NV{}, std::integral_constant<int, 64>{});
    else if (d == 128) go(NV{}, std::integral_constant<int, 128>{});
    else go(NV{}, std::integral_constant<int, 256>{});
  } else {
    if (d == 64) go(MX{}, std::integral_constant<int, 64>{});
    else if (d == 128) go(MX{}, std::integral_constant<int, 128>{});
    else go(MX{}, std::integral_constant<int, 256>{});
  }
  return launch_status("q_mean_bias");
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
