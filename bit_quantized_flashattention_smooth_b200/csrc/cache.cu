// cache.cu -- appending tokens to a 4-bit KV cache for decode.
//
// The cache holds K-hat rows (blocks of BETA channels, independent per token)
// and V-hat^T rows (blocks of BETA tokens along each channel), in the same
// layouts and by the same block rules as the fused quantize kernel, at a fixed
// capacity Np = pad128(capacity).  Appending tokens [pos, pos + T):
//   K: each new row is scaled by 1/s and block-quantized in place.
//   V: every token block the new tokens touch is quantized again from its raw
//      values: the tokens before pos come from the caller's `v_tail` buffer
//      (the raw V of the partially filled last block), the new ones from
//      v_new, tokens not yet written are 0 as in a one-shot quantization.
//   v_tail is then updated with the raw V of the new partial block.
// The cache after any sequence of appends equals the one-shot quantization of
// the whole sequence (the block rules see the same values), which the tests
// check bit for bit.  (Decode-side cache append is a deployment need of this
// library; the paper describes prefill and decode over a given cache.)
#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

template <typename T>
__device__ __forceinline__ float to_f32(T x) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) return __bfloat162float(x);
  else return __half2float(x);
}

// One block of BETA values -> packed E2M1 codes and the scale code (the block
// rules of the quantize kernel: NVFP4 scale fl32(amax/6) to UE4M3, element
// multiplier fl32(1/scale); MXFP4 shared exponent floor(log2 amax) - 2).
template <int FMT, int BETA>
__device__ __forceinline__ uint32_t append_quant_block(const float (&v)[BETA], uint32_t (&packed)[BETA / 8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < BETA; ++i) amax = fmaxf(amax, fabsf(v[i]));
  float mult;
  uint32_t sc;
  uint32_t keep = 0xFFFFFFFFu;
  if constexpr (FMT == HIFA4_NVFP4) {
    sc = cvt_e4m3(__fdiv_rn(amax, 6.0f));
    mult = sc == 0 ? 0.0f : __fdiv_rn(1.0f, ue4m3_to_f32(sc));
    if (sc == 0) keep = 0u;
  } else {
    const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
    sc = ef >= 2u ? ef - 2u : 0u;
    mult = __uint_as_float((254u - sc) << 23);
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

struct AppendArgs {
  const void *k_new, *v_new;
  const float* inv_s;
  uint8_t *kc, *ks, *vc, *vs;
  void* v_tail;
  int B, Hkv, T, d, pos, Np;
  int g0, nblk;                 // first V block touched and how many
  int64_t sf_k_head, sf_v_head;
};

// One launch.  Threads [0, nk) each quantize one (K row, block); threads
// [nk, nk + nv) each own one (head, channel) of V and walk the touched token
// blocks in order: every block is quantized again from its raw values (the
// tokens before pos from v_tail, which only this thread reads or writes for
// its channel, the new ones from v_new, tokens not yet written 0), and the
// channel's tail is then rewritten with the raw V of the new partial block.
template <int FMT, typename T>
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendArgs a) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  const int nb = a.d / BETA;
  const int64_t nk = static_cast<int64_t>(a.B) * a.Hkv * a.T * nb;
  const int64_t nv = static_cast<int64_t>(a.B) * a.Hkv * a.d;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < nk) {
    // ---- K: one (row, block) ----
    const int blk = static_cast<int>(idx % nb);
    const int64_t r = idx / nb;                  // (bh, t)
    const int t = static_cast<int>(r % a.T);
    const int64_t bh = r / a.T;
    const int kvh = static_cast<int>(bh % a.Hkv);
    const int p = a.pos + t;
    const T* src = static_cast<const T*>(a.k_new) + r * a.d + blk * BETA;
    float v[BETA];
#pragma unroll
    for (int i = 0; i < BETA; ++i) {
      v[i] = to_f32(src[i]);
      if (a.inv_s != nullptr) v[i] = __fmul_rn(v[i], a.inv_s[kvh * a.d + blk * BETA + i]);
    }
    uint32_t packed[BETA / 8];
    const uint32_t sc = append_quant_block<FMT, BETA>(v, packed);
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.kc + (bh * a.Np + p) * static_cast<int64_t>(a.d / 2) + blk * (BETA / 2));
#pragma unroll
    for (int w = 0; w < BETA / 8; ++w) dst[w] = packed[w];
    const int wpr = (nb + 3) / 4;
    a.ks[bh * a.sf_k_head + sf_word_offset(p, blk / 4, wpr) + (blk % 4)] = static_cast<uint8_t>(sc);
    return;
  }
  if (idx >= nk + nv) return;
  // ---- V: one (head, channel), all touched blocks, then the tail ----
  const int64_t vi = idx - nk;
  const int c = static_cast<int>(vi % a.d);
  const int64_t bh = vi / a.d;
  T* tail = static_cast<T*>(a.v_tail) + bh * BETA * a.d;
  const T* vn = static_cast<const T*>(a.v_new) + bh * static_cast<int64_t>(a.T) * a.d;
  const int nkc = a.Np / (4 * BETA);
  for (int gi = 0; gi < a.nblk; ++gi) {
    const int g = a.g0 + gi;
    const int tok0 = g * BETA;
    float val[BETA];
#pragma unroll
    for (int i = 0; i < BETA; ++i) {
      const int tok = tok0 + i;
      float x = 0.0f;
      if (tok < a.pos) x = to_f32(tail[(tok - a.g0 * BETA) * a.d + c]);          // only in block g0
      else if (tok < a.pos + a.T) x = to_f32(vn[static_cast<int64_t>(tok - a.pos) * a.d + c]);
      val[i] = x;
    }
    uint32_t packed[BETA / 8];
    const uint32_t sc = append_quant_block<FMT, BETA>(val, packed);
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.vc + (bh * a.d + c) * static_cast<int64_t>(a.Np / 2) + tok0 / 2);
#pragma unroll
    for (int w = 0; w < BETA / 8; ++w) dst[w] = packed[w];
    a.vs[bh * a.sf_v_head + sf_word_offset(c, g / 4, nkc) + (g % 4)] = static_cast<uint8_t>(sc);
  }
  // tail <- raw V of the new partially filled block (tokens before pos in
  // the same block are already in place)
  const int end = a.pos + a.T;
  const int start = end / BETA * BETA;
  for (int tok = start > a.pos ? start : a.pos; tok < end; ++tok)
    tail[(tok - start) * a.d + c] = vn[static_cast<int64_t>(tok - a.pos) * a.d + c];
}

template <int FMT, typename T>
static hifa4_status append_t(const AppendArgs& a, cudaStream_t st) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  const int64_t n = static_cast<int64_t>(a.B) * a.Hkv * a.T * (a.d / BETA) + static_cast<int64_t>(a.B) * a.Hkv * a.d;
  kv_append_kernel<FMT, T><<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a);
  return launch_status("kv_cache_append");
}

hifa4_status kv_append_launch(const void* k_new, const void* v_new, int dt, int B, int Hkv, int T, int d,
                              const float* inv_s, int fmt, int pos, int capacity, uint8_t* kc, uint8_t* ks,
                              uint8_t* vc, uint8_t* vs, void* v_tail, cudaStream_t st) {
  const int beta = beta_of(fmt);
  AppendArgs a;
  a.k_new = k_new; a.v_new = v_new; a.inv_s = inv_s;
  a.kc = kc; a.ks = ks; a.vc = vc; a.vs = vs; a.v_tail = v_tail;
  a.B = B; a.Hkv = Hkv; a.T = T; a.d = d; a.pos = pos;
  a.Np = static_cast<int>(pad128(capacity));
  a.g0 = pos / beta;
  a.nblk = (pos + T - 1) / beta - a.g0 + 1;
  a.sf_k_head = static_cast<int64_t>(hifa4_scale_bytes(capacity, d, static_cast<hifa4_format>(fmt)));
  a.sf_v_head = static_cast<int64_t>(hifa4_scale_bytes(d, a.Np, static_cast<hifa4_format>(fmt)));
  if (dt == HIFA4_BF16)
    return fmt == HIFA4_NVFP4 ? append_t<HIFA4_NVFP4, __nv_bfloat16>(a, st) : append_t<HIFA4_MXFP4, __nv_bfloat16>(a, st);
  return fmt == HIFA4_NVFP4 ? append_t<HIFA4_NVFP4, __half>(a, st) : append_t<HIFA4_MXFP4, __half>(a, st);
}

}  // namespace hifa4
