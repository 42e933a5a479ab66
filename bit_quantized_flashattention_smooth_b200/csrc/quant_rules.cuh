// quant_rules.cuh -- the element-wise block quantizer shared by the fused
// scale + quantize kernel and the attention kernel's in-kernel Q path: one
// block of BETA values -> E2M1 codes + scale code, NVFP4 (UE4M3 scale
// fl32(amax/6) per 16) or MXFP4 (OCP MX v1.0, UE8M0 exponent per 32), all
// decisions in IEEE fp32.  Block rules: "HiFA4: Training-Free 4-bit
// FlashAttention on Ascend HIF4 NPUs for LLM Inference", Abstract para 2
// (Q, K and V quantized to 4 bits in blocks); the formats are NVIDIA's NVFP4
// and the OCP Microscaling v1.0 MXFP4.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

// 1: element multiplies as packed fp32 pairs (FMUL2); 0: scalar multiplies.
// Both round each product to nearest: the results are identical.
#ifndef HIFA4_QUANT_PACKED_MUL
#define HIFA4_QUANT_PACKED_MUL 1
#endif

namespace hifa4 {

__device__ __forceinline__ float2 qmul2(float2 a, float2 b) {
#if HIFA4_QUANT_PACKED_MUL
  return fmul2(a, b);
#else
  return make_float2(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y));
#endif
}

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

// The scale decision of one block from its amax: returns the scale code and
// sets the element multiplier fl32(1/scale) and the code mask (0 when the
// scale is 0, so that no -0 codes appear).  inv_tab[c] = fl32(1 / UE4M3(c)) *
// 2^TAB_LOG2 (0 for c = 0), in shared memory; the power of two is taken out
// exactly.
template <int FMT, int TAB_LOG2 = 0>
__device__ __forceinline__ uint32_t block_scale(float amax, const float* inv_tab, float& mult, uint32_t& keep) {
  uint32_t sc;
  keep = 0xFFFFFFFFu;
  if constexpr (FMT == HIFA4_NVFP4) {
    // fl32(amax/6): the reciprocal-and-residual form is IEEE-exact on
    // [2^-122, 2^20] (checked on the GPU); below, both give scale code 0
    sc = cvt_e4m3(div6_any(amax));
    mult = TAB_LOG2 == 0 ? inv_tab[sc] : __fmul_rn(inv_tab[sc], __uint_as_float(static_cast<uint32_t>(127 - TAB_LOG2) << 23));
    if (sc == 0) keep = 0u;                             // scale 0: every code 0 (no -0 codes)
  } else {
    const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
    sc = ef >= 2u ? ef - 2u : 0u;                       // E + 127, E = floor(log2 amax) - 2
    mult = __uint_as_float((254u - sc) << 23);          // 2^-E
  }
  return sc;
}

// Quantize one block of BETA fp32 values in place into packed codes
// (BETA/2 bytes, element 2i in the low nibble) and return the scale code.
template <int FMT, int BETA, int TAB_LOG2 = 0>
__device__ __forceinline__ uint32_t quant_block(const float (&v)[BETA], uint32_t (&packed)[BETA / 8],
                                                const float* inv_tab) {
  float amax = fmaxf(fabsf(v[0]), fabsf(v[1]));
#pragma unroll
  for (int i = 2; i + 1 < BETA; i += 2) amax = fmax3(amax, fabsf(v[i]), fabsf(v[i + 1]));
  float mult;
  uint32_t keep;
  const uint32_t sc = block_scale<FMT, TAB_LOG2>(amax, inv_tab, mult, keep);
  const float2 m2 = make_float2(mult, mult);
#pragma unroll
  for (int w = 0; w < BETA / 8; ++w) {
    const float* e = v + 8 * w;
    packed[w] = keep & cvt_e2m1x8(qmul2(make_float2(e[0], e[1]), m2), qmul2(make_float2(e[2], e[3]), m2),
                                  qmul2(make_float2(e[4], e[5]), m2), qmul2(make_float2(e[6], e[7]), m2));
  }
  return sc;
}

}  // namespace hifa4
