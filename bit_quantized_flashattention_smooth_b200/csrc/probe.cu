// probe.cu -- measurement / conformance kernels:
//  * fp4_mma_probe: one 128 x n block-scaled FP4 product (TMA-loaded operands,
//    tcgen05.cp scale copies, tcgen05.mma) repeated R times into one TMEM
//    accumulator; with many CTAs it measures the dense FP4 tensor peak, with
//    one CTA it checks operand / scale layouts against a CPU product.
//  * convert_probe: the hardware E2M1 / E4M3 conversions element by element,
//    to check the written rounding rules against the instructions.
#include <cstdint>
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

template <int N, int K, int FMT>
__global__ void __launch_bounds__(128, 1)
    fp4_mma_probe_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const uint8_t* __restrict__ a_sf, const uint8_t* __restrict__ b_sf, int repeats,
                         float* __restrict__ d_out) {
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  constexpr int ROW = K / 2;
  constexpr int NKC = (K / BETA + 3) / 4;
  constexpr int NRG = (N + 127) / 128;
  constexpr int SZ_A = 128 * ROW, SZ_B = N * ROW;
  constexpr int OFF_A = 0, OFF_B = SZ_A, OFF_ASF = OFF_B + SZ_B, OFF_BSF = OFF_ASF + NKC * 512;
  constexpr int OFF_BAR = OFF_BSF + NRG * NKC * 512;
  constexpr int TM_D = 0, TM_SFA = 256, TM_SFB = TM_SFA + 4 * NKC;
  constexpr bool MX = FMT == HIFA4_MXFP4;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_load = sbase + OFF_BAR, bar_mma = sbase + OFF_BAR + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 20);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(bar_load, SZ_A + SZ_B + NKC * 512 + NRG * NKC * 512);
    tma_load_2d(sbase + OFF_A, &tm_a, 0, 0, bar_load);
    tma_load_2d(sbase + OFF_B, &tm_b, 0, 0, bar_load);
    bulk_load(sbase + OFF_ASF, a_sf, NKC * 512, bar_load);
    bulk_load(sbase + OFF_BSF, b_sf, NRG * NKC * 512, bar_load);
    ok = mbar_wait(bar_load, 0, abort_flag, kErrTimeoutOther);
    if (ok) {
      tc_fence_after();
      for (int kc = 0; kc < NKC; ++kc) {
        tc_cp_32x128b_warpx4(tmem + TM_SFA + 4 * kc, make_sf_desc(sbase + OFF_ASF + kc * 512));
        for (int rg = 0; rg < NRG; ++rg)
          // B scale matrix: row groups first, then chunks (tiled layout order)
          tc_cp_32x128b_warpx4(tmem + TM_SFB + 4 * (kc * NRG + rg),
                               make_sf_desc(sbase + OFF_BSF + (rg * NKC + kc) * 512));
      }
      for (int rep = 0; rep < repeats; ++rep) {
#pragma unroll
        for (int ks = 0; ks < K / 64; ++ks) {
          const uint32_t chunk = MX ? ks / 2 : ks, byte = MX ? 2 * (ks % 2) : 0;
          const uint64_t a = make_kmajor_desc(sbase + OFF_A + ks * 32, ROW);
          const uint64_t b = make_kmajor_desc(sbase + OFF_B + ks * 32, ROW);
          const uint32_t idesc = idesc_fp4(128, N, MX, byte, byte);
          const uint32_t sfa = (tmem + TM_SFA + 4 * chunk) | (byte << 30);
          const uint32_t sfb = (tmem + TM_SFB + 4 * chunk * NRG) | (byte << 30);
          const uint32_t acc = (rep > 0 || ks > 0) ? 1u : 0u;
          if constexpr (MX) mma_mxfp4(tmem + TM_D, a, b, idesc, sfa, sfb, acc);
          else mma_nvfp4(tmem + TM_D, a, b, idesc, sfa, sfb, acc);
        }
      }
      tc_commit(bar_mma);
    }
  }
  __syncwarp();
  ok = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, abort_flag, kErrTimeoutOther));
  if (ok) {
    tc_fence_after();
    if (blockIdx.x == 0) {
      const int r = threadIdx.x;
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
      for (int cc = 0; cc < N / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16_wait(tmem + lane_base + TM_D + cc * 16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) d_out[r * N + cc * 16 + i] = __uint_as_float(v[i]);
      }
    }
  } else {
    drain_after_abort();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool make_tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, int swizzle_bytes);

template <int N, int K, int FMT>
static hifa4_status launch_probe_t(const uint8_t* ac, const uint8_t* as, const uint8_t* bc, const uint8_t* bs,
                                   int repeats, int ctas, float* d_out, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, ac, K / 2, 128, K / 2, 128, K / 2) || !make_tmap_2d(&tb, bc, K / 2, N, K / 2, N, K / 2)) {
    set_last_error("cuTensorMapEncodeTiled failed");
    return HIFA4_ERR_CUDA;
  }
  constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  constexpr int NKC = (K / BETA + 3) / 4, NRG = (N + 127) / 128;
  int smem = 128 * K / 2 + N * K / 2 + NKC * 512 + NRG * NKC * 512 + 64 + 1024;
  if (smem < 116 * 1024) smem = 116 * 1024;  // one CTA per SM: it owns all TMEM columns
  auto kern = fp4_mma_probe_kernel<N, K, FMT>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  kern<<<ctas, 128, smem, st>>>(ta, tb, as, bs, repeats, d_out);
  return launch_status("fp4_mma_probe");
}

template <int N, int K>
static hifa4_status launch_probe_f(int fmt, const uint8_t* ac, const uint8_t* as, const uint8_t* bc,
                                   const uint8_t* bs, int repeats, int ctas, float* d_out, cudaStream_t st) {
  if (fmt == HIFA4_NVFP4) return launch_probe_t<N, K, HIFA4_NVFP4>(ac, as, bc, bs, repeats, ctas, d_out, st);
  return launch_probe_t<N, K, HIFA4_MXFP4>(ac, as, bc, bs, repeats, ctas, d_out, st);
}

hifa4_status fp4_mma_probe_launch(const uint8_t* ac, const uint8_t* as, const uint8_t* bc, const uint8_t* bs, int n,
                                  int k, int fmt, int repeats, int ctas, float* d_out, cudaStream_t st) {
#define HIFA4_PROBE_CASE(NN, KK) \
  if (n == NN && k == KK) return launch_probe_f<NN, KK>(fmt, ac, as, bc, bs, repeats, ctas, d_out, st);
  HIFA4_PROBE_CASE(64, 128)
  HIFA4_PROBE_CASE(128, 128)
  HIFA4_PROBE_CASE(256, 128)
  HIFA4_PROBE_CASE(64, 256)
  HIFA4_PROBE_CASE(128, 256)
  HIFA4_PROBE_CASE(256, 256)
#undef HIFA4_PROBE_CASE
  set_last_error("fp4_mma_probe: unsupported n=%d k=%d", n, k);
  return HIFA4_ERR_UNSUPPORTED;
}

__global__ void convert_probe_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ e2m1,
                                     uint8_t* __restrict__ e4m3) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    e2m1[i] = static_cast<uint8_t>(cvt_e2m1x2(0.0f, v) & 0xFu);
    e4m3[i] = static_cast<uint8_t>(cvt_e4m3(v));
  }
}

// Every float bit pattern in [lo, hi): count where div6_rn differs from the
// IEEE quotient, or div6_rn_x256 from 2^8 times it; record the smallest
// failing pattern.
__global__ void div6_probe_kernel(uint32_t lo, uint32_t hi, unsigned long long* count, uint32_t* first_bad) {
  for (uint64_t b = lo + static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < hi;
       b += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const float a = __uint_as_float(static_cast<uint32_t>(b));
    const float q = __fdiv_rn(a, 6.0f);
    if (__float_as_uint(div6_rn(a)) != __float_as_uint(q) ||
        __float_as_uint(div6_rn_x256(a)) != __float_as_uint(__fmul_rn(q, 256.0f))) {
      atomicAdd(count, 1ull);
      atomicMin(first_bad, static_cast<uint32_t>(b));
    }
  }
}

hifa4_status div6_probe_launch(uint32_t lo, uint32_t hi, unsigned long long* count, uint32_t* first_bad,
                               cudaStream_t st) {
  div6_probe_kernel<<<148 * 16, 256, 0, st>>>(lo, hi, count, first_bad);
  return launch_status("div6_probe");
}

hifa4_status convert_probe_launch(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3, cudaStream_t st) {
  convert_probe_kernel<<<148 * 8, 256, 0, st>>>(x, n, e2m1, e4m3);
  return launch_status("convert_probe");
}

__global__ void exp2_poly_probe_kernel(const float* __restrict__ y, int64_t n, float* __restrict__ out) {
  for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float y1 = i + 1 < n ? y[i + 1] : 0.0f;
    const float2 r = exp2_poly2(make_float2(y[i], y1));
    out[i] = r.x;
    if (i + 1 < n) out[i + 1] = r.y;
  }
}
hifa4_status exp2_poly_probe_launch(const float* y, int64_t n, float* out, cudaStream_t st) {
  if (n == 0) return HIFA4_OK;
  exp2_poly_probe_kernel<<<148 * 4, 256, 0, st>>>(y, n, out);
  return launch_status("exp2_poly_probe");
}

// E2M1 codes of 2^y for `n` values y, two ways: from the exponential-free
// code argument (codes_map) and from the MUFU 2^y (codes_ex2), both through
// the same RNE, saturating conversion; one code per byte.
__global__ void e2m1_map_probe_kernel(const float* __restrict__ y, int64_t n, uint8_t* __restrict__ codes_map,
                                      uint8_t* __restrict__ codes_ex2) {
  for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float y0 = y[i], y1 = i + 1 < n ? y[i + 1] : -100.0f;
    const float2 w = e2m1_arg_from_log2(make_float2(y0, y1));
    const uint32_t a = cvt_e2m1x2(w.y, w.x);
    const uint32_t b = cvt_e2m1x2(ex2_approx(y1), ex2_approx(y0));
    codes_map[i] = static_cast<uint8_t>(a & 15u);
    codes_ex2[i] = static_cast<uint8_t>(b & 15u);
    if (i + 1 < n) {
      codes_map[i + 1] = static_cast<uint8_t>((a >> 4) & 15u);
      codes_ex2[i + 1] = static_cast<uint8_t>((b >> 4) & 15u);
    }
  }
}
hifa4_status e2m1_map_probe_launch(const float* y, int64_t n, uint8_t* cm, uint8_t* ce, cudaStream_t st) {
  if (n == 0) return HIFA4_OK;
  e2m1_map_probe_kernel<<<148 * 4, 256, 0, st>>>(y, n, cm, ce);
  return launch_status("e2m1_map_probe");
}

// The failure path of the bounded mbarrier wait, exercised on purpose: one
// warp waits on a barrier that nothing arrives at.  The wait gives up after
// its time limit, raises the abort flag and ORs kErrTimeoutOther into the
// device error word; the kernel then returns normally (no trap, no hang).
// status[0] = 1 if the wait (wrongly) succeeded, status[1] = abort flag.
__global__ void wait_timeout_probe_kernel(unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, kErrTimeoutOther);
  if (threadIdx.x == 0) {
    status[0] = ok ? 1u : 0u;
    status[1] = static_cast<unsigned int>(abort_flag);
  }
}
hifa4_status wait_timeout_probe_launch(unsigned int* status, cudaStream_t st) {
  wait_timeout_probe_kernel<<<1, 32, 0, st>>>(status);
  return launch_status("wait_timeout_probe");
}

}  // namespace hifa4
