// attn_bf16.cu -- plain BF16 FlashAttention forward on sm_100a, the in-house
// reference the 4-bit kernel is measured against.
//
// Same machinery as the 4-bit kernel, without quantization: one CTA = one
// 128-row query tile of one (batch, q head), 64-key tiles in ascending order,
//   warps 0-3   softmax, one thread per query row (TMEM lane): tcgen05.ld the
//               S row, online max m and normalizer l (fp32, over the
//               unrounded P), P = 2^(S*c - m) rounded to bf16 and stored
//               swizzled into shared memory as the A operand of the PV MMA;
//               when m rises, O is rescaled in TMEM after the previous PV MMA
//               retired.  Epilogue O / l, lse = m + log2 l (base 2).
//   warp 4      TMA producer: Q tile once, K tiles into a 2-stage ring, V^T
//               tiles into a single stage.
//   warp 5      MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 accumulate)
//               for S = Q K^T and O += P V, completion by tcgen05.commit.
// Operands are K-major in 128-byte swizzle atoms (64 bf16 per row); V comes
// pre-transposed (V^T [B, Hkv, d, N]) so that the PV B operand is K-major as
// well (transpose_v_bf16 below).  Every wait is bounded (ptx.cuh).
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

struct Bf16Params {
  int B, Hq, Hkv, N, G;
  int num_qtiles;
  float c_log2;  // softmax_scale * log2(e)
  int causal;
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
struct Bf16Cfg {
  // K tiles double-buffered, V^T single (two CTAs per SM must fit in 228 KB)
  static constexpr int BM = 128, BN = 64, NS = 2, NSV = 1;
  static constexpr int ATOMS = D / 64;                      // 128-byte atoms per Q/K row
  static constexpr int SZ_Q = ATOMS * BM * 128;
  static constexpr int SZ_K = ATOMS * BN * 128;
  static constexpr int SZ_V = D * 128;                      // D rows x 64 keys
  static constexpr int SZ_P = BM * 128;                     // 128 rows x 64 keys
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + SZ_Q;
  static constexpr int OFF_V = OFF_K + NS * SZ_K;
  static constexpr int OFF_P = OFF_V + NSV * SZ_V;
  static constexpr int OFF_BAR = OFF_P + SZ_P;
  // q_full, k_full[NS], k_empty[NS], v_full[NSV], v_empty[NSV], s_full, s_empty, p_full, p_empty
  static constexpr int NBAR = 1 + 2 * NS + 2 * NSV + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int TM_S = 0;
  static constexpr int TM_O = BN;
  static constexpr int TMEM_ALLOC = BN + D <= 128 ? 128 : (BN + D <= 256 ? 256 : 512);
  static constexpr int CTAS_PER_SM = 512 / TMEM_ALLOC > 2 ? 2 : 512 / TMEM_ALLOC;
  static_assert(SMEM_BYTES * CTAS_PER_SM <= 226 * 1024, "shared memory for the resident CTAs");
};

template <int D>
__global__ void __launch_bounds__(192, Bf16Cfg<D>::CTAS_PER_SM)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const Bf16Params p) {
  using C = Bf16Cfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NS, B_VFULL = 1 + 2 * C::NS, B_VEMPTY = B_VFULL + C::NSV,
            B_SFULL = B_VEMPTY + C::NSV, B_SEMPTY = B_SFULL + 1, B_PFULL = B_SEMPTY + 1, B_PEMPTY = B_PFULL + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  // heavy (late) query tiles first for causal balance
  const int bhq = blockIdx.x % (p.B * p.Hq);
  const int qtile = p.num_qtiles - 1 - static_cast<int>(blockIdx.x / (p.B * p.Hq));
  const int b = bhq / p.Hq, hq = bhq % p.Hq;
  const int kvbh = b * p.Hkv + hq / p.G;
  const int row0 = qtile * C::BM;
  const int kv_end = p.causal ? min(p.N, row0 + C::BM) : p.N;
  const int nkt = (kv_end + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::NSV; ++s) {
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_VEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SEMPTY), 4);
    mbar_init(BAR(B_PFULL), 4);
    mbar_init(BAR(B_PEMPTY), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // =============================== TMA producer ===============================
    if (lane == 0) {
      mbar_arrive_expect_tx(BAR(B_QFULL), C::SZ_Q);
      for (int a = 0; a < C::ATOMS; ++a)
        tma_load_2d(sbase + C::OFF_Q + a * C::BM * 128, &tm_q, a * 128, bhq * p.N + row0, BAR(B_QFULL));
      for (int j = 0; j < nkt; ++j) {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait(BAR(B_KEMPTY + st), ph ^ 1, abort_flag, kErrTimeoutTma)) break;
        mbar_arrive_expect_tx(BAR(B_KFULL + st), C::SZ_K);
        for (int a = 0; a < C::ATOMS; ++a)
          tma_load_2d(sbase + C::OFF_K + st * C::SZ_K + a * BN * 128, &tm_k, a * 128, kvbh * p.N + j * BN,
                      BAR(B_KFULL + st));
        const int sv = j % C::NSV;
        if (!mbar_wait(BAR(B_VEMPTY + sv), ((j / C::NSV) & 1) ^ 1, abort_flag, kErrTimeoutTma)) break;
        mbar_arrive_expect_tx(BAR(B_VFULL + sv), C::SZ_V);
        tma_load_2d(sbase + C::OFF_V + sv * C::SZ_V, &tm_v, j * BN * 2, kvbh * D, BAR(B_VFULL + sv));
      }
    }
  } else if (warp == 5) {
    // ================================ MMA issuer ================================
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16(128, BN, true, false, false);
      constexpr uint32_t kIdO = idesc_f16(128, D, true, false, false);
      bool ok = mbar_wait(BAR(B_QFULL), 0, abort_flag, kErrTimeoutMma);
      auto issue_s = [&](int j) -> bool {
        const int st = j % C::NS;
        if (!mbar_wait(BAR(B_KFULL + st), (j / C::NS) & 1, abort_flag, kErrTimeoutMma)) return false;
        if (!mbar_wait(BAR(B_SEMPTY), (j & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks & 3) * 32;           // K-step within the 128-byte atom
          const uint64_t a = make_kmajor_desc(sbase + C::OFF_Q + (ks >> 2) * C::BM * 128 + off, 128);
          const uint64_t bk = make_kmajor_desc(sbase + C::OFF_K + st * C::SZ_K + (ks >> 2) * BN * 128 + off, 128);
          mma_f16(tmem + C::TM_S, a, bk, kIdS, ks > 0 ? 1u : 0u);
        }
        tc_commit(BAR(B_SFULL));
        tc_commit(BAR(B_KEMPTY + st));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int sv = j % C::NSV;
        if (!mbar_wait(BAR(B_PFULL), j & 1, abort_flag, kErrTimeoutMma)) return false;
        if (!mbar_wait(BAR(B_VFULL + sv), (j / C::NSV) & 1, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t a = make_kmajor_desc(sbase + C::OFF_P + ks * 32, 128);
          const uint64_t bv = make_kmajor_desc(sbase + C::OFF_V + sv * C::SZ_V + ks * 32, 128);
          mma_f16(tmem + C::TM_O, a, bv, kIdO, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(BAR(B_VEMPTY + sv));
        tc_commit(BAR(B_PEMPTY));
        return true;
      };
      if (ok && nkt > 0) ok = issue_s(0);
      for (int j = 0; ok && j < nkt; ++j) {
        if (j + 1 < nkt) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      if (!ok) drain_after_abort();
    }
  } else {
    // ================================== softmax ==================================
    const int r = threadIdx.x;                       // row == TMEM lane (warps 0-3)
    const int row = row0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float c = p.c_log2;
    const float2 c2 = make_float2(c, c);
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkt && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_SFULL), j & 1, abort_flag, kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
      {
        uint32_t v[BN];
        tmem_ld64_wait(tmem + lane_base + C::TM_S, v);
#pragma unroll
        for (int i = 0; i < BN; ++i) s[i] = __uint_as_float(v[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_SEMPTY));
      const int kbase = j * BN;
      if ((kbase + BN > p.N) || (p.causal && kbase + BN - 1 > row0)) {
        const int lim = p.causal ? min(p.N, row + 1) : p.N;
#pragma unroll
        for (int k = 0; k < BN; ++k) s[k] = (kbase + k >= lim) ? -INFINITY : s[k];
      }
      // c > 0: max of fl32(S*c) is fl32(max S * c)
      float mx = fmax3(s[0], s[1], s[2]);
#pragma unroll
      for (int k = 3; k + 1 < BN; k += 2) mx = fmax3(mx, s[k], s[k + 1]);
      mx = fmaxf(mx, s[BN - 1]);
      const float m_new = fmaxf(m, __fmul_rn(mx, c));
      const float alpha = (m_new == m) ? 1.0f : ex2_approx(m - m_new);
      const float2 nm2 = make_float2(-m_new, -m_new);
      uint32_t pk[BN / 2];
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < BN; i += 2) {
        const float2 y = ffma2(make_float2(s[i], s[i + 1]), c2, nm2);
        const float2 pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
        acc = fadd2(acc, pp);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l = fmaf(alpha, l, acc.x + acc.y);
      // the single P buffer (and O) are free once PV_{j-1} retired
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(BAR(B_PEMPTY), (j - 1) & 1, abort_flag, kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      {
        unsigned char* prow = smem + C::OFF_P + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) * 16)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        tc_fence_after();
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          uint32_t v[64];
          const uint32_t a0 = tmem + lane_base + C::TM_O + cc * 64;
          tmem_ld64_wait(a0, v);
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            const float2 t0 = fmul2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), a2);
            v[i] = __float_as_uint(t0.x);
            v[i + 1] = __float_as_uint(t0.y);
          }
          tmem_st64(a0, v);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();   // P is read by the MMA (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_PFULL));
      m = m_new;
    }
    // epilogue: O is final once the last PV MMA retired
    const bool ready = __all_sync(0xffffffffu, ok && nkt > 0 &&
                                                  mbar_wait(BAR(B_PEMPTY), (nkt - 1) & 1, abort_flag, kErrTimeoutSoftmax));
    if (ready) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool store = row < p.N;
      const int64_t orow = (static_cast<int64_t>(bhq) * p.N + row) * D;
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16_wait(tmem + lane_base + C::TM_O + cc * 16, v);
        if (store) {
          uint32_t packed[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
            packed[i] = *reinterpret_cast<uint32_t*>(&hh);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.o + orow + cc * 16);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
      }
      if (store && p.lse) p.lse[static_cast<int64_t>(bhq) * p.N + row] = m + log2f(l);
    }
  }
  if (*abort_flag) drain_after_abort();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_ALLOC);
}

// V [B, Hkv, N, d] -> V^T [B, Hkv, d, N] (bf16), 32 x 32 tiles through shared memory.
__global__ void transpose_v_bf16_kernel(const __nv_bfloat16* __restrict__ v, int N, int d,
                                        __nv_bfloat16* __restrict__ vt) {
  __shared__ __nv_bfloat16 t[32][33];
  const int64_t head = blockIdx.z;
  const int n0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  const __nv_bfloat16* src = v + head * N * d;
  __nv_bfloat16* dst = vt + head * N * d;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, cc = c0 + threadIdx.x;
    if (n < N && cc < d) t[i][threadIdx.x] = src[static_cast<int64_t>(n) * d + cc];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int cc = c0 + i, n = n0 + threadIdx.x;
    if (n < N && cc < d) dst[static_cast<int64_t>(cc) * N + n] = t[threadIdx.x][i];
  }
}

bool make_tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, int swizzle_bytes);

template <int D>
static hifa4_status launch_bf16_t(const void* q, const void* k, const void* vt, const Bf16Params& p, cudaStream_t st) {
  using C = Bf16Cfg<D>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_2d(&tq, q, static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(p.B) * p.Hq * p.N, 128, C::BM, 128) ||
      !make_tmap_2d(&tk, k, static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(p.B) * p.Hkv * p.N, 128, C::BN, 128) ||
      !make_tmap_2d(&tv, vt, static_cast<uint64_t>(p.N) * 2, static_cast<uint64_t>(p.B) * p.Hkv * D, 128, D, 128)) {
    set_last_error("bf16_attn_fwd: tensor map encoding failed");
    return HIFA4_ERR_CUDA;
  }
  auto kern = attn_fwd_bf16_kernel<D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * p.num_qtiles;
  kern<<<grid, 192, C::SMEM_BYTES, st>>>(tq, tk, tv, p);
  return launch_status("bf16_attn_fwd");
}

hifa4_status bf16_attn_launch(const void* q, const void* k, const void* vt, int B, int Hq, int Hkv, int N, int d,
                              float softmax_scale, int causal, void* o, float* lse, cudaStream_t st) {
  Bf16Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.num_qtiles = (N + 127) / 128;
  p.c_log2 = softmax_scale * 1.4426950408889634f;
  p.causal = causal;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  if (B == 0 || N == 0) return HIFA4_OK;
  if (d == 64) return launch_bf16_t<64>(q, k, vt, p, st);
  if (d == 128) return launch_bf16_t<128>(q, k, vt, p, st);
  return launch_bf16_t<256>(q, k, vt, p, st);
}

hifa4_status transpose_v_bf16_launch(const void* v, int B, int Hkv, int N, int d, void* vt, cudaStream_t st) {
  if (B == 0 || N == 0) return HIFA4_OK;
  dim3 grid((N + 31) / 32, (d + 31) / 32, B * Hkv);
  transpose_v_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(static_cast<const __nv_bfloat16*>(v), N, d,
                                                        static_cast<__nv_bfloat16*>(vt));
  return launch_status("bf16_transpose_v");
}

}  // namespace hifa4
