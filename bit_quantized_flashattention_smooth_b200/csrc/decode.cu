// decode.cu -- split-KV decode over a 4-bit KV cache, and the split combine.
//
// Method: the prefill recurrence of "HiFA4: Training-Free 4-bit FlashAttention
// on Ascend HIF4 NPUs for LLM Inference" (Abstract paras 1-2) for one query
// per head: Smooth-QK-scaled query quantized to 4 bits, S = Q-hat K-hat^T and
// O += P-hat V-hat as block-scaled FP4 GEMMs, online softmax, and under
// P-Reordering the normalizer accumulated from the same P-hat inside the PV
// GEMM.  Keys are split into chunks that run in parallel and are merged with
// their log-sum-exp weights.
//
// B200 design, one CTA per (batch, kv head, split), "swap AB": the 128 keys of
// a tile are the M dimension of the MMA and the G query heads of the group
// (padded to N = 16) are the N dimension, so the tensor core is not wasted on
// 127 empty query rows:
//   S^T [128 keys x 16]   = K-hat tile (A, from the cache by TMA) x Q-hat^T (B)
//   O^T [128 ch   x 16]  += V-hat^T tile (A, channel-major cache) x P-hat^T (B)
//   L^T [128      x 16]  += ones (A) x P-hat^T (B)      (fused normalizer)
// The softmax warps hold one key per thread (TMEM lane) and reduce across keys
// with warp shuffles plus a 4-warp exchange in shared memory.  The kernel is
// bound by HBM: it streams each K/V tile once through a 2-stage TMA ring.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

struct DecodeParams {
  const void* q;        // [B][Hq][d] bf16/fp16
  const float* s;       // [Hkv][d] or null
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  int64_t sf_k_head, sf_v_head;
  int B, Hq, Hkv, G, kv_len, Np, split_len, splits;
  int q_fp16;
  float c_log2;
  float tau;            // rescale threshold (log2 units); 0 = exact running max
  float* ws;            // [B][Hq][splits][d+2]: acc (true units), m, l
};

template <int FMT>
struct DecCfg {
  static constexpr int D = 128, BN = 128, NQ = 16;          // head dim, keys per tile, padded queries
  static constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  static constexpr int NS = 2;                               // two stages, four CTAs per SM
  static constexpr int ROW = 64;                            // bytes per 128-element 4-bit row
  static constexpr int NKC = (D / BETA + 3) / 4;            // scale chunks per 128 keys / 128 channels
  static constexpr int SZ_K = BN * ROW, SZ_V = D * ROW, SZ_QB = NQ * ROW, SZ_ONES = 128 * ROW;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NS * SZ_K;
  static constexpr int OFF_ONES = OFF_V + NS * SZ_V;
  static constexpr int OFF_Q = OFF_ONES + SZ_ONES;
  static constexpr int OFF_P = OFF_Q + SZ_QB;                // 2 buffers
  static constexpr int OFF_KSF = OFF_P + 2 * SZ_QB;
  static constexpr int OFF_VSF = OFF_KSF + NS * NKC * 512;
  static constexpr int OFF_QSF = OFF_VSF + NS * NKC * 512;
  static constexpr int OFF_PSF = OFF_QSF + NKC * 512;        // 2 buffers
  static constexpr int OFF_ONESF = OFF_PSF + 2 * NKC * 512;
  static constexpr int OFF_RED = OFF_ONESF + 512;            // [2 parities][max | sum][4 warps][8] floats
  static constexpr int OFF_INV = OFF_RED + 2 * 2 * 4 * 8 * 4;
  static constexpr int OFF_BAR = OFF_INV + 512;
  // k_full/k_empty/v_full/v_empty [NS], s_full, s_empty, p_full/p_empty [2], o_full/o_empty [2]
  static constexpr int NBAR = 4 * NS + 2 + 4 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // TMEM columns: S (one buffer), per-tile O and L partials (two buffers each), scales
  static constexpr int TM_S = 0;
  static constexpr int TM_O = 16;
  static constexpr int TM_L = 48;
  static constexpr int TM_SFK = 80;
  static constexpr int TM_SFQ = TM_SFK + 4 * NKC;
  static constexpr int TM_SFV = TM_SFQ + 4 * NKC;
  static constexpr int TM_SFP = TM_SFV + 4 * NKC;
  static constexpr int TM_SF1 = TM_SFP + 4 * NKC;
  static constexpr int TMEM_ALLOC = 128;
  static_assert(TM_SF1 + 4 <= TMEM_ALLOC, "TMEM budget");
  static_assert(SMEM_BYTES * 4 <= 227 * 1024, "four CTAs per SM");
};

__device__ __forceinline__ uint32_t swz64(uint32_t r, uint32_t c) { return c ^ ((r >> 1) & 3); }

// G = query heads per kv head (1, 2, 4 or 8); the MMA N dimension is 16.
template <int FMT, bool PREORDER, int G>
__global__ void __launch_bounds__(192, 4)
    attn_decode_fp4_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const DecodeParams p) {
  using C = DecCfg<FMT>;
  constexpr bool MX = FMT == HIFA4_MXFP4;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const int B_KFULL = 0, B_KEMPTY = C::NS, B_VFULL = 2 * C::NS, B_VEMPTY = 3 * C::NS, B_SFULL = 4 * C::NS,
            B_SEMPTY = B_SFULL + 1, B_PFULL = B_SEMPTY + 1, B_PEMPTY = B_PFULL + 2, B_OFULL = B_PEMPTY + 2,
            B_OEMPTY = B_OFULL + 2, B_RED = B_OEMPTY + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);

  const int sp = blockIdx.x % p.splits;
  const int bh = blockIdx.x / p.splits;      // b * Hkv + h
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int k_begin = sp * p.split_len;
  const int k_end = min(p.kv_len, k_begin + p.split_len);
  const int ntile = (k_end - k_begin + C::BN - 1) / C::BN;
  const float kGP = FMT == HIFA4_NVFP4 ? 0.00390625f : 1.0f;

  // ---------------------------------------------------------------- setup ---
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_KEMPTY + s), 1);
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_VEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SEMPTY), 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(B_PFULL + s), 4);
      mbar_init(BAR(B_PEMPTY + s), 1);
      mbar_init(BAR(B_OFULL + s), 1);
      mbar_init(BAR(B_OEMPTY + s), 4);
    }
    mbar_init(BAR(B_RED), 4);      // cross-warp reductions of the softmax warps (one arrival per warp)
    *abort_flag = 0;
    fence_mbar_init();
  }
  // ones A operand (128 rows of E2M1 1.0) and its scale chunk (1.0 on every row)
  for (int i = threadIdx.x; i < C::SZ_ONES / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem + C::OFF_ONES)[i] = 0x22222222u;
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    reinterpret_cast<uint32_t*>(smem + C::OFF_ONESF)[i] = (FMT == HIFA4_NVFP4 ? 0x38u : 0x7Fu) * 0x01010101u;
    const float sd = __fmul_rn(ue4m3_to_f32(i), kGP);
    reinterpret_cast<float*>(smem + C::OFF_INV)[i] = i == 0 ? 0.0f : __fdiv_rn(1.0f, sd);
  }
  // the query rows of this group: fl32(q * s) quantized along d (B operand,
  // 16 rows, rows >= G are zero) and its scale chunk(s)
  for (int i = threadIdx.x; i < C::SZ_QB / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(smem + C::OFF_Q)[i] = 0u;
  for (int i = threadIdx.x; i < C::NKC * 128; i += blockDim.x) reinterpret_cast<uint32_t*>(smem + C::OFF_QSF)[i] = 0u;
  __syncthreads();
  if (warp == 0) {
    constexpr int NBLK = G * (C::D / C::BETA);
    for (int t = lane; t < NBLK; t += 32) {
      const int g = t / (C::D / C::BETA), blk = t % (C::D / C::BETA);
      const int hq = h * G + g;
      float v[C::BETA];
      for (int i = 0; i < C::BETA; ++i) {
        const int c = blk * C::BETA + i;
        const int64_t off = (static_cast<int64_t>(b) * p.Hq + hq) * C::D + c;
        float x = p.q_fp16 ? __half2float(reinterpret_cast<const __half*>(p.q)[off])
                           : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[off]);
        v[i] = p.s ? __fmul_rn(x, p.s[h * C::D + c]) : x;
      }
      float amax = 0.0f;
      for (int i = 0; i < C::BETA; ++i) amax = fmaxf(amax, fabsf(v[i]));
      uint32_t sc;
      float mult;
      if constexpr (FMT == HIFA4_NVFP4) {
        sc = cvt_e4m3(__fdiv_rn(amax, 6.0f));
        mult = sc == 0 ? 0.0f : __fdiv_rn(1.0f, ue4m3_to_f32(sc));
      } else {
        const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
        sc = ef >= 2u ? ef - 2u : 0u;
        mult = __uint_as_float((254u - sc) << 23);
      }
      for (int i = 0; i < C::BETA; i += 2) {
        uint32_t byte = cvt_e2m1x2(__fmul_rn(v[i + 1], mult), __fmul_rn(v[i], mult));
        if (FMT == HIFA4_NVFP4 && sc == 0) byte = 0;
        const int kb = (blk * C::BETA + i) / 2;   // byte in the 64-byte row
        smem[C::OFF_Q + g * C::ROW + swz64(g, kb >> 4) * 16 + (kb & 15)] = static_cast<unsigned char>(byte);
      }
      smem[C::OFF_QSF + (blk / 4) * 512 + g * 16 + (blk % 4)] = static_cast<unsigned char>(sc);
    }
  }
  fence_proxy_async_smem();
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      for (int j = 0; j < ntile; ++j) {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        const int key0 = k_begin + j * C::BN;
        if (!mbar_wait(BAR(B_KEMPTY + st), ph ^ 1, abort_flag, kErrTimeoutTma)) break;
        mbar_arrive_expect_tx(BAR(B_KFULL + st), C::SZ_K + C::NKC * 512);
        tma_load_2d(sbase + C::OFF_K + st * C::SZ_K, &tm_k, 0, bh * p.Np + key0, BAR(B_KFULL + st));
        bulk_load(sbase + C::OFF_KSF + st * C::NKC * 512,
                  p.k_sf + bh * p.sf_k_head + static_cast<int64_t>(key0 >> 7) * C::NKC * 512, C::NKC * 512,
                  BAR(B_KFULL + st));
        if (!mbar_wait(BAR(B_VEMPTY + st), ph ^ 1, abort_flag, kErrTimeoutTma)) break;
        mbar_arrive_expect_tx(BAR(B_VFULL + st), C::SZ_V + C::NKC * 512);
        tma_load_2d(sbase + C::OFF_V + st * C::SZ_V, &tm_v, key0 / 2, bh * C::D, BAR(B_VFULL + st));
        bulk_load(sbase + C::OFF_VSF + st * C::NKC * 512,
                  p.v_sf + bh * p.sf_v_head + static_cast<int64_t>(key0 / (4 * C::BETA)) * 512, C::NKC * 512,
                  BAR(B_VFULL + st));
      }
    }
  } else if (warp == 5) {
    // ================================= MMA issuer =================================
    if (lane == 0) {
      auto mma = [&](uint32_t d_t, uint64_t a, uint64_t bd, uint32_t idesc, uint32_t sfa, uint32_t sfb, uint32_t acc) {
        if constexpr (MX) mma_mxfp4(d_t, a, bd, idesc, sfa, sfb, acc);
        else mma_nvfp4(d_t, a, bd, idesc, sfa, sfb, acc);
      };
      bool ok = true;
      tc_fence_after();
      for (int kc = 0; kc < C::NKC; ++kc)
        tc_cp_32x128b_warpx4(tmem + C::TM_SFQ + 4 * kc, make_sf_desc(sbase + C::OFF_QSF + kc * 512));
      tc_cp_32x128b_warpx4(tmem + C::TM_SF1, make_sf_desc(sbase + C::OFF_ONESF));
      // S^T_j = K-hat_j Q-hat^T into the single S buffer
      auto issue_s = [&](int j) -> bool {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait(BAR(B_KFULL + st), ph, abort_flag, kErrTimeoutMma)) return false;
        if (!mbar_wait(BAR(B_SEMPTY), (j & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
        for (int kc = 0; kc < C::NKC; ++kc)
          tc_cp_32x128b_warpx4(tmem + C::TM_SFK + 4 * kc, make_sf_desc(sbase + C::OFF_KSF + (st * C::NKC + kc) * 512));
#pragma unroll
        for (int ks = 0; ks < C::D / 64; ++ks) {
          const uint32_t chunk = MX ? ks / 2 : ks, byte = MX ? 2 * (ks % 2) : 0;
          mma(tmem + C::TM_S, make_kmajor_desc(sbase + C::OFF_K + st * C::SZ_K + ks * 32, C::ROW),
              make_kmajor_desc(sbase + C::OFF_Q + ks * 32, C::ROW), idesc_fp4(128, C::NQ, MX, byte, byte),
              (tmem + C::TM_SFK + 4 * chunk) | (byte << 30), (tmem + C::TM_SFQ + 4 * chunk) | (byte << 30),
              ks > 0 ? 1u : 0u);
        }
        tc_commit(BAR(B_SFULL));
        tc_commit(BAR(B_KEMPTY + st));
        return true;
      };
      // this tile's partials O_j^T = V-hat_j^T P-hat_j^T and L_j^T = ones P-hat_j^T
      // into a fresh buffer (no accumulation across tiles in TMEM)
      auto issue_pv = [&](int j) -> bool {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        const int pb = j & 1;
        if (!mbar_wait(BAR(B_PFULL + pb), (j >> 1) & 1, abort_flag, kErrTimeoutMma)) return false;
        if (!mbar_wait(BAR(B_VFULL + st), ph, abort_flag, kErrTimeoutMma)) return false;
        if (!mbar_wait(BAR(B_OEMPTY + pb), ((j >> 1) & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
        for (int kc = 0; kc < C::NKC; ++kc) {
          tc_cp_32x128b_warpx4(tmem + C::TM_SFV + 4 * kc, make_sf_desc(sbase + C::OFF_VSF + (st * C::NKC + kc) * 512));
          tc_cp_32x128b_warpx4(tmem + C::TM_SFP + 4 * kc, make_sf_desc(sbase + C::OFF_PSF + (pb * C::NKC + kc) * 512));
        }
#pragma unroll
        for (int ks = 0; ks < C::BN / 64; ++ks) {
          const uint32_t chunk = MX ? ks / 2 : ks, byte = MX ? 2 * (ks % 2) : 0;
          const uint64_t bp = make_kmajor_desc(sbase + C::OFF_P + pb * C::SZ_QB + ks * 32, C::ROW);
          const uint32_t sfp = (tmem + C::TM_SFP + 4 * chunk) | (byte << 30);
          mma(tmem + C::TM_O + pb * C::NQ, make_kmajor_desc(sbase + C::OFF_V + st * C::SZ_V + ks * 32, C::ROW), bp,
              idesc_fp4(128, C::NQ, MX, byte, byte), (tmem + C::TM_SFV + 4 * chunk) | (byte << 30), sfp,
              ks > 0 ? 1u : 0u);
          mma(tmem + C::TM_L + pb * C::NQ, make_kmajor_desc(sbase + C::OFF_ONES + ks * 32, C::ROW), bp,
              idesc_fp4(128, C::NQ, MX, byte, byte), (tmem + C::TM_SF1) | (byte << 30), sfp, ks > 0 ? 1u : 0u);
        }
        tc_commit(BAR(B_OFULL + pb));
        tc_commit(BAR(B_VEMPTY + st));
        tc_commit(BAR(B_PEMPTY + pb));
        return true;
      };
      if (ntile > 0) ok = issue_s(0);
      for (int j = 0; ok && j < ntile; ++j) {
        if (j + 1 < ntile) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      if (!ok) drain_after_abort();
    }
  } else {
    // ================================== softmax ==================================
    // thread t = key t of the tile (TMEM lane t) for the scores, and output
    // channel t for the PV partials; columns = the group's G queries
    const int t = threadIdx.x;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float* inv_tab = reinterpret_cast<const float*>(smem + C::OFF_INV);
    float m[G], lp[G], acc[G], lacc[G], alpha_prev[G];
#pragma unroll
    for (int q = 0; q < G; ++q) {
      m[q] = -INFINITY;
      lp[q] = 0.0f;
      acc[q] = 0.0f;
      lacc[q] = 0.0f;
      alpha_prev[q] = 0.0f;
    }
    // fold the partials of tile jj (already complete or about to be) into the
    // register accumulators, scaled by that tile's alpha
    auto fold = [&](int jj) -> bool {
      const int ob = jj & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_OFULL + ob), (jj >> 1) & 1, abort_flag, kErrTimeoutSoftmax)))
        return false;
      tc_fence_after();
      uint32_t o[16], l[16];
      tmem_ld16_wait(tmem + lane_base + C::TM_O + ob * C::NQ, o);
      tmem_ld16_wait(tmem + lane_base + C::TM_L + ob * C::NQ, l);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_OEMPTY + ob));
#pragma unroll
      for (int q = 0; q < G; ++q) {
        acc[q] = fmaf(alpha_prev[q], acc[q], __uint_as_float(o[q]));
        lacc[q] = fmaf(alpha_prev[q], lacc[q], __uint_as_float(l[q]));
      }
      return true;
    };
    bool ok = true;
    for (int j = 0; j < ntile && ok; ++j) {
      const int pb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_SFULL), j & 1, abort_flag, kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16_wait(tmem + lane_base + C::TM_S, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_SEMPTY));
      const bool valid = k_begin + j * C::BN + t < k_end;
      float x[G];
#pragma unroll
      for (int q = 0; q < G; ++q) x[q] = valid ? __fmul_rn(__uint_as_float(v[q]), p.c_log2) : -INFINITY;
      // tile max per query: warp shuffle, then across the 4 warps
      float* rbuf = red + (j & 1) * 2 * 4 * 8;
#pragma unroll
      for (int q = 0; q < G; ++q) {
        float mx = x[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == q) rbuf[warp * 8 + q] = mx;
      }
      // exchange round 2j (the sums of the inconsistent mode use round 2j+1)
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_RED));
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_RED), PREORDER ? (j & 1) : 0, abort_flag, kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      float alpha[G], mnew[G];
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const float tm = fmaxf(fmaxf(rbuf[q], rbuf[8 + q]), fmaxf(rbuf[16 + q], rbuf[24 + q]));
        mnew[q] = tm > m[q] + p.tau ? tm : m[q];     // lazy: the max moves by more than tau
        alpha[q] = (mnew[q] == m[q]) ? 1.0f : ex2_approx(m[q] - mnew[q]);
      }
      // P-hat buffer pb was last read by PV_{j-2}
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(BAR(B_PEMPTY + pb), ((j >> 1) & 1) ^ 1, abort_flag,
                                                        kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      unsigned char* pbuf = smem + C::OFF_P + pb * C::SZ_QB;
      unsigned char* psf = smem + C::OFF_PSF + pb * C::NKC * 512;
      float psum[G];
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const float yq = __fsub_rn(x[q], mnew[q]);
        const float pr = ex2_approx(yq);
        psum[q] = pr;
        uint32_t sc;
        float mult;
        if constexpr (FMT == HIFA4_NVFP4) {
          // block amax over BETA consecutive keys (lanes)
          float bm = pr;
#pragma unroll
          for (int o = C::BETA / 2; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
          sc = cvt_e4m3(div6_rn_x256(bm));
          mult = inv_tab[sc];
        } else {
          // shared exponent from the block maximum of y (exact, see ptx.cuh)
          float ym = yq;
#pragma unroll
          for (int o = C::BETA / 2; o > 0; o >>= 1) ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, o));
          sc = mx_scale_from_ymax(ym);
          mult = __uint_as_float((254u - sc) << 23);
        }
        const float y = __fmul_rn(pr, mult);
        const float y_odd = __shfl_down_sync(0xffffffffu, y, 1);
        if ((t & 1) == 0) {
          const uint32_t byte = cvt_e2m1x2(y_odd, y);
          const int kb = t >> 1;
          pbuf[q * C::ROW + swz64(q, kb >> 4) * 16 + (kb & 15)] = static_cast<unsigned char>(byte);
        }
        if ((t % C::BETA) == 0) {
          const int blk = t / C::BETA;
          psf[(blk / 4) * 512 + q * 16 + (blk % 4)] = static_cast<unsigned char>(sc);
        }
      }
      if constexpr (G < C::NQ) {
        // rows G..15 of the P-hat tile stay zero (written once per buffer)
        if (j < 2) {
          for (int i = t; i < (C::NQ - G) * C::ROW / 4; i += 128)
            reinterpret_cast<uint32_t*>(pbuf + G * C::ROW)[i] = 0u;
          for (int i = t; i < (C::NQ - G) * C::NKC; i += 128) {
            const int r = G + i / C::NKC, kc = i % C::NKC;
            *reinterpret_cast<uint32_t*>(psf + kc * 512 + r * 16) = 0u;
          }
        }
      }
      if constexpr (!PREORDER) {
        float* sbuf = rbuf + 4 * 8;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          float sm = psum[q];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
          if (lane == q) sbuf[warp * 8 + q] = sm;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_RED));
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_RED), 1, abort_flag, kErrTimeoutSoftmax))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int q = 0; q < G; ++q)
          lp[q] = fmaf(alpha[q], lp[q], (sbuf[q] + sbuf[8 + q]) + (sbuf[16 + q] + sbuf[24 + q]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_PFULL + pb));
      // the previous tile's partials are complete by now: fold them in
      if (j > 0 && !fold(j - 1)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int q = 0; q < G; ++q) {
        m[q] = mnew[q];
        alpha_prev[q] = alpha[q];
      }
    }
    // ------------------------------------------------------------- epilogue ---
    const bool ready = __all_sync(0xffffffffu, ok && ntile > 0) && fold(ntile - 1);
    const int c = t;  // TMEM lane = output channel
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const int hq = h * G + q;
      float* w = p.ws + ((static_cast<int64_t>(b) * p.Hq + hq) * p.splits + sp) * (C::D + 2);
      if (ready) {
        w[c] = acc[q] * kGP;
        if (c == 0) {
          w[C::D] = m[q];
          w[C::D + 1] = PREORDER ? lacc[q] * kGP : lp[q];
        }
      } else if (ntile == 0) {
        // an empty split (never launched by the host) contributes nothing
        if (c == 0) w[C::D] = -INFINITY;
      } else {
        // a wait gave up: poison this warp's channels, so the combine turns
        // them into NaN instead of reading what an earlier call left here
        w[c] = __int_as_float(0x7fc00000);
      }
    }
  }
  if (*abort_flag) drain_after_abort();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_ALLOC);
}

// Merge the splits of each (b, hq): O = sum w_s acc_s / sum w_s l_s with
// w_s = 2^(m_s - max m).  One warp per query row, d = 128 (4 channels/lane).
__global__ void decode_combine_kernel(const float* __restrict__ ws, int rows, int splits, int d, void* o, int o_fp16) {
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* base = ws + static_cast<int64_t>(row) * splits * (d + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, base[s * (d + 2) + d]);
  float den = 0.0f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < splits; ++s) {
    const float* w = base + s * (d + 2);
    const float ms = w[d];
    if (ms == -INFINITY) continue;
    const float wt = exp2f(ms - M);
    den = fmaf(wt, w[d + 1], den);
    for (int i = 0; i < 4; ++i) acc[i] = fmaf(wt, w[lane * 4 + i], acc[i]);
  }
  const float inv = 1.0f / den;
  for (int i = 0; i < 4; ++i) {
    const int64_t off = static_cast<int64_t>(row) * d + lane * 4 + i;
    if (o_fp16) reinterpret_cast<__half*>(o)[off] = __float2half_rn(acc[i] * inv);
    else reinterpret_cast<__nv_bfloat16*>(o)[off] = __float2bfloat16_rn(acc[i] * inv);
  }
}

bool make_tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, int swizzle_bytes);

int decode_default_splits(int B, int Hkv, int kv_len, int block_n) {
  // about three waves of CTAs over 148 SMs (4 resident each), each split
  // keeping at least 16 key tiles to amortize the per-CTA setup and the combine
  const int tiles = (kv_len + block_n - 1) / block_n;
  int splits = 1;
  while (static_cast<int64_t>(B) * Hkv * splits < 3 * 148 * 4 && (tiles / (splits * 2)) >= 16) splits *= 2;
  return splits;
}

template <int FMT, bool PRE, int G>
static hifa4_status launch_decode_t(const uint8_t* kc, const uint8_t* vc, const DecodeParams& p, cudaStream_t st) {
  using C = DecCfg<FMT>;
  CUtensorMap tk, tv;
  const uint64_t Np = static_cast<uint64_t>(p.Np);
  if (!make_tmap_2d(&tk, kc, C::D / 2, static_cast<uint64_t>(p.B) * p.Hkv * Np, C::D / 2, C::BN, C::D / 2) ||
      !make_tmap_2d(&tv, vc, Np / 2, static_cast<uint64_t>(p.B) * p.Hkv * C::D, C::BN / 2, C::D, C::BN / 2)) {
    set_last_error("cuTensorMapEncodeTiled failed");
    return HIFA4_ERR_CUDA;
  }
  auto kern = attn_decode_fp4_kernel<FMT, PRE, G>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  kern<<<static_cast<unsigned>(p.B) * p.Hkv * p.splits, 192, C::SMEM_BYTES, st>>>(tk, tv, p);
  return launch_status("attn_decode");
}

hifa4_status decode_launch(const void* q, int q_dt, const float* s, const uint8_t* kc, const uint8_t* ks,
                           const uint8_t* vc, const uint8_t* vs, int B, int Hq, int Hkv, int kv_len, int kv_cap,
                           int d, int fmt,
                           float softmax_scale, int mode, int block_n, int num_splits, int* num_splits_used,
                           void* workspace, size_t ws_bytes, void* o, int o_dt, float tau, cudaStream_t st) {
  if (num_splits == 0) num_splits = decode_default_splits(B, Hkv, kv_len, block_n);
  const int tiles = (kv_len + block_n - 1) / block_n;
  if (num_splits > tiles) num_splits = tiles;
  const int split_len = ((kv_len + num_splits - 1) / num_splits + block_n - 1) / block_n * block_n;
  const int used = (kv_len + split_len - 1) / split_len;
  if (ws_bytes < static_cast<size_t>(B) * Hq * used * (d + 2) * sizeof(float)) {
    set_last_error("attn_decode: workspace too small (%zu bytes)", ws_bytes);
    return HIFA4_ERR_INVALID_ARG;
  }
  DecodeParams p;
  p.q = q;
  p.s = s;
  p.k_sf = ks;
  p.v_sf = vs;
  p.Np = static_cast<int>(pad128(kv_cap));          // the cache layout's padded length
  p.sf_k_head = static_cast<int64_t>(hifa4_scale_bytes(kv_cap, d, static_cast<hifa4_format>(fmt)));
  p.sf_v_head = static_cast<int64_t>(hifa4_scale_bytes(d, p.Np, static_cast<hifa4_format>(fmt)));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.kv_len = kv_len;
  p.split_len = split_len;
  p.splits = used;
  p.q_fp16 = q_dt == HIFA4_FP16;
  p.c_log2 = softmax_scale * 1.4426950408889634f;
  p.tau = tau;
  p.ws = static_cast<float*>(workspace);
  hifa4_status r = HIFA4_ERR_UNSUPPORTED;
  const bool pre = mode == HIFA4_NORM_PREORDER;
#define HIFA4_DEC_G(GG)                                                                          \
  if (p.G == GG) {                                                                               \
    if (fmt == HIFA4_NVFP4)                                                                      \
      r = pre ? launch_decode_t<HIFA4_NVFP4, true, GG>(kc, vc, p, st)                            \
              : launch_decode_t<HIFA4_NVFP4, false, GG>(kc, vc, p, st);                          \
    else                                                                                         \
      r = pre ? launch_decode_t<HIFA4_MXFP4, true, GG>(kc, vc, p, st)                            \
              : launch_decode_t<HIFA4_MXFP4, false, GG>(kc, vc, p, st);                          \
  }
  HIFA4_DEC_G(1)
  HIFA4_DEC_G(2)
  HIFA4_DEC_G(4)
  HIFA4_DEC_G(8)
#undef HIFA4_DEC_G
  if (r == HIFA4_ERR_UNSUPPORTED) set_last_error("attn_decode: GQA group %d not in {1,2,4,8}", p.G);
  if (r != HIFA4_OK) return r;
  const int rows = B * Hq;
  decode_combine_kernel<<<(rows + 3) / 4, 128, 0, st>>>(p.ws, rows, used, d, o, o_dt == HIFA4_FP16);
  if (num_splits_used) *num_splits_used = used;
  return launch_status("decode_combine");
}

}  // namespace hifa4

// ---------------------------------------------------------------------------
// Decode without any device allocation by the caller.
//
// Some callers cannot call cudaMalloc: an inference-server plugin or a custom
// operator that is handed only its input and output buffers by the host
// framework (whose caching allocator owns all device memory), or a latency-
// critical serving loop where an allocation may block or synchronize the
// device.  hifa4_attn_decode_noalloc serves them: the split partials live in a
// library-owned scratch array in device global memory, declared below.  Every
// GPU that loads this library holds this array until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device

// The scratch itself.  In host code this symbol is only a host-side stand-in
// for the device array: its device address must come from
// cudaGetSymbolAddress on the device in question (see scratch_for_current).
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};   // the context each address belongs to

// cuCtxGetCurrent through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

// Device address of the scratch on the current device.  It is looked up on
// the first call on a device and again whenever the device's context has
// changed since (after cudaDeviceReset, or when a host framework released and
// re-created the primary context, the module and its array are loaded anew).
hifa4_status scratch_for_current(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    hifa4::set_last_error("attn_decode_noalloc: no usable current CUDA device");
    return HIFA4_ERR_CUDA;
  }
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) {
    hifa4::set_last_error("attn_decode_noalloc: cuCtxGetCurrent is not available");
    return HIFA4_ERR_CUDA;
  }
  // null before the runtime has made this device's context current
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev] || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    // (the lookup also makes the device's primary context current)
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      hifa4::set_last_error("attn_decode_noalloc: cudaGetSymbolAddress failed on device %d: %s", dev,
                            cudaGetErrorString(e));
      return HIFA4_ERR_CUDA;
    }
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
      hifa4::set_last_error("attn_decode_noalloc: no current CUDA context on device %d", dev);
      return HIFA4_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return HIFA4_OK;
}

}  // namespace

extern "C" HIFA4_API size_t hifa4_decode_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

extern "C" HIFA4_API hifa4_status hifa4_attn_decode_noalloc(
    const void* q, hifa4_dtype q_dt, const float* s, const uint8_t* k_codes, const uint8_t* k_scales,
    const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int Hq, int Hkv, int kv_len, int d, hifa4_format fmt,
    float softmax_scale, hifa4_norm_mode mode, int block_n, int num_splits, int* num_splits_used, void* o,
    hifa4_dtype o_dt, hifa4_stream_t stream) {
  // Size of the split partials this call needs, computed as the decode does.
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || kv_len <= 0 || d <= 0 || num_splits < 0) {
    hifa4::set_last_error("attn_decode_noalloc: bad shape");
    return HIFA4_ERR_INVALID_ARG;
  }
  const int bn = 128;
  int splits = num_splits == 0 ? hifa4::decode_default_splits(B, Hkv, kv_len, bn) : num_splits;
  const int tiles = (kv_len + bn - 1) / bn;
  if (splits > tiles) splits = tiles;
  const int split_len = ((kv_len + splits - 1) / splits + bn - 1) / bn * bn;
  const int used = (kv_len + split_len - 1) / split_len;
  const size_t need = static_cast<size_t>(B) * Hq * used * (static_cast<size_t>(d) + 2) * sizeof(float);
  if (need > kNoAllocScratchBytes) {
    hifa4::set_last_error(
        "attn_decode_noalloc: this call needs %zu bytes of split scratch but the library-owned scratch holds at "
        "most %zu bytes; lower num_splits or the batch, or use hifa4_attn_decode with a caller workspace",
        need, kNoAllocScratchBytes);
    return HIFA4_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  hifa4_status st = scratch_for_current(&scratch);
  if (st != HIFA4_OK) return st;
  // Every split that completes writes all of its partials before the combine
  // reads them, so the scratch needs no clearing between calls; a split whose
  // bounded wait gave up writes NaN markers instead (the output turns NaN and
  // the device error word is set), never leaving an earlier call's partials
  // to be read as its own.
  return hifa4_attn_decode(q, q_dt, s, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, kv_len, d, fmt,
                           softmax_scale, mode, block_n, num_splits, num_splits_used, scratch, kNoAllocScratchBytes, o,
                           o_dt, stream);
}
