// attn_fwd.cu -- 4-bit FlashAttention forward on sm_100a with Smooth-QK'd,
// block-scaled FP4 operands and P-Reordering.
//
// Method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for
// LLM Inference", Abstract paras 1-2: QK^T and PV are 4-bit GEMMs, the online
// softmax keeps a running max m and normalizer l, the attention weights are
// quantized to P-hat per tile, and under P-Reordering l is accumulated from
// the same P-hat that feeds the PV GEMM, fused into that GEMM.
//
// B200 design (one CTA = one 128-row query tile of one (batch, q head)),
// with NH = 1 or 2 softmax warpgroups per row (1 for 64-key tiles, 2 for
// 128-key tiles; W = 4 * NH softmax warps):
//   warp W      TMA producer: Q-hat tile once, then K-hat / V-hat^T tiles and
//               their tiled scale chunks into an NS-stage ring (mbarriers).
//   warp W+1    MMA issuer (one thread): copies scale chunks shared->TMEM with
//               tcgen05.cp, issues block-scaled tcgen05.mma for S = Q K^T
//               into a TMEM S buffer, and for O += P-hat V-hat plus
//               L += P-hat * ones (the fused normalizer: a 16-row all-ones B
//               tile, so column 0 of L is sum(P-hat) with the same P-hat
//               codes and scales as O).  Completion is signalled with
//               tcgen05.commit onto mbarriers.
//   warps 0..W-1 softmax: thread (h, r) owns TMEM lane r (query row r) and
//               the h-th of NH column slices of S, P-hat and O; with NH = 2
//               the row max is exchanged in shared memory.  Per key tile:
//               tcgen05.ld the S row, block maxima, online max, block scales,
//               P = 2^(S*c - m) and its E2M1 codes in registers, codes stored
//               swizzled into shared memory as the A operand of the PV MMA,
//               scales into a TMEM-copy chunk; when m rises, rescale the row
//               of O and L in TMEM (after the previous PV MMA retired).
//               Epilogue: O / l, lse, optional debug sums.
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "quant_rules.cuh"

// Tuning knobs (measured on the 32-head, 4096-token causal prefill):
// element pairs (of every eight pairs) whose 2^y (or code argument) runs on
// the FMA pipe instead of MUFU (-1: 2 at d <= 128 and 1 at d = 256, the
// fastest of 0..3 for each), and softmax warpgroups per row for 64-key tiles.
#ifndef HIFA4_POLY_PAIRS
#define HIFA4_POLY_PAIRS -1
#endif
// 1: where only the P-hat codes are needed (P-Reordering without the debug
// sums), those FMA-pipe pairs take the exponential-free code argument
// instead of 2^y; 0: 2^y by the polynomial everywhere
#ifndef HIFA4_CODE_MAP
#define HIFA4_CODE_MAP 1
#endif
// 1: where only the P-hat codes are needed, P = 2^(S*c - m) is formed first
// and multiplied by the block multiplier afterwards (the exponentials then
// need only the row max, not the block scales); 0: the multiplier is folded
// into the exponent; -1: per shape (measured: first at d = 256, 1.024 times
// faster; folded at d = 128, 1.03 times faster)
#ifndef HIFA4_EXP_FIRST
#define HIFA4_EXP_FIRST -1
#endif
#ifndef HIFA4_ATTN_NH_BN64
#define HIFA4_ATTN_NH_BN64 1
#endif
// with one softmax warpgroup per row: a correction warpgroup rescales O
// 1: a softmax warp that does not rescale O in tile j waits for no PV
// product (the S_j wait already covers PV_{j-2}, the last reader of the P-hat
// buffer it is about to overwrite); one that rescales waits for PV_{j-1}.
// 0: every tile waits for PV_{j-1}.
#ifndef HIFA4_RELAX_PV
#define HIFA4_RELAX_PV 1
#endif
// 1: with three or more K/V stages, a key tile's K-hat and V-hat^T copies
// (with their scales) complete on one barrier per stage, awaited once by the
// MMA issuer before S_j (measured 1.2 % faster at d = 128; with two stages,
// d = 256, S_j would wait for V_j's stage and it is 10 % slower); 0: one
// barrier each, V's awaited before PV_j.
#ifndef HIFA4_KV_ONE_BAR
#define HIFA4_KV_ONE_BAR 1
#endif
#ifndef HIFA4_ATTN_CORR
#define HIFA4_ATTN_CORR 0
#endif
// 1: two MMA-issuing warps, one for S = Q K^T and one for O += P V, so that
// the next tile's S never queues behind the previous tile's PV issue
#ifndef HIFA4_TWO_ISSUERS
#define HIFA4_TWO_ISSUERS 0
#endif

namespace hifa4 {

struct AttnParams {
  // Q in its input dtype ([B][Hq][N][d]) and the Smooth-QK scales s ([Hkv][d],
  // or null): the softmax warps scale and quantize their query tile in the
  // kernel (the fused path); null: Q-hat comes from q codes / q_sf.
  const void* q_raw;
  const float* q_s;
  int q_fp16;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  int64_t sf_qk_head;   // bytes of one head's Q/K scale matrix
  int64_t sf_v_head;    // bytes of one head's V^T scale matrix
  int B, Hq, Hkv, N, Np, G;
  int num_qtiles;
  float c_log2;         // softmax_scale * log2(e)
  float tau;            // rescale threshold (log2 units); 0 = exact running max
  int causal;
  int out_fp16;
  void* o;
  float* lse;
  float* dbg_l_phat;
  float* dbg_l_p;
  AttnDump dump;        // all null unless hifa4_attn_fwd_dump
  const float* qk_bias; // [B*Hq][Np]: the Q-Mean term mu . K-hat per key, or null
  int nkt_all;          // key tiles of a whole row, ceil(N / BN): the dump's tile stride
};

template <int D, int BN, int FMT>
struct AttnCfg {
  static constexpr int BETA = FMT == HIFA4_NVFP4 ? 16 : 32;
  static constexpr int BM = 128;
  // softmax warpgroups per query row: 2 split each row's key columns (and O
  // columns) between two warpgroups, 1 gives each thread a whole row
  static constexpr int NH = BN == 64 ? HIFA4_ATTN_NH_BN64 : 2;
  // correction warps (4, one per TMEM lane quadrant) rescale the O rows
  // when the running max rises, off the softmax warps' path
  static constexpr int CORR = (NH == 1 && HIFA4_ATTN_CORR) ? 1 : 0;
  static constexpr int NS = D == 256 ? 2 : 3;               // K/V pipeline stages
  static constexpr bool KV_ONE = HIFA4_KV_ONE_BAR && NS >= 3;  // one full barrier per K/V stage
  static constexpr int QROW = D / 2;                        // bytes per Q/K row
  static constexpr int PROW = BN / 2;                       // bytes per P-hat / V^T row
  static constexpr int KSTEPS_S = D / 64;
  static constexpr int KSTEPS_P = BN / 64;
  static constexpr int NKC_Q = (D / BETA + 3) / 4;          // scale chunks per Q/K row group
  static constexpr int NRG_V = (D + 127) / 128;             // 128-row groups of V^T
  // The fused normalizer's 16 all-ones rows follow the V^T rows of every V
  // stage, so one MMA of N = D + 16 writes O and L; otherwise a second
  // N = 16 MMA reads a separate ones tile.
  // (D a multiple of 128 keeps the ones rows in a scale row group of their
  // own; with D = 64 they would fall among V's zero-padded scale rows)
  static constexpr bool FUSE_L = D == 128;
  static constexpr int NRG_B = NRG_V + (FUSE_L ? 1 : 0);    // B-operand row groups of the PV MMA
  static constexpr int NCH_V = (BN / BETA + 3) / 4;         // V^T scale chunks per tile per row group
  static constexpr int NKC_P = (BN / BETA + 3) / 4;         // P-hat scale chunks per tile
  // TMEM columns with `nsb` S buffers: S, O, L (16), scale regions.
  static constexpr int cols(int nsb) {
    return nsb * BN + D + 16 + 8 * NKC_Q + 4 * NKC_P + 4 * NCH_V * NRG_B + (FUSE_L ? 0 : 4);
  }
  // Prefer a footprint of 256 columns so that two CTAs share an SM (twice the
  // softmax warps per scheduler); otherwise own all 512 columns.
  static constexpr int NSB = cols(2) <= 256 ? 2 : (cols(1) <= 256 ? 1 : (cols(2) <= 512 ? 2 : 1));
  static constexpr int TMEM_ALLOC = cols(NSB) <= 256 ? 256 : 512;
  static constexpr int CTAS_PER_SM = TMEM_ALLOC == 256 ? 2 : 1;
  // a second MMA-issuing warp where the register file allows it (two CTAs of
  // two softmax warpgroups each would leave too few registers per thread)
  static constexpr int TWO_ISSUERS = (HIFA4_TWO_ISSUERS && (NH == 1 || CTAS_PER_SM == 1)) ? 1 : 0;
  static constexpr int WARP_TMA = 4 * NH + 4 * CORR;
  static constexpr int WARP_MMA = WARP_TMA + 1;             // issues S (and PV with one issuer)
  static constexpr int WARP_PV = WARP_MMA + TWO_ISSUERS;     // issues PV
  static constexpr int NTHREADS = 32 * (WARP_PV + 1);
  // shared memory layout (byte offsets; operand tiles 1024-aligned)
  static constexpr int SZ_Q = BM * QROW;
  static constexpr int SZ_K = BN * QROW;
  static constexpr int SZ_V = D * PROW;
  static constexpr int SZ_P = BM * PROW;
  static constexpr int SZ_ONES = 16 * PROW;
  static constexpr int SZ_VX = SZ_V + (FUSE_L ? SZ_ONES : 0);   // a V stage: the V^T tile, then the ones rows
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + SZ_Q;
  static constexpr int OFF_V = OFF_K + NS * SZ_K;
  static constexpr int OFF_P = OFF_V + NS * SZ_VX;
  static constexpr int OFF_ONES = OFF_P + 2 * SZ_P;
  static constexpr int OFF_QSF = (OFF_ONES + SZ_ONES + 1023) / 1024 * 1024;
  static constexpr int OFF_KSF = OFF_QSF + NKC_Q * 512;
  static constexpr int OFF_VSF = OFF_KSF + NS * NKC_Q * 512;
  static constexpr int OFF_PSF = OFF_VSF + NS * NRG_V * NCH_V * 512;
  static constexpr int OFF_ONESF = OFF_PSF + 2 * NKC_P * 512;
  static constexpr int OFF_INV = OFF_ONESF + 512;           // 128 floats: 1/scale per UE4M3 code
  static constexpr int OFF_LOG = OFF_INV + 512;             // 128 floats: log2 of the above
  static constexpr int OFF_XM = OFF_LOG + 512;              // row-max exchange [2][2][128] floats, or
                                                            // the correction warps' alpha [3][128]
  static constexpr int OFF_LP = OFF_XM + 2048;              // normalizer exchange [2][128] floats
  static constexpr int OFF_BIAS = OFF_LP + 1024;            // Q-Mean score term per key: [NS][BN] floats
  static constexpr int OFF_BAR = OFF_BIAS + NS * BN * 4;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
  // s_full[NSB], s_empty[NSB], p_full[2], p_empty[2], o_ready
  static constexpr int NBAR = 1 + 4 * NS + 2 * NSB + 4 + 1 + 3 + 24 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr int TM_S = 0;
  static constexpr int TM_O = NSB * BN;
  static constexpr int TM_L = TM_O + D;
  static constexpr int TM_SFA_Q = TM_L + 16;
  static constexpr int TM_SFB_K = TM_SFA_Q + 4 * NKC_Q;
  static constexpr int TM_SFA_P = TM_SFB_K + 4 * NKC_Q;
  static constexpr int TM_SFB_V = TM_SFA_P + 4 * NKC_P;
  // V^T scale chunk (lc, row group rg) at TM_SFB_V + 4 * (lc * NRG_B + rg);
  // with FUSE_L, group NRG_V of every chunk holds the ones rows' scales
  static constexpr int TM_SFB_1 = TM_SFB_V + 4 * NCH_V * NRG_B;
  static constexpr int TM_COLS_USED = TM_SFB_1 + (FUSE_L ? 0 : 4);
  static_assert(TM_COLS_USED <= TMEM_ALLOC, "TMEM budget");
  // Dynamic shared memory requested: enough that at most CTAS_PER_SM CTAs are
  // resident (a further CTA would stall in tcgen05.alloc).
  static constexpr int SMEM_REQ = CTAS_PER_SM == 1 ? (SMEM_BYTES > 116 * 1024 ? SMEM_BYTES : 116 * 1024)
                                                   : (SMEM_BYTES > 80 * 1024 ? SMEM_BYTES : 80 * 1024);
  static_assert(CTAS_PER_SM == 1 || SMEM_REQ <= 112 * 1024, "two CTAs per SM must fit");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Reductions as shallow trees (3-input max), not dependent chains.
template <int N>
__device__ __forceinline__ float tree_max(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return fmaxf(v[0], v[1]);
  } else {
    constexpr int M = (N + 2) / 3;
    float t[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
      const int a = 3 * i;
      if (a + 2 < N) t[i] = fmax3(v[a], v[a + 1], v[a + 2]);
      else if (a + 1 < N) t[i] = fmaxf(v[a], v[a + 1]);
      else t[i] = v[a];
    }
    return tree_max<M>(t);
  }
}
template <int N>
__device__ __forceinline__ float tree_sum(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else {
    float t[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) t[i] = v[2 * i] + v[2 * i + 1];
    return tree_sum<N / 2>(t);
  }
}

__device__ __forceinline__ uint32_t swz_chunk(uint32_t r, uint32_t c, uint32_t row_bytes) {
  // physical 16-byte chunk of logical chunk c in row r under the swizzle that
  // matches row_bytes (32/64/128); buffers are 1024-byte aligned.
  return c ^ ((r * row_bytes >> 7) & (row_bytes / 16 - 1));
}

// Scale this warp's 32 TMEM lanes of an HD-column O slice (and, with_l, the
// L column) by alpha: chunks of at most 64 columns, one TMEM round trip each,
// L riding along with the first.  The caller waits for the stores.
template <int HD>
__device__ __forceinline__ void rescale_o_rows(uint32_t a0, uint32_t al, bool with_l_slice, float alpha) {
  constexpr int RC = HD < 64 ? HD : 64;
  static_assert(RC == 32 || RC == 64, "O slice chunks of 32 or 64 columns");
  const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
  for (int cc = 0; cc < HD / RC; ++cc) {
    uint32_t v[RC];
    uint32_t lv = 0;
    const bool with_l = with_l_slice && cc == 0;
    if (with_l) {
      if constexpr (RC == 64) tmem_ld64_and1_wait(a0 + cc * RC, v, al, lv);
      else tmem_ld32_and1_wait(a0 + cc * RC, v, al, lv);
    } else {
      if constexpr (RC == 64) tmem_ld64_wait(a0 + cc * RC, v);
      else tmem_ld32_wait(a0 + cc * RC, v);
    }
#pragma unroll
    for (int i = 0; i < RC; i += 2) {
      const float2 t0 = fmul2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), a2);
      v[i] = __float_as_uint(t0.x);
      v[i + 1] = __float_as_uint(t0.y);
    }
    if constexpr (RC == 64) tmem_st64(a0 + cc * RC, v);
    else tmem_st32(a0 + cc * RC, v);
    if (with_l) tmem_st1(al, __float_as_uint(__uint_as_float(lv) * alpha));
  }
}

template <int D, int BN, int FMT, bool PREORDER, bool EXT>
__global__ void __launch_bounds__(AttnCfg<D, BN, FMT>::NTHREADS, AttnCfg<D, BN, FMT>::CTAS_PER_SM)
    attn_fwd_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D, BN, FMT>;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t bar0 = smem_u32(bars);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NS, B_VFULL = 1 + 2 * C::NS, B_VEMPTY = 1 + 3 * C::NS,
            B_SFULL = 1 + 4 * C::NS, B_SEMPTY = B_SFULL + C::NSB, B_PFULL = B_SEMPTY + C::NSB,
            B_PEMPTY = B_PFULL + 2, B_ORDY = B_PEMPTY + 2, B_XM = B_ORDY + 1, B_EP1 = B_XM + 1, B_EP2 = B_EP1 + 1,
            B_AF = B_EP2 + 1,   // [quadrant][4]: softmax warp -> correction warp, alpha of tile j ready
            B_OC = B_AF + 16,   // [quadrant][2]: correction warp -> MMA, O rescaled for PV_j
            B_XQ = B_OC + 8;    // [quadrant]: row-max exchange of the two warps sharing a lane quadrant
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  // ---- work item: heavy (late) query tiles first for causal balance ----
  const int bhq = blockIdx.x % (p.B * p.Hq);
  const int qtile = p.num_qtiles - 1 - static_cast<int>(blockIdx.x / (p.B * p.Hq));
  const int b = bhq / p.Hq, hq = bhq % p.Hq;
  const int kvbh = b * p.Hkv + hq / p.G;
  const int row0 = qtile * C::BM;
  const int kv_end = p.causal ? min(p.N, row0 + C::BM) : p.N;
  const int nkt = (kv_end + BN - 1) / BN;
  // Q-Mean auxiliary: add the score term mu . K-hat of each key (EXT only;
  // needs the single K/V barrier per stage, d <= 128)
  const bool qbias = EXT && C::KV_ONE && p.qk_bias != nullptr;

  // ---- setup ----
  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), p.q_raw != nullptr ? 4 * C::NH : 1);   // fused: one arrival per softmax warp
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_KEMPTY + s), 1);
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_VEMPTY + s), 1);
    }
    for (int s = 0; s < C::NSB; ++s) {
      mbar_init(BAR(B_SFULL + s), 1);
      mbar_init(BAR(B_SEMPTY + s), 4 * C::NH);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(B_PFULL + s), 4 * C::NH);
      mbar_init(BAR(B_PEMPTY + s), 1);
    }
    mbar_init(BAR(B_XM), 8);      // (unused: the exchange is per lane quadrant, below)
    for (int q = 0; q < 4; ++q) mbar_init(BAR(B_XQ + q), 2);   // the two warps of quadrant q
    mbar_init(BAR(B_EP1), 4);     // epilogue: half 1 -> half 0
    mbar_init(BAR(B_EP2), 4);     // epilogue: half 0 -> half 1
    for (int i = 0; i < 24; ++i) mbar_init(BAR(B_AF + i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // constant operands of the fused normalizer: 16 rows of E2M1 1.0 (code 2)
  // and their scale chunk (scale 1.0 for rows 0..15 in every block byte).
  for (int i = threadIdx.x; i < C::SZ_ONES / 4; i += blockDim.x) {
    reinterpret_cast<uint32_t*>(smem + C::OFF_ONES)[i] = 0x22222222u;
    if constexpr (C::FUSE_L)
      for (int st = 0; st < C::NS; ++st)
        reinterpret_cast<uint32_t*>(smem + C::OFF_V + st * C::SZ_VX + C::SZ_V)[i] = 0x22222222u;
  }
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    const uint32_t one = FMT == HIFA4_NVFP4 ? 0x38u : 0x7Fu;
    // word i of the chunk sits at byte 4*i: line (i/4) = row%32, word (i%4) = row/32
    const int row_of_word = (i >> 2) + 32 * (i & 3);
    reinterpret_cast<uint32_t*>(smem + C::OFF_ONESF)[i] = row_of_word < 16 ? one * 0x01010101u : 0u;
    // fl32(1 / (UE4M3(i) * g_P)), the P-hat element multiplier of scale code i
    const float sd = __fmul_rn(ue4m3_to_f32(i), FMT == HIFA4_NVFP4 ? 0.00390625f : 1.0f);
    const float inv = i == 0 ? 0.0f : __fdiv_rn(1.0f, sd);
    reinterpret_cast<float*>(smem + C::OFF_INV)[i] = inv;
    reinterpret_cast<float*>(smem + C::OFF_LOG)[i] = i == 0 ? -INFINITY : log2f(inv);
  }
  // fused path: the Smooth-QK scales of this head's kv group, staged in the
  // normalizer-exchange area (free until the epilogue)
  if (p.q_raw != nullptr && p.q_s != nullptr)
    for (int i = threadIdx.x; i < D; i += blockDim.x)
      reinterpret_cast<float*>(smem + C::OFF_LP)[i] = p.q_s[static_cast<int64_t>(hq / p.G) * D + i];
  fence_proxy_async_smem();
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  if (warp == C::WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::WARP_TMA) {
    // =============================== TMA producer ===============================
    if (lane == 0) {
      if (p.q_raw == nullptr) {
        const uint8_t* qsf = p.q_sf + static_cast<int64_t>(bhq) * p.sf_qk_head + static_cast<int64_t>(qtile) * C::NKC_Q * 512;
        mbar_arrive_expect_tx(BAR(B_QFULL), C::SZ_Q + C::NKC_Q * 512);
        tma_load_2d(sbase + C::OFF_Q, &tm_q, 0, bhq * p.Np + row0, BAR(B_QFULL));
        bulk_load(sbase + C::OFF_QSF, qsf, C::NKC_Q * 512, BAR(B_QFULL));
      }
      const int nkc_v_row = p.Np / (4 * C::BETA);  // V^T scale chunks per row group
      for (int j = 0; j < nkt; ++j) {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait(BAR(B_KEMPTY + st), ph ^ 1, abort_flag, kErrTimeoutTma)) break;
        // with one barrier per stage it expects the V copies' bytes too (and
        // the Q-Mean score terms of the tile's keys)
        mbar_arrive_expect_tx(BAR(B_KFULL + st), C::SZ_K + C::NKC_Q * 512 +
                                                     (C::KV_ONE ? C::SZ_V + C::NRG_V * C::NCH_V * 512 : 0) +
                                                     (C::KV_ONE && qbias ? BN * 4 : 0));
        tma_load_2d(sbase + C::OFF_K + st * C::SZ_K, &tm_k, 0, kvbh * p.Np + j * BN, BAR(B_KFULL + st));
        bulk_load(sbase + C::OFF_KSF + st * C::NKC_Q * 512,
                  p.k_sf + static_cast<int64_t>(kvbh) * p.sf_qk_head + static_cast<int64_t>((j * BN) >> 7) * C::NKC_Q * 512,
                  C::NKC_Q * 512, BAR(B_KFULL + st));
        if (!mbar_wait(BAR(B_VEMPTY + st), ph ^ 1, abort_flag, kErrTimeoutTma)) break;
        const uint32_t vbar = BAR((C::KV_ONE ? B_KFULL : B_VFULL) + st);
        if (!C::KV_ONE) mbar_arrive_expect_tx(vbar, C::SZ_V + C::NRG_V * C::NCH_V * 512);
        tma_load_2d(sbase + C::OFF_V + st * C::SZ_VX, &tm_v, j * C::PROW, kvbh * D, vbar);
        // the tile's Q-Mean score terms go with V: stage st is free once PV of
        // its previous tile retired, which the softmax warps' use precedes
        if (C::KV_ONE && qbias)
          bulk_load(sbase + C::OFF_BIAS + st * BN * 4, p.qk_bias + static_cast<int64_t>(bhq) * p.Np + j * BN, BN * 4,
                    vbar);
        const int chunk0 = (j * BN) / (4 * C::BETA);
        for (int rg = 0; rg < C::NRG_V; ++rg)
          bulk_load(sbase + C::OFF_VSF + (st * C::NRG_V + rg) * C::NCH_V * 512,
                    p.v_sf + static_cast<int64_t>(kvbh) * p.sf_v_head + static_cast<int64_t>(rg * nkc_v_row + chunk0) * 512,
                    C::NCH_V * 512, vbar);
      }
    }
  } else if (warp == C::WARP_MMA || warp == C::WARP_PV) {
    // ================================ MMA issuers ================================
    // With two issuers, warp WARP_MMA issues every S = Q K_j^T as soon as its
    // K tile has landed and the S buffer is free, and warp WARP_PV every
    // O += P-hat V_j as soon as P-hat_j is written; they touch disjoint TMEM
    // columns and shared memory.  With one, WARP_MMA interleaves both.
    const bool s_role = warp == C::WARP_MMA;
    const bool pv_role = warp == C::WARP_PV;
    if (lane == 0) {
      constexpr bool MX = FMT == HIFA4_MXFP4;
      auto mma = [&](uint32_t d_t, uint64_t a, uint64_t bdesc, uint32_t idesc, uint32_t sfa, uint32_t sfb, uint32_t acc) {
        if constexpr (MX) mma_mxfp4(d_t, a, bdesc, idesc, sfa, sfb, acc);
        else mma_nvfp4(d_t, a, bdesc, idesc, sfa, sfb, acc);
      };
      bool ok = true;
      if (s_role) {
        ok = mbar_wait(BAR(B_QFULL), 0, abort_flag, kErrTimeoutMma);
        if (ok) {
          tc_fence_after();
          for (int kc = 0; kc < C::NKC_Q; ++kc)
            tc_cp_32x128b_warpx4(tmem + C::TM_SFA_Q + 4 * kc, make_sf_desc(sbase + C::OFF_QSF + kc * 512));
        }
      }
      if (pv_role) {
        // scales of the fused normalizer's ones rows (constant, written at setup)
        if constexpr (C::FUSE_L) {
          for (int lc = 0; lc < C::NCH_V; ++lc)
            tc_cp_32x128b_warpx4(tmem + C::TM_SFB_V + 4 * (lc * C::NRG_B + C::NRG_V),
                                 make_sf_desc(sbase + C::OFF_ONESF));
        } else {
          tc_cp_32x128b_warpx4(tmem + C::TM_SFB_1, make_sf_desc(sbase + C::OFF_ONESF));
        }
      }
      // S_j = Q K_j^T into S buffer j % NSB
      auto issue_s = [&](int j) -> bool {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        const int sb = j % C::NSB;
        if (!mbar_wait(BAR(B_KFULL + st), ph, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
        // 64-key tiles: a 128-row chunk of K scales serves tiles 2i and 2i+1,
        // so it is copied on even tiles only (the copy of tile 2i+2 is issued
        // after, and so executes after, the MMAs of tile 2i+1).  It needs only
        // the K tile, so it goes before the wait for the S buffer.
        if (!(BN == 64 && (j & 1)))
          for (int kc = 0; kc < C::NKC_Q; ++kc)
            tc_cp_32x128b_warpx4(tmem + C::TM_SFB_K + 4 * kc,
                                 make_sf_desc(sbase + C::OFF_KSF + st * C::NKC_Q * 512 + kc * 512));
        if (!mbar_wait(BAR(B_SEMPTY + sb), ((j / C::NSB) & 1) ^ 1, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t half_off = (BN == 64 && (j & 1)) ? 2u : 0u;  // rows 64..127 of the K row group
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS_S; ++ks) {
          const uint32_t chunk = MX ? ks / 2 : ks;
          const uint32_t byte = MX ? 2 * (ks % 2) : 0;
          const uint64_t a = make_kmajor_desc(sbase + C::OFF_Q + ks * 32, C::QROW);
          const uint64_t bd = make_kmajor_desc(sbase + C::OFF_K + st * C::SZ_K + ks * 32, C::QROW);
          const uint32_t idesc = idesc_fp4(128, BN, MX, byte, byte);
          mma(tmem + C::TM_S + sb * BN, a, bd, idesc, (tmem + C::TM_SFA_Q + 4 * chunk) | (byte << 30),
              (tmem + C::TM_SFB_K + 4 * chunk + half_off) | (byte << 30), ks > 0 ? 1u : 0u);
        }
        tc_commit(BAR(B_SFULL + sb));
        tc_commit(BAR(B_KEMPTY + st));
        return true;
      };
      // O += P-hat V-hat_j ; L += P-hat ones (the same MMA when FUSE_L)
      auto issue_pv = [&](int j) -> bool {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        const int pb = j & 1;
        // V_j landed: with one barrier per stage the S_j wait covered it (S_j
        // is issued first by the same thread), unless a second thread issues PV
        if (!C::KV_ONE || C::TWO_ISSUERS)
          if (!mbar_wait(BAR((C::KV_ONE ? B_KFULL : B_VFULL) + st), ph, abort_flag, kErrTimeoutMma)) return false;
        tc_fence_after();
        // V_j's scales need only V_j: copied before the wait for P-hat_j (the
        // copy executes after PV_{j-1}, issued earlier by this thread)
        for (int lc = 0; lc < C::NCH_V; ++lc)
          for (int rg = 0; rg < C::NRG_V; ++rg)
            tc_cp_32x128b_warpx4(tmem + C::TM_SFB_V + 4 * (lc * C::NRG_B + rg),
                                 make_sf_desc(sbase + C::OFF_VSF + ((st * C::NRG_V + rg) * C::NCH_V + lc) * 512));
        if (!mbar_wait(BAR(B_PFULL + pb), (j >> 1) & 1, abort_flag, kErrTimeoutMma)) return false;
        if constexpr (C::CORR) {
          // O (and L) rescaled for this tile's max by every lane quadrant
          // (tile j >= 1 is phase (j-1)/2 of barrier (j-1)%2: the correction
          // warps run at most two tiles ahead of this wait)
          if (j > 0)
            for (int q = 0; q < 4; ++q)
              if (!mbar_wait(BAR(B_OC + 2 * q + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag, kErrTimeoutMma))
                return false;
        }
        tc_fence_after();
        for (int pc = 0; pc < C::NKC_P; ++pc)
          tc_cp_32x128b_warpx4(tmem + C::TM_SFA_P + 4 * pc,
                               make_sf_desc(sbase + C::OFF_PSF + pb * C::NKC_P * 512 + pc * 512));
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS_P; ++ks) {
          const int kk = j * BN + ks * 64;                        // first key of this K-step
          const uint32_t pchunk = MX ? ks / 2 : ks;
          const uint32_t pbyte = MX ? 2 * (ks % 2) : 0;
          const uint32_t vchunk = kk / (4 * C::BETA) - (j * BN) / (4 * C::BETA);
          const uint32_t vbyte = (kk / C::BETA) % 4;
          const uint64_t a = make_kmajor_desc(sbase + C::OFF_P + pb * C::SZ_P + ks * 32, C::PROW);
          const uint64_t bv = make_kmajor_desc(sbase + C::OFF_V + st * C::SZ_VX + ks * 32, C::PROW);
          const uint32_t acc = (j > 0 || ks > 0) ? 1u : 0u;
          const uint32_t sfa = (tmem + C::TM_SFA_P + 4 * pchunk) | (pbyte << 30);
          if constexpr (C::FUSE_L) {
            // B = [V^T tile; 16 ones rows]: columns D..D+15 of the result, L,
            // follow O in TMEM
            mma(tmem + C::TM_O, a, bv, idesc_fp4(128, D + 16, MX, pbyte, vbyte), sfa,
                (tmem + C::TM_SFB_V + 4 * vchunk * C::NRG_B) | (vbyte << 30), acc);
          } else {
            mma(tmem + C::TM_O, a, bv, idesc_fp4(128, D, MX, pbyte, vbyte), sfa,
                (tmem + C::TM_SFB_V + 4 * vchunk * C::NRG_B) | (vbyte << 30), acc);
            const uint64_t b1 = make_kmajor_desc(sbase + C::OFF_ONES + ks * 32, C::PROW);
            mma(tmem + C::TM_L, a, b1, idesc_fp4(128, 16, MX, pbyte, pbyte), sfa,
                (tmem + C::TM_SFB_1) | (pbyte << 30), acc);
          }
        }
        tc_commit(BAR(B_VEMPTY + st));
        tc_commit(BAR(B_PEMPTY + pb));
        return true;
      };
      if constexpr (C::TWO_ISSUERS) {
        if (s_role)
          for (int j = 0; ok && j < nkt; ++j) ok = issue_s(j);
        else
          for (int j = 0; ok && j < nkt; ++j) ok = issue_pv(j);
      } else {
        if (ok && nkt > 0) ok = issue_s(0);
        for (int j = 0; ok && j < nkt; ++j) {
          if (j + 1 < nkt) ok = issue_s(j + 1);
          if (ok) ok = issue_pv(j);
        }
      }
      if (!ok) drain_after_abort();
    }
  } else if (C::CORR && warp >= 4) {
    // ================================ correction ================================
    // Warp 4+q owns TMEM lanes [32q, 32q+32).  For every key tile j >= 1 it
    // takes alpha_j = 2^(m_{j-1} - m_j) of its rows from the softmax warp of
    // the same quadrant and, when any of them is below 1, scales those rows of
    // O and L after PV_{j-1} retired; PV_j waits for it.
    const int q = warp - 4;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float* xa = reinterpret_cast<const float*>(smem + C::OFF_XM);
    bool ok = true;
    for (int j = 1; j < nkt && ok; ++j) {
      // tile j's alpha is phase (j-1)/4 of barrier (j-1)%4 of this quadrant
      // (the softmax warp runs at most two tiles ahead: its tile j+3 waits for
      // PV_{j+1}, which waits for this warp's tile j+1)
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_AF + 4 * q + ((j - 1) & 3)), ((j - 1) >> 2) & 1, abort_flag,
                                             kErrTimeoutSoftmax))) {
        ok = false;
        break;
      }
      const float alpha = xa[(j % 3) * 128 + r];
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        // PV_{j-1} retired (its P-hat buffer's earlier phase is known complete)
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_PEMPTY + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag,
                                               kErrTimeoutSoftmax))) {
          ok = false;
          break;
        }
        tc_fence_after();
        rescale_o_rows<D>(tmem + lane_base + C::TM_O, tmem + lane_base + C::TM_L, true, alpha);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_OC + 2 * q + ((j - 1) & 1)));
    }
  } else {
    // ================================== softmax ==================================
    // Two warpgroups share each query row: thread (hw, r) owns TMEM lane r,
    // key columns [hw*BN/2, (hw+1)*BN/2) of S and P-hat, and output columns
    // [hw*D/2, (hw+1)*D/2) of O.  The row maximum is exchanged through
    // shared memory once per key tile.
    constexpr int HB = BN / C::NH;                   // key columns per thread
    constexpr int HD = D / C::NH;                    // output columns per thread
    constexpr int NBH = HB / C::BETA;                // P-hat blocks per thread
    const int hw = warp >> 2;                        // column half
    const int r = threadIdx.x & 127;                 // row == TMEM lane
    const int row = row0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c = p.c_log2;
    float m = -INFINITY;
    float l_p = 0.0f;
    // the running sum of P: the normalizer of the inconsistent mode, else a
    // debug output only (its pointers reach the EXT instantiation alone).  At
    // d = 256 the production kernel knows at compile time that it forms no
    // sum (measured 1.7 % faster); at d <= 128 the runtime test schedules
    // better (1.3 % faster), although the pointer is always null there.
    const bool want_lp = !PREORDER || ((EXT || D != 256) && (p.dbg_l_p != nullptr || (EXT && p.dump.sum_p != nullptr)));
    constexpr float kGP = FMT == HIFA4_NVFP4 ? 0.00390625f : 1.0f;   // g_P = 2^-8 (NVFP4)
    // pairs (of every eight) whose 2^y runs on the FMA pipe instead of MUFU
    constexpr int kPolyPairs = HIFA4_POLY_PAIRS >= 0 ? HIFA4_POLY_PAIRS : (D == 256 ? 1 : 2);
    const float* inv_tab = reinterpret_cast<const float*>(smem + C::OFF_INV);
    const float* log_tab = reinterpret_cast<const float*>(smem + C::OFF_LOG);
    float* xm = reinterpret_cast<float*>(smem + C::OFF_XM);  // [2 parities][2 halves][128]
    if (p.q_raw != nullptr) {
      // Fused Smooth-QK + Q quantization: thread (hw, r) scales and quantizes
      // its share of row r of the query tile by the rules of the quantize
      // kernel (shared code), and writes the codes and scale bytes where the
      // tensor copy would have put them (the swizzled Q tile, the 512-byte
      // scale chunks).  Rows past N quantize zeros.
      constexpr int NBQ = D / C::BETA;               // blocks per Q row
      constexpr int NBQT = NBQ / C::NH;              // this thread's blocks
      constexpr int NCH = NBQT * C::BETA / 8;        // its 16-byte chunks of the row
      const float* srow = p.q_s != nullptr ? reinterpret_cast<const float*>(smem + C::OFF_LP) : nullptr;
      unsigned char* qrow = smem + C::OFF_Q + r * C::QROW;
      unsigned char* qsfb = smem + C::OFF_QSF + (r & 31) * 16 + (r >> 5) * 4;
      // all of the thread's loads in flight at once (one memory latency)
      uint4 raw[NCH];
      {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q_raw) +
                                                          (static_cast<int64_t>(bhq) * p.N + row) * D +
                                                          hw * NBQT * C::BETA);
#pragma unroll
        for (int i = 0; i < NCH; ++i) raw[i] = row < p.N ? src[i] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int bt = 0; bt < NBQT; ++bt) {
        const int bq = hw * NBQT + bt;
        float v[C::BETA];
#pragma unroll
        for (int k8 = 0; k8 < C::BETA / 8; ++k8) {
          const uint4 u = raw[bt * (C::BETA / 8) + k8];
          const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float2 f;
            if (p.q_fp16) f = __half22float2(*reinterpret_cast<const __half2*>(&wd[e2]));
            else f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[e2]));
            const int e = 8 * k8 + 2 * e2;
            v[e] = srow != nullptr ? __fmul_rn(f.x, srow[bq * C::BETA + e]) : f.x;
            v[e + 1] = srow != nullptr ? __fmul_rn(f.y, srow[bq * C::BETA + e + 1]) : f.y;
          }
        }
        uint32_t packed[C::BETA / 8];
        // the shared table holds 1/(scale * g_P) for P-hat: take g_P = 2^-8 back out
        const uint32_t sc = quant_block<FMT, C::BETA, FMT == HIFA4_NVFP4 ? 8 : 0>(v, packed, inv_tab);
        const int byte0 = bq * (C::BETA / 2);        // first code byte of the block in the row
        unsigned char* dst = qrow + swz_chunk(r, byte0 / 16, C::QROW) * 16 + (byte0 % 16);
        if constexpr (C::BETA == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        qsfb[(bq / 4) * 512 + (bq % 4)] = static_cast<unsigned char>(sc);
      }
      if (NBQ < 4 && hw == C::NH - 1)
        for (int bb = NBQ; bb < 4; ++bb) qsfb[bb] = 0;   // the row's only scale word: unused bytes
      fence_proxy_async_smem();                          // codes and scales are read by the MMA
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_QFULL));
    }
    bool ok = true;
    for (int j = 0; j < nkt && ok; ++j) {
      const int sb = j % C::NSB;
      const int pb = j & 1;
      // A failed wait (a timeout, or another role's abort) only clears ok: the
      // rest of the tile runs on whatever TMEM and shared memory hold (every
      // access stays inside the CTA's own allocations, and every later wait
      // returns at once on the abort flag), the loop then ends and no output
      // is written.  No branch out of the middle of the tile (measured 0.7 %
      // faster on the long context than breaking out here).
      ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_SFULL + sb), (j / C::NSB) & 1, abort_flag, kErrTimeoutSoftmax));
      tc_fence_after();
      float s[HB];
      {
        // load and wait in one asm statement each (the destination registers
        // fill asynchronously)
        uint32_t v[HB];
        const uint32_t sa = tmem + lane_base + C::TM_S + sb * BN + hw * HB;
        if constexpr (HB == 64) {
          tmem_ld64_wait(sa, v);
        } else {
#pragma unroll
          for (int cc = 0; cc < HB / 32; ++cc) tmem_ld32_wait(sa + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * cc));
        }
#pragma unroll
        for (int i = 0; i < HB; ++i) s[i] = __uint_as_float(v[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_SEMPTY + sb));
      if (qbias) {
        // the score terms of this tile's keys landed with its K/V copies (the
        // stage's barrier: its next phase, tile j + NS, needs PV_j, which
        // needs this warp's P-hat_j, so the parity wait is exact)
        const int st = j % C::NS;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(BAR(B_KFULL + st), (j / C::NS) & 1, abort_flag, kErrTimeoutSoftmax))) {
          ok = false;
          break;
        }
        const float4* b4 = reinterpret_cast<const float4*>(smem + C::OFF_BIAS + st * BN * 4 + hw * HB * 4);
#pragma unroll
        for (int i = 0; i < HB / 4; ++i) {
          const float4 bb = b4[i];
          s[4 * i] = __fadd_rn(s[4 * i], bb.x);
          s[4 * i + 1] = __fadd_rn(s[4 * i + 1], bb.y);
          s[4 * i + 2] = __fadd_rn(s[4 * i + 2], bb.z);
          s[4 * i + 3] = __fadd_rn(s[4 * i + 3], bb.w);
        }
      }
      // mask (only tiles that reach past the diagonal or past N need it)
      const int kbase = j * BN + hw * HB;
      const bool need_mask = (j * BN + BN > p.N) || (p.causal && j * BN + BN - 1 > row0);
      if (need_mask) {
        const int lim = p.causal ? min(p.N, row + 1) : p.N;
#pragma unroll
        for (int k = 0; k < HB; ++k) s[k] = (kbase + k >= lim) ? -INFINITY : s[k];
      }
      // Block maxima of S; c > 0, so the maximum of x = fl32(S * c) over a
      // block is fl32(max S * c) and needs no pass over x.
      float bms[NBH];
#pragma unroll
      for (int blk = 0; blk < NBH; ++blk) bms[blk] = tree_max<C::BETA>(s + blk * C::BETA);
      float m_new;
      if constexpr (C::NH == 2) {
        float* xb = xm + (j & 1) * 256;
        xb[hw * 128 + r] = __fmul_rn(tree_max<NBH>(bms), c);
        __syncwarp();             // the warp's stores are ordered before lane 0's release
        // only the two warps that share these rows synchronize (phase j of
        // their quadrant's barrier; neither can arrive for tile j+1 before
        // both passed tile j, so a parity wait is exact)
        if (lane == 0) mbar_arrive(BAR(B_XQ + (warp & 3)));
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_XQ + (warp & 3)), j & 1, abort_flag, kErrTimeoutSoftmax))) {
          ok = false;
          break;
        }
        m_new = fmaxf(xb[r], xb[128 + r]);
      } else {
        m_new = __fmul_rn(tree_max<NBH>(bms), c);
      }
      // The running max moves only when the tile's max exceeds it by more
      // than tau (tau = 0: whenever it rises); otherwise P is taken against
      // the stale max and may reach 2^tau.  m = -inf always moves.
      m_new = m_new > m + p.tau ? m_new : m;
      const float alpha = (m_new == m) ? 1.0f : ex2_approx(m - m_new);
      // whether any row of this warp rescales O (voted early: its latency
      // hides behind the block scales and the exponentials)
      const bool warp_rescale = __any_sync(0xffffffffu, m_new != m);
      if constexpr (C::CORR) {
        if (j > 0) {
          reinterpret_cast<float*>(smem + C::OFF_XM)[(j % 3) * 128 + r] = alpha;
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(B_AF + 4 * (warp & 3) + ((j - 1) & 3)));
        }
      }
      // Block scales first, from y_max = fl32(x_max - m) of each block: the
      // maximum of P over the block is 2^(y_max) (2^y is monotonic), and the
      // MXFP4 exponent follows from y_max exactly.
      float mult[NBH];
      uint32_t scb[NBH];
#pragma unroll
      for (int blk = 0; blk < NBH; ++blk) {
        const float ym = __fadd_rn(__fmul_rn(bms[blk], c), -m_new);
        if constexpr (FMT == HIFA4_NVFP4) {
          const float t = div6_rn_x256(ex2_approx(ym));                  // fl32(amax/6) / g_P, g_P = 2^-8
          scb[blk] = cvt_e4m3(t);
          mult[blk] = inv_tab[scb[blk]];                                  // fl32(1/(scale*g_P)), 0 for scale 0
        } else {
          scb[blk] = mx_scale_from_ymax(ym);
          mult[blk] = __uint_as_float((254u - scb[blk]) << 23);
        }
      }
      // P = 2^(S*c - m) element by element (MUFU ex2 for most pairs, the
      // FMA-pipe polynomial for kPolyPairs of every eight pairs), then the E2M1
      // codes of P * mult.
      uint32_t codes[HB / 8];
      float psum = 0.0f;
      const float2 c2 = make_float2(c, c);
      const float2 nm2 = make_float2(-m_new, -m_new);
      // one straight-line body per choice of the running sum of P (a branch
      // per element would split the block the compiler schedules)
      auto quant_tile = [&](auto lp_tag) {
        constexpr bool LP = decltype(lp_tag)::value;
        // codes only, exponentials first: P, then P * mult (LP without the sum)
        constexpr bool MULT = !LP && (HIFA4_EXP_FIRST < 0 ? D == 256 : HIFA4_EXP_FIRST != 0);
        float2 acc = make_float2(0.0f, 0.0f);
        // Without the sum of P, the multiplier folds into the exponent:
        // P * mult = 2^(S*c - m + log2 mult), one packed FMA per pair.
        float lnb[NBH];
        if constexpr (!LP && !MULT) {
#pragma unroll
          for (int blk = 0; blk < NBH; ++blk) {
            const float lm = FMT == HIFA4_NVFP4 ? log_tab[scb[blk]] : static_cast<float>(127 - static_cast<int>(scb[blk]));
            lnb[blk] = lm - m_new;
          }
        }
#pragma unroll
        for (int w = 0; w < HB / 8; ++w) {
          const int blk = (8 * w) / C::BETA;
          const float2 m2 = make_float2(mult[blk], mult[blk]);
          const float2 nb2 = (LP || MULT) ? nm2 : make_float2(lnb[blk], lnb[blk]);
          float2 e[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = 8 * w + 2 * q;
            const float2 y = ffma2(make_float2(s[i], s[i + 1]), c2, nb2);
            const int pair16 = (i % 16) / 2;
            float2 pp;
            if (pair16 < kPolyPairs) {
              // codes only (no sum of P): the exponential-free code argument
              if constexpr (!LP && !MULT && HIFA4_CODE_MAP) pp = e2m1_arg_from_log2(y);
              else pp = exp2_poly2(y);
            } else {
              pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
            }
            if constexpr (LP) {
              acc = fadd2(acc, pp);
              e[q] = fmul2(pp, m2);
            } else if constexpr (MULT) {
              e[q] = fmul2(pp, m2);
            } else {
              e[q] = pp;
            }
          }
          codes[w] = cvt_e2m1x8(e[0], e[1], e[2], e[3]);
        }
        if constexpr (LP) psum = acc.x + acc.y;
      };
      if (want_lp) quant_tile(std::true_type{});
      else quant_tile(std::false_type{});
      if (want_lp) l_p = fmaf(alpha, l_p, psum);
      if (EXT && p.dump.codes != nullptr && row < p.N) {
        // debug view of this tile: the codes and scales as they go to the
        // PV MMA, the running max, and (on the path that forms P) sum(P)
        const int64_t rt = (static_cast<int64_t>(bhq) * p.N + row) * p.nkt_all + j;
        uint4* dc = reinterpret_cast<uint4*>(p.dump.codes + rt * (BN / 2) + hw * (HB / 2));
#pragma unroll
        for (int ch = 0; ch < HB / 32; ++ch)
          dc[ch] = make_uint4(codes[4 * ch], codes[4 * ch + 1], codes[4 * ch + 2], codes[4 * ch + 3]);
        uint8_t* ds = p.dump.scales + rt * (BN / C::BETA) + hw * NBH;
#pragma unroll
        for (int blk = 0; blk < NBH; ++blk) ds[blk] = static_cast<uint8_t>(scb[blk]);
        if (hw == 0) p.dump.m[rt] = m_new;
        if (p.dump.sum_p != nullptr) {
          if constexpr (C::NH == 1) p.dump.sum_p[rt] = psum;
          else atomicAdd(p.dump.sum_p + rt, psum);     // two column halves; the caller zero-fills
        }
      }
      // Two uses of earlier PV products before the P-hat store and the O
      // rescale below:
      // - the P-hat buffer pb was last read by PV_{j-2}.  With one
      //   MMA-issuing thread, S_j was issued after PV_{j-2}, and a commit
      //   completes only after every earlier MMA of its thread, so the S_j
      //   wait above already covered that product.  (With a second issuer
      //   nothing orders the two, and PV_{j-2} is awaited here.)
      // - a warp that rescales O (a warp-uniform vote) needs PV_{j-1} retired.
      //   Its barrier is phase (j-1)/2 of buffer (j-1)%2, whose next phase
      //   PV_{j+1} cannot complete before this tile's P-hat exists, and whose
      //   earlier phase PV_{j-3} completed before S_j: the parity wait is exact.
      // With the correction warps the rescale is theirs.
      int jw = -1;
      if (!C::CORR && (!HIFA4_RELAX_PV || warp_rescale)) jw = j - 1;
      else if (C::TWO_ISSUERS) jw = j - 2;
      if (jw >= 0)
        ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_PEMPTY + (jw & 1)), (jw >> 1) & 1, abort_flag, kErrTimeoutSoftmax)) &&
             ok;
      {
        unsigned char* prow = smem + C::OFF_P + pb * C::SZ_P + r * C::PROW;
#pragma unroll
        for (int ch = 0; ch < HB / 32; ++ch) {
          const uint32_t phys = swz_chunk(r, hw * (HB / 32) + ch, C::PROW);
          *reinterpret_cast<uint4*>(prow + phys * 16) =
              make_uint4(codes[4 * ch], codes[4 * ch + 1], codes[4 * ch + 2], codes[4 * ch + 3]);
        }
        unsigned char* psf = smem + C::OFF_PSF + pb * C::NKC_P * 512 + (r & 31) * 16 + (r >> 5) * 4;
        if constexpr (NBH % 4 == 0) {
          // whole scale words: this thread's blocks 4i..4i+3 are the 4 bytes of
          // one word of chunk (hw * NBH) / 4 + i
#pragma unroll
          for (int wd = 0; wd < NBH / 4; ++wd)
            *reinterpret_cast<uint32_t*>(psf + ((hw * NBH) / 4 + wd) * 512) =
                scb[4 * wd] | (scb[4 * wd + 1] << 8) | (scb[4 * wd + 2] << 16) | (scb[4 * wd + 3] << 24);
        } else if constexpr (NBH == 2) {
          // two blocks: bytes 2hw, 2hw+1 of the row's word (one chunk per tile)
          *reinterpret_cast<uint16_t*>(psf + 2 * hw) = static_cast<uint16_t>(scb[0] | (scb[1] << 8));
        } else {
#pragma unroll
          for (int blk = 0; blk < NBH; ++blk) {
            const int gb = hw * NBH + blk;                     // block index within the tile
            psf[(gb / 4) * 512 + (gb % 4)] = static_cast<unsigned char>(scb[blk]);
          }
        }
      }
      // rescale this slice of the O row (and L) when the max rose (PV_{j-1}
      // retired: awaited above)
      if (!C::CORR && j > 0 && warp_rescale) {
        tc_fence_after();
        rescale_o_rows<HD>(tmem + lane_base + C::TM_O + hw * HD, tmem + lane_base + C::TM_L, hw == 0, alpha);
        tmem_wait_st();
      }
      fence_proxy_async_smem();   // the P-hat codes and scales are read by the MMA (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_PFULL + pb));
      m = m_new;
    }
    // ---------------------------------- epilogue ----------------------------------
    // the two halves' partial sums of P (same recurrence) add up to l_p
    float* lpx = reinterpret_cast<float*>(smem + C::OFF_LP);
    if constexpr (C::NH == 2) {
      if (hw == 1) {
        lpx[r] = l_p;
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_EP1));
      } else {
        ok = __all_sync(0xffffffffu, ok && mbar_wait(BAR(B_EP1), 0, abort_flag, kErrTimeoutSoftmax));
        l_p += lpx[r];
      }
    }
    // O and L are final once the last PV MMA retired.  Its completion is
    // awaited on the P-hat buffer's barrier, whose earlier phases are all
    // known to be complete here (the P-hat waits above); the o_ready barrier
    // may lag by two phases when the last tiles needed no rescale, and a
    // parity wait cannot tell phase k from phase k-2.
    const int jl = nkt - 1;
    const bool ready = __all_sync(0xffffffffu, ok && nkt > 0 &&
                                                  mbar_wait(BAR(B_PEMPTY + (jl & 1)), (jl >> 1) & 1, abort_flag,
                                                            kErrTimeoutSoftmax));
    if (ready) {
      tc_fence_after();
      uint32_t lv;
      tmem_ld1_wait(tmem + lane_base + C::TM_L, lv);
      const float l_acc = __uint_as_float(lv);           // sum of P-hat in MMA units (P-hat / g_P)
      const float l_phat = l_acc * kGP;
      const bool store = row < p.N;
      const int64_t orow = (static_cast<int64_t>(bhq) * p.N + row) * D + hw * HD;
      // INCONSISTENT: only half 0 holds the full l_p; share it
      float l_used = l_phat;
      if constexpr (!PREORDER && C::NH == 1) {
        l_used = l_p;
      } else if constexpr (!PREORDER) {
        // half 1 needs the full l_p of its row for the output scale
        if (hw == 0) {
          lpx[128 + r] = l_p;
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(B_EP2));
          l_used = l_p;
        } else {
          if (!mbar_wait(BAR(B_EP2), 0, abort_flag, kErrTimeoutSoftmax)) atomicOr(&g_device_error, kErrTimeoutSoftmax);
          l_used = lpx[128 + r];
        }
      }
      const float o_mul = kGP / l_used;                   // O_acc is in units of 1/g_P
#pragma unroll
      for (int cc = 0; cc < HD / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16_wait(tmem + lane_base + C::TM_O + hw * HD + cc * 16, v);
        if (store) {
          uint32_t packed[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = __uint_as_float(v[2 * i]) * o_mul, bb = __uint_as_float(v[2 * i + 1]) * o_mul;
            if (p.out_fp16) {
              __half2 hh = __floats2half2_rn(a, bb);
              packed[i] = *reinterpret_cast<uint32_t*>(&hh);
            } else {
              __nv_bfloat162 hh = __floats2bfloat162_rn(a, bb);
              packed[i] = *reinterpret_cast<uint32_t*>(&hh);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + orow + cc * 16);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
      }
      if (store && hw == 0) {
        const int64_t ri = static_cast<int64_t>(bhq) * p.N + row;
        if (p.lse) p.lse[ri] = m + log2f(l_used);
        if (EXT && p.dbg_l_phat) p.dbg_l_phat[ri] = l_phat;
        if (EXT && p.dbg_l_p) p.dbg_l_p[ri] = l_p;
      }
    }
  }

  // ---- teardown: every role is done; release TMEM ----
  if (*abort_flag) drain_after_abort();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_ALLOC);
}

// ------------------------------------------------------------------ host ---
bool make_tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, int swizzle_bytes);

template <int D, int BN, int FMT, bool PRE>
static hifa4_status launch_attn_t(const uint8_t* qc, const uint8_t* kc, const uint8_t* vc, const AttnParams& p,
                                  cudaStream_t st) {
  // the optional extras (the debug views -- the P-hat dump, the sums of P
  // and P-hat -- and the Q-Mean score term) are their own instantiation: the
  // production kernel carries none of their code
  const bool ext = p.dump.codes != nullptr || p.dbg_l_p != nullptr || p.dbg_l_phat != nullptr || p.qk_bias != nullptr;
  using C = AttnCfg<D, BN, FMT>;
  CUtensorMap tq, tk, tv;
  const uint64_t Np = static_cast<uint64_t>(p.Np);
  // the fused path quantizes Q in the kernel: its map is never used (built on K)
  const uint8_t* qmap = p.q_raw != nullptr ? kc : qc;
  const uint64_t qrows = static_cast<uint64_t>(p.B) * (p.q_raw != nullptr ? p.Hkv : p.Hq) * Np;
  if (!make_tmap_2d(&tq, qmap, D / 2, qrows, D / 2, 128, D / 2) ||
      !make_tmap_2d(&tk, kc, D / 2, static_cast<uint64_t>(p.B) * p.Hkv * Np, D / 2, BN, D / 2) ||
      !make_tmap_2d(&tv, vc, Np / 2, static_cast<uint64_t>(p.B) * p.Hkv * D, BN / 2, D, BN / 2)) {
    set_last_error("cuTensorMapEncodeTiled failed");
    return HIFA4_ERR_CUDA;
  }
  auto kern = ext ? attn_fwd_fp4_kernel<D, BN, FMT, PRE, true> : attn_fwd_fp4_kernel<D, BN, FMT, PRE, false>;
  const int smem = C::SMEM_REQ;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * p.num_qtiles;
  kern<<<grid, C::NTHREADS, smem, st>>>(tq, tk, tv, p);
  return launch_status("attn_fwd");
}

template <int D, int BN>
static hifa4_status launch_attn_fm(int fmt, int mode, const uint8_t* qc, const uint8_t* kc, const uint8_t* vc,
                                   const AttnParams& p, cudaStream_t st) {
  if (fmt == HIFA4_NVFP4)
    return mode == HIFA4_NORM_PREORDER ? launch_attn_t<D, BN, HIFA4_NVFP4, true>(qc, kc, vc, p, st)
                                       : launch_attn_t<D, BN, HIFA4_NVFP4, false>(qc, kc, vc, p, st);
  return mode == HIFA4_NORM_PREORDER ? launch_attn_t<D, BN, HIFA4_MXFP4, true>(qc, kc, vc, p, st)
                                     : launch_attn_t<D, BN, HIFA4_MXFP4, false>(qc, kc, vc, p, st);
}

hifa4_status attn_fwd_launch(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                             const uint8_t* vc, const uint8_t* vs, int B, int Hq, int Hkv, int N, int d, int fmt,
                             float softmax_scale, int causal, int mode, int block_n, void* o, int o_dt, float* lse,
                             float* dbg_l_phat, float* dbg_l_p, float rescale_threshold, const void* q_raw,
                             int q_dt, const float* q_s, const AttnDump* dump, const float* qk_bias,
                             cudaStream_t st) {
  AttnParams p;
  p.qk_bias = qk_bias;
  p.dump = dump != nullptr ? *dump : AttnDump{nullptr, nullptr, nullptr, nullptr};
  p.q_raw = q_raw;
  p.q_s = q_s;
  p.q_fp16 = q_dt == HIFA4_FP16;
  p.q_sf = qs;
  p.k_sf = ks;
  p.v_sf = vs;
  p.sf_qk_head = static_cast<int64_t>(hifa4_scale_bytes(N, d, static_cast<hifa4_format>(fmt)));
  p.Np = static_cast<int>(pad128(N));
  p.sf_v_head = static_cast<int64_t>(hifa4_scale_bytes(d, p.Np, static_cast<hifa4_format>(fmt)));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.num_qtiles = p.Np / 128;
  p.c_log2 = softmax_scale * 1.4426950408889634f;
  p.tau = rescale_threshold;
  p.causal = causal;
  p.out_fp16 = o_dt == HIFA4_FP16;
  p.o = o;
  p.lse = lse;
  p.dbg_l_phat = dbg_l_phat;
  p.dbg_l_p = dbg_l_p;
  if (block_n == 0) block_n = 128;
  p.nkt_all = (N + block_n - 1) / block_n;
  if (d == 64 && block_n == 64) return launch_attn_fm<64, 64>(fmt, mode, qc, kc, vc, p, st);
  if (d == 64 && block_n == 128) return launch_attn_fm<64, 128>(fmt, mode, qc, kc, vc, p, st);
  if (d == 128 && block_n == 64) return launch_attn_fm<128, 64>(fmt, mode, qc, kc, vc, p, st);
  if (d == 128 && block_n == 128) return launch_attn_fm<128, 128>(fmt, mode, qc, kc, vc, p, st);
  if (d == 256 && block_n == 128) return launch_attn_fm<256, 128>(fmt, mode, qc, kc, vc, p, st);
  set_last_error("attn_fwd: unsupported (d=%d, block_n=%d)", d, block_n);
  return HIFA4_ERR_UNSUPPORTED;
}

}  // namespace hifa4
