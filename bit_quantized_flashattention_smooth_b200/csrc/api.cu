// api.cu -- the C ABI (include/hifa4.h): argument validation, status codes,
// thread-local error strings, the device error word and TMA descriptor
// creation.  Kernels live in quantize.cu, attn_fwd.cu, decode.cu, probe.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hifa4 {

__device__ unsigned int g_device_error = 0;

static thread_local char g_last_error[512] = "";

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

hifa4_status launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("%s: %s", what, cudaGetErrorString(e));
    return HIFA4_ERR_CUDA;
  }
  return HIFA4_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D byte tensor [rows][inner_bytes] (row pitch inner_bytes), box
// [box_rows][box_inner], swizzle matching the box row (32/64/128 bytes).
bool make_tmap_2d(CUtensorMap* tm, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner_bytes, rows};
  cuuint64_t strides[1] = {inner_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

hifa4_status quantize_qkv_launch(const void*, const void*, const void*, int, int, int, int, int, int, const float*,
                                 const float*, int, uint8_t*, uint8_t*, uint8_t*, uint8_t*, uint8_t*, uint8_t*,
                                 const float*, cudaStream_t);
hifa4_status calib_q_mean_launch(const void*, int, int, int, int, int, int, int, const float*, float*, cudaStream_t);
hifa4_status q_mean_bias_launch(const uint8_t*, const uint8_t*, const float*, int, int, int, int, int, int, float*,
                                cudaStream_t);
hifa4_status calibrate_launch(const void*, const void*, int, int, int, int, int, int, int, float, int, float*, float*,
                              cudaStream_t);
hifa4_status attn_fwd_launch(const uint8_t*, const uint8_t*, const uint8_t*, const uint8_t*, const uint8_t*,
                             const uint8_t*, int, int, int, int, int, int, float, int, int, int, void*, int, float*,
                             float*, float*, float, const void*, int, const float*, const AttnDump*, const float*,
                             cudaStream_t);
hifa4_status decode_launch(const void*, int, const float*, const uint8_t*, const uint8_t*, const uint8_t*,
                           const uint8_t*, int, int, int, int, int, int, int, float, int, int, int, int*, void*, size_t,
                           void*, int, float, cudaStream_t);
hifa4_status kv_append_launch(const void*, const void*, int, int, int, int, int, const float*, int, int, int,
                              uint8_t*, uint8_t*, uint8_t*, uint8_t*, void*, cudaStream_t);
int decode_default_splits(int B, int Hkv, int kv_len, int block_n);
hifa4_status fp4_mma_probe_launch(const uint8_t*, const uint8_t*, const uint8_t*, const uint8_t*, int, int, int, int,
                                  int, float*, cudaStream_t);
hifa4_status convert_probe_launch(const float*, int64_t, uint8_t*, uint8_t*, cudaStream_t);
hifa4_status div6_probe_launch(uint32_t, uint32_t, unsigned long long*, uint32_t*, cudaStream_t);
hifa4_status exp2_poly_probe_launch(const float*, int64_t, float*, cudaStream_t);
hifa4_status e2m1_map_probe_launch(const float*, int64_t, uint8_t*, uint8_t*, cudaStream_t);
hifa4_status wait_timeout_probe_launch(unsigned int*, cudaStream_t);
hifa4_status bf16_attn_launch(const void*, const void*, const void*, int, int, int, int, int, float, int, void*, float*,
                              cudaStream_t);
hifa4_status transpose_v_bf16_launch(const void*, int, int, int, int, void*, cudaStream_t);

}  // namespace hifa4

using namespace hifa4;

#define HIFA4_REQUIRE(cond, code, ...) \
  do {                                 \
    if (!(cond)) {                     \
      set_last_error(__VA_ARGS__);     \
      return code;                     \
    }                                  \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool valid_d(int d) { return d == 64 || d == 128 || d == 256; }
static bool valid_fmt(int f) { return f == HIFA4_NVFP4 || f == HIFA4_MXFP4; }
static bool valid_dt(int t) { return t == HIFA4_BF16 || t == HIFA4_FP16; }
// Largest rescale threshold: with a stale running max P reaches 2^tau, and the
// NVFP4 P-hat scale fl32(amax/6)/2^-8 must stay within UE4M3's 448 (2^tau <= 10.5).
static float max_tau(int fmt) { return fmt == HIFA4_NVFP4 ? 3.0f : 8.0f; }
static bool valid_tau(int fmt, float tau) { return tau >= 0.0f && tau <= max_tau(fmt); }

extern "C" {

size_t hifa4_codes_bytes(int64_t rows, int k) {
  if (rows < 0 || k <= 0) return 0;
  return static_cast<size_t>(pad128(rows)) * static_cast<size_t>(k) / 2;
}

size_t hifa4_scale_bytes(int64_t rows, int k, hifa4_format fmt) {
  if (rows < 0 || k <= 0 || !valid_fmt(fmt)) return 0;
  const int64_t nb = k / beta_of(fmt);
  const int64_t nkc = (nb + 3) / 4;
  return static_cast<size_t>(pad128(rows) / 128 * nkc * 512);
}

hifa4_status hifa4_calibrate_smooth_qk(const void* q, const void* k, hifa4_dtype dt, int B, int Hq, int Hkv,
                                       int n_cal, int ld_tok, int d, float alpha, int enable, float* s_out,
                                       float* inv_s_out, hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && k && s_out && inv_s_out, HIFA4_ERR_INVALID_ARG, "calibrate: null pointer");
  HIFA4_REQUIRE(valid_dt(dt), HIFA4_ERR_INVALID_ARG, "calibrate: bad dtype %d", (int)dt);
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0, HIFA4_ERR_INVALID_ARG,
                "calibrate: bad heads B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  HIFA4_REQUIRE(n_cal > 0 && n_cal <= ld_tok, HIFA4_ERR_INVALID_ARG, "calibrate: need 0 < n_cal <= ld_tok");
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "calibrate: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(alpha >= 0.0f && alpha <= 1.0f, HIFA4_ERR_INVALID_ARG, "calibrate: alpha outside [0,1]");
  HIFA4_REQUIRE(enable >= 0 && enable <= 2, HIFA4_ERR_INVALID_ARG, "calibrate: enable must be 0, 1 or 2");
  return calibrate_launch(q, k, dt, B, Hq, Hkv, n_cal, ld_tok, d, alpha, enable, s_out, inv_s_out,
                          static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_quantize_qkv(const void* q, const void* k, const void* v, hifa4_dtype dt, int B, int Hq,
                                int Hkv, int N, int d, const float* s, const float* inv_s, hifa4_format fmt,
                                uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales,
                                uint8_t* vt_codes, uint8_t* vt_scales, hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && k && v && q_codes && q_scales && k_codes && k_scales && vt_codes && vt_scales,
                HIFA4_ERR_INVALID_ARG, "quantize_qkv: null pointer");
  HIFA4_REQUIRE(valid_dt(dt) && valid_fmt(fmt), HIFA4_ERR_INVALID_ARG, "quantize_qkv: bad dtype/format");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "quantize_qkv: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "quantize_qkv: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(q_codes) && aligned16(q_scales) &&
                    aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) && aligned16(vt_scales) &&
                    (!s || aligned16(s)) && (!inv_s || aligned16(inv_s)),
                HIFA4_ERR_INVALID_ARG, "quantize_qkv: pointers must be 16-byte aligned");
  return quantize_qkv_launch(q, k, v, dt, B, Hq, Hkv, N, d, s, inv_s, fmt, q_codes, q_scales, k_codes, k_scales,
                             vt_codes, vt_scales, nullptr, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_quantize_kv(const void* k, const void* v, hifa4_dtype dt, int B, int Hkv, int N, int d,
                               const float* inv_s, hifa4_format fmt, uint8_t* k_codes, uint8_t* k_scales,
                               uint8_t* vt_codes, uint8_t* vt_scales, hifa4_stream_t stream) {
  HIFA4_REQUIRE(k && v && k_codes && k_scales && vt_codes && vt_scales, HIFA4_ERR_INVALID_ARG,
                "quantize_kv: null pointer");
  HIFA4_REQUIRE(valid_dt(dt) && valid_fmt(fmt), HIFA4_ERR_INVALID_ARG, "quantize_kv: bad dtype/format");
  HIFA4_REQUIRE(B > 0 && Hkv > 0 && N > 0, HIFA4_ERR_INVALID_ARG, "quantize_kv: bad shape");
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "quantize_kv: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(aligned16(k) && aligned16(v) && aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) &&
                    aligned16(vt_scales) && (!inv_s || aligned16(inv_s)),
                HIFA4_ERR_INVALID_ARG, "quantize_kv: pointers must be 16-byte aligned");
  return quantize_qkv_launch(nullptr, k, v, dt, B, Hkv, Hkv, N, d, nullptr, inv_s, fmt, nullptr, nullptr, k_codes,
                             k_scales, vt_codes, vt_scales, nullptr, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_calibrate_q_mean(const void* q, hifa4_dtype dt, int B, int Hq, int Hkv, int n_cal, int ld_tok,
                                   int d, const float* s, float* mu_out, hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && mu_out, HIFA4_ERR_INVALID_ARG, "calibrate_q_mean: null pointer");
  HIFA4_REQUIRE(valid_dt(dt), HIFA4_ERR_INVALID_ARG, "calibrate_q_mean: bad dtype %d", (int)dt);
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0, HIFA4_ERR_INVALID_ARG,
                "calibrate_q_mean: bad heads B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  HIFA4_REQUIRE(n_cal > 0 && n_cal <= ld_tok, HIFA4_ERR_INVALID_ARG, "calibrate_q_mean: need 0 < n_cal <= ld_tok");
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "calibrate_q_mean: d=%d not in {64,128,256}", d);
  return calib_q_mean_launch(q, dt, B, Hq, Hkv, n_cal, ld_tok, d, s, mu_out, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_quantize_qkv_qmean(const void* q, const void* k, const void* v, hifa4_dtype dt, int B, int Hq,
                                      int Hkv, int N, int d, const float* s, const float* inv_s, const float* q_mu,
                                      hifa4_format fmt, uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes,
                                      uint8_t* k_scales, uint8_t* vt_codes, uint8_t* vt_scales,
                                      hifa4_stream_t stream) {
  HIFA4_REQUIRE(q_mu && aligned16(q_mu), HIFA4_ERR_INVALID_ARG,
                "quantize_qkv_qmean: q_mu must be a 16-byte aligned device pointer");
  HIFA4_REQUIRE(q && k && v && q_codes && q_scales && k_codes && k_scales && vt_codes && vt_scales,
                HIFA4_ERR_INVALID_ARG, "quantize_qkv_qmean: null pointer");
  HIFA4_REQUIRE(valid_dt(dt) && valid_fmt(fmt), HIFA4_ERR_INVALID_ARG, "quantize_qkv_qmean: bad dtype/format");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "quantize_qkv_qmean: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "quantize_qkv_qmean: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(q_codes) && aligned16(q_scales) &&
                    aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) && aligned16(vt_scales) &&
                    (!s || aligned16(s)) && (!inv_s || aligned16(inv_s)),
                HIFA4_ERR_INVALID_ARG, "quantize_qkv_qmean: pointers must be 16-byte aligned");
  return quantize_qkv_launch(q, k, v, dt, B, Hq, Hkv, N, d, s, inv_s, fmt, q_codes, q_scales, k_codes, k_scales,
                             vt_codes, vt_scales, q_mu, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_q_mean_bias(const uint8_t* k_codes, const uint8_t* k_scales, const float* q_mu, int B, int Hq,
                               int Hkv, int N, int d, hifa4_format fmt, float* bias_out, hifa4_stream_t stream) {
  HIFA4_REQUIRE(k_codes && k_scales && q_mu && bias_out, HIFA4_ERR_INVALID_ARG, "q_mean_bias: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt), HIFA4_ERR_INVALID_ARG, "q_mean_bias: bad format");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "q_mean_bias: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(Hq / Hkv <= 8, HIFA4_ERR_UNSUPPORTED, "q_mean_bias: at most 8 query heads per kv head");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq <= 65535, HIFA4_ERR_UNSUPPORTED,
                "q_mean_bias: B*Hq=%lld exceeds 65535 (one grid row per batch and query head)",
                static_cast<long long>(B) * Hq);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "q_mean_bias: d=%d not in {64,128,256}", d);
  return q_mean_bias_launch(k_codes, k_scales, q_mu, B, Hq, Hkv, N, d, fmt, bias_out,
                            static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_attn_fwd(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                            const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales, int B,
                            int Hq, int Hkv, int N, int d, hifa4_format fmt, float softmax_scale, int causal,
                            hifa4_norm_mode mode, int block_n, void* o, hifa4_dtype o_dt, float* lse,
                            float* dbg_l_phat, float* dbg_l_p, hifa4_stream_t stream) {
  return hifa4_attn_fwd_ex(q_codes, q_scales, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, N, d, fmt,
                           softmax_scale, causal, mode, block_n, o, o_dt, lse, dbg_l_phat, dbg_l_p, 0.0f, stream);
}

hifa4_status hifa4_attn_fwd_ex(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                               const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales, int B,
                               int Hq, int Hkv, int N, int d, hifa4_format fmt, float softmax_scale, int causal,
                               hifa4_norm_mode mode, int block_n, void* o, hifa4_dtype o_dt, float* lse,
                               float* dbg_l_phat, float* dbg_l_p, float rescale_threshold, hifa4_stream_t stream) {
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_tau(fmt, rescale_threshold), HIFA4_ERR_INVALID_ARG,
                "attn_fwd: rescale_threshold must be in [0, %g] for this format", max_tau(fmt));
  HIFA4_REQUIRE(q_codes && q_scales && k_codes && k_scales && vt_codes && vt_scales && o, HIFA4_ERR_INVALID_ARG,
                "attn_fwd: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_dt(o_dt), HIFA4_ERR_INVALID_ARG, "attn_fwd: bad format/dtype");
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_fwd: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "attn_fwd: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "attn_fwd: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(block_n == 0 || block_n == 64 || block_n == 128, HIFA4_ERR_UNSUPPORTED,
                "attn_fwd: block_n=%d not in {0,64,128}", block_n);
  HIFA4_REQUIRE(!(d == 256 && block_n == 64), HIFA4_ERR_UNSUPPORTED, "attn_fwd: d=256 needs block_n=128");
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_fwd: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q_codes) && aligned16(q_scales) && aligned16(k_codes) && aligned16(k_scales) &&
                    aligned16(vt_codes) && aligned16(vt_scales) && aligned16(o),
                HIFA4_ERR_INVALID_ARG, "attn_fwd: pointers must be 16-byte aligned");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq * pad128(N) < (int64_t(1) << 31), HIFA4_ERR_UNSUPPORTED,
                "attn_fwd: problem too large");
  return attn_fwd_launch(q_codes, q_scales, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, N, d, fmt,
                         softmax_scale, causal, mode, block_n, o, o_dt, lse, dbg_l_phat, dbg_l_p, rescale_threshold,
                         nullptr, 0, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_attn_fwd_qmean(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                                  const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales,
                                  const float* qk_bias, int B, int Hq, int Hkv, int N, int d, hifa4_format fmt,
                                  float softmax_scale, int causal, hifa4_norm_mode mode, int block_n, void* o,
                                  hifa4_dtype o_dt, float* lse, float rescale_threshold, hifa4_stream_t stream) {
  HIFA4_REQUIRE(qk_bias && aligned16(qk_bias), HIFA4_ERR_INVALID_ARG,
                "attn_fwd_qmean: qk_bias must be a 16-byte aligned device pointer");
  HIFA4_REQUIRE(d == 64 || d == 128, HIFA4_ERR_UNSUPPORTED, "attn_fwd_qmean: d=%d not in {64,128}", d);
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_tau(fmt, rescale_threshold), HIFA4_ERR_INVALID_ARG,
                "attn_fwd_qmean: rescale_threshold must be in [0, %g] for this format", max_tau(fmt));
  HIFA4_REQUIRE(q_codes && q_scales && k_codes && k_scales && vt_codes && vt_scales && o, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_qmean: null pointer");
  HIFA4_REQUIRE(valid_dt(o_dt), HIFA4_ERR_INVALID_ARG, "attn_fwd_qmean: bad dtype");
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_qmean: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_qmean: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(block_n == 0 || block_n == 64 || block_n == 128, HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_qmean: block_n=%d not in {0,64,128}", block_n);
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_fwd_qmean: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q_codes) && aligned16(q_scales) && aligned16(k_codes) && aligned16(k_scales) &&
                    aligned16(vt_codes) && aligned16(vt_scales) && aligned16(o),
                HIFA4_ERR_INVALID_ARG, "attn_fwd_qmean: pointers must be 16-byte aligned");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq * pad128(N) < (int64_t(1) << 31), HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_qmean: problem too large");
  return attn_fwd_launch(q_codes, q_scales, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, N, d, fmt,
                         softmax_scale, causal, mode, block_n, o, o_dt, lse, nullptr, nullptr, rescale_threshold,
                         nullptr, 0, nullptr, nullptr, qk_bias, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_attn_fwd_dump(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                                 const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales, int B,
                                 int Hq, int Hkv, int N, int d, hifa4_format fmt, float softmax_scale, int causal,
                                 hifa4_norm_mode mode, int block_n, void* o, hifa4_dtype o_dt, float rescale_threshold,
                                 uint8_t* phat_codes, uint8_t* phat_scales, float* tile_m, float* tile_sum_p,
                                 hifa4_stream_t stream) {
  HIFA4_REQUIRE(phat_codes && phat_scales && tile_m, HIFA4_ERR_INVALID_ARG, "attn_fwd_dump: null dump pointer");
  HIFA4_REQUIRE(aligned16(phat_codes), HIFA4_ERR_INVALID_ARG, "attn_fwd_dump: phat_codes must be 16-byte aligned");
  // the shared checks of the forward (no launch happens on failure)
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_tau(fmt, rescale_threshold), HIFA4_ERR_INVALID_ARG,
                "attn_fwd_dump: rescale_threshold must be in [0, %g] for this format", max_tau(fmt));
  HIFA4_REQUIRE(q_codes && q_scales && k_codes && k_scales && vt_codes && vt_scales && o, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_dump: null pointer");
  HIFA4_REQUIRE(valid_dt(o_dt), HIFA4_ERR_INVALID_ARG, "attn_fwd_dump: bad dtype");
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_dump: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_dump: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "attn_fwd_dump: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(block_n == 0 || block_n == 64 || block_n == 128, HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_dump: block_n=%d not in {0,64,128}", block_n);
  HIFA4_REQUIRE(!(d == 256 && block_n == 64), HIFA4_ERR_UNSUPPORTED, "attn_fwd_dump: d=256 needs block_n=128");
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_fwd_dump: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q_codes) && aligned16(q_scales) && aligned16(k_codes) && aligned16(k_scales) &&
                    aligned16(vt_codes) && aligned16(vt_scales) && aligned16(o),
                HIFA4_ERR_INVALID_ARG, "attn_fwd_dump: pointers must be 16-byte aligned");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq * pad128(N) < (int64_t(1) << 31), HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_dump: problem too large");
  AttnDump dump{phat_codes, phat_scales, tile_m, tile_sum_p};
  return attn_fwd_launch(q_codes, q_scales, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, N, d, fmt,
                         softmax_scale, causal, mode, block_n, o, o_dt, nullptr, nullptr, nullptr, rescale_threshold,
                         nullptr, 0, nullptr, &dump, nullptr, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_attn_fwd_fused(const void* q, hifa4_dtype q_dt, const float* s, const uint8_t* k_codes,
                                  const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales, int B,
                                  int Hq, int Hkv, int N, int d, hifa4_format fmt, float softmax_scale, int causal,
                                  hifa4_norm_mode mode, int block_n, void* o, hifa4_dtype o_dt, float* lse,
                                  float* dbg_l_phat, float* dbg_l_p, float rescale_threshold,
                                  hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && k_codes && k_scales && vt_codes && vt_scales && o, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_fused: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_dt(o_dt) && valid_dt(q_dt), HIFA4_ERR_INVALID_ARG,
                "attn_fwd_fused: bad format/dtype");
  HIFA4_REQUIRE(valid_tau(fmt, rescale_threshold), HIFA4_ERR_INVALID_ARG,
                "attn_fwd_fused: rescale_threshold must be in [0, %g] for this format", max_tau(fmt));
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_fused: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0, HIFA4_ERR_INVALID_ARG,
                "attn_fwd_fused: bad shape B=%d Hq=%d Hkv=%d N=%d", B, Hq, Hkv, N);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "attn_fwd_fused: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(block_n == 0 || block_n == 64 || block_n == 128, HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_fused: block_n=%d not in {0,64,128}", block_n);
  HIFA4_REQUIRE(!(d == 256 && block_n == 64), HIFA4_ERR_UNSUPPORTED, "attn_fwd_fused: d=256 needs block_n=128");
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_fwd_fused: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q) && aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) &&
                    aligned16(vt_scales) && aligned16(o) && (!s || aligned16(s)),
                HIFA4_ERR_INVALID_ARG, "attn_fwd_fused: pointers must be 16-byte aligned");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq * pad128(N) < (int64_t(1) << 31), HIFA4_ERR_UNSUPPORTED,
                "attn_fwd_fused: problem too large");
  return attn_fwd_launch(nullptr, nullptr, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, N, d, fmt,
                         softmax_scale, causal, mode, block_n, o, o_dt, lse, dbg_l_phat, dbg_l_p, rescale_threshold,
                         q, q_dt, s, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

size_t hifa4_decode_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || d <= 0 || num_splits <= 0) return 0;
  return static_cast<size_t>(B) * Hq * num_splits * (d + 2) * sizeof(float);
}

int hifa4_decode_default_splits(int B, int Hkv, int kv_len, int block_n) {
  return decode_default_splits(B, Hkv, kv_len, block_n);
}

hifa4_status hifa4_attn_decode(const void* q, hifa4_dtype q_dt, const float* s, const uint8_t* k_codes,
                               const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales, int B,
                               int Hq, int Hkv, int kv_len, int d, hifa4_format fmt, float softmax_scale,
                               hifa4_norm_mode mode, int block_n, int num_splits, int* num_splits_used,
                               void* workspace, size_t ws_bytes, void* o, hifa4_dtype o_dt,
                               hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && k_codes && k_scales && vt_codes && vt_scales && o && workspace, HIFA4_ERR_INVALID_ARG,
                "attn_decode: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_dt(q_dt) && valid_dt(o_dt), HIFA4_ERR_INVALID_ARG,
                "attn_decode: bad format/dtype");
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_decode: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && kv_len > 0, HIFA4_ERR_INVALID_ARG,
                "attn_decode: bad shape");
  HIFA4_REQUIRE(d == 128, HIFA4_ERR_UNSUPPORTED, "attn_decode: d=%d (only 128)", d);
  HIFA4_REQUIRE(Hq / Hkv == 1 || Hq / Hkv == 2 || Hq / Hkv == 4 || Hq / Hkv == 8, HIFA4_ERR_UNSUPPORTED,
                "attn_decode: GQA group %d not in {1,2,4,8}", Hq / Hkv);
  HIFA4_REQUIRE(block_n == 0 || block_n == 128, HIFA4_ERR_UNSUPPORTED, "attn_decode: block_n must be 128");
  HIFA4_REQUIRE(num_splits >= 0, HIFA4_ERR_INVALID_ARG, "attn_decode: num_splits < 0");
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_decode: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q) && aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) &&
                    aligned16(vt_scales) && aligned16(o) && aligned16(workspace) && (!s || aligned16(s)),
                HIFA4_ERR_INVALID_ARG, "attn_decode: pointers must be 16-byte aligned");
  return decode_launch(q, q_dt, s, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, kv_len, kv_len, d, fmt,
                       softmax_scale, mode, 128, num_splits, num_splits_used, workspace, ws_bytes, o, o_dt, 0.0f,
                       static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_attn_decode_cache(const void* q, hifa4_dtype q_dt, const float* s, const uint8_t* k_codes,
                                     const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales,
                                     int B, int Hq, int Hkv, int kv_len, int kv_capacity, int d, hifa4_format fmt,
                                     float softmax_scale, hifa4_norm_mode mode, int block_n, int num_splits,
                                     int* num_splits_used, void* workspace, size_t ws_bytes, void* o,
                                     hifa4_dtype o_dt, float rescale_threshold, hifa4_stream_t stream) {
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_tau(fmt, rescale_threshold), HIFA4_ERR_INVALID_ARG,
                "attn_decode_cache: rescale_threshold must be in [0, %g] for this format", max_tau(fmt));
  HIFA4_REQUIRE(kv_capacity >= kv_len, HIFA4_ERR_INVALID_ARG, "attn_decode_cache: kv_len %d > capacity %d", kv_len,
                kv_capacity);
  HIFA4_REQUIRE(q && k_codes && k_scales && vt_codes && vt_scales && o && workspace, HIFA4_ERR_INVALID_ARG,
                "attn_decode_cache: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt) && valid_dt(q_dt) && valid_dt(o_dt), HIFA4_ERR_INVALID_ARG,
                "attn_decode_cache: bad format/dtype");
  HIFA4_REQUIRE(mode == HIFA4_NORM_PREORDER || mode == HIFA4_NORM_INCONSISTENT, HIFA4_ERR_INVALID_ARG,
                "attn_decode_cache: bad normalizer mode");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && kv_len > 0, HIFA4_ERR_INVALID_ARG,
                "attn_decode_cache: bad shape");
  HIFA4_REQUIRE(d == 128, HIFA4_ERR_UNSUPPORTED, "attn_decode_cache: d=%d (only 128)", d);
  HIFA4_REQUIRE(Hq / Hkv == 1 || Hq / Hkv == 2 || Hq / Hkv == 4 || Hq / Hkv == 8, HIFA4_ERR_UNSUPPORTED,
                "attn_decode_cache: GQA group %d not in {1,2,4,8}", Hq / Hkv);
  HIFA4_REQUIRE(block_n == 0 || block_n == 128, HIFA4_ERR_UNSUPPORTED, "attn_decode_cache: block_n must be 128");
  HIFA4_REQUIRE(num_splits >= 0 && softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "attn_decode_cache: bad arguments");
  HIFA4_REQUIRE(aligned16(q) && aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) &&
                    aligned16(vt_scales) && aligned16(o) && aligned16(workspace) && (!s || aligned16(s)),
                HIFA4_ERR_INVALID_ARG, "attn_decode_cache: pointers must be 16-byte aligned");
  return decode_launch(q, q_dt, s, k_codes, k_scales, vt_codes, vt_scales, B, Hq, Hkv, kv_len, kv_capacity, d, fmt,
                       softmax_scale, mode, 128, num_splits, num_splits_used, workspace, ws_bytes, o, o_dt,
                       rescale_threshold, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_kv_cache_append(const void* k_new, const void* v_new, hifa4_dtype dt, int B, int Hkv, int T,
                                   int d, const float* inv_s, hifa4_format fmt, int pos, int capacity,
                                   uint8_t* k_codes, uint8_t* k_scales, uint8_t* vt_codes, uint8_t* vt_scales,
                                   void* v_tail, hifa4_stream_t stream) {
  HIFA4_REQUIRE(k_new && v_new && k_codes && k_scales && vt_codes && vt_scales && v_tail, HIFA4_ERR_INVALID_ARG,
                "kv_cache_append: null pointer");
  HIFA4_REQUIRE(valid_dt(dt) && valid_fmt(fmt), HIFA4_ERR_INVALID_ARG, "kv_cache_append: bad dtype/format");
  HIFA4_REQUIRE(B > 0 && Hkv > 0 && T > 0 && pos >= 0 && pos + T <= capacity, HIFA4_ERR_INVALID_ARG,
                "kv_cache_append: bad shape (B=%d Hkv=%d T=%d pos=%d capacity=%d)", B, Hkv, T, pos, capacity);
  HIFA4_REQUIRE(valid_d(d), HIFA4_ERR_UNSUPPORTED, "kv_cache_append: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(aligned16(k_codes) && aligned16(k_scales) && aligned16(vt_codes) && aligned16(vt_scales) &&
                    (!inv_s || aligned16(inv_s)),
                HIFA4_ERR_INVALID_ARG, "kv_cache_append: cache pointers must be 16-byte aligned");
  return kv_append_launch(k_new, v_new, dt, B, Hkv, T, d, inv_s, fmt, pos, capacity, k_codes, k_scales, vt_codes,
                          vt_scales, v_tail, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_fp4_mma_probe(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                                 const uint8_t* b_scales, int n, int k, hifa4_format fmt, int repeats, int ctas,
                                 float* d_out, hifa4_stream_t stream) {
  HIFA4_REQUIRE(a_codes && a_scales && b_codes && b_scales && d_out, HIFA4_ERR_INVALID_ARG,
                "fp4_mma_probe: null pointer");
  HIFA4_REQUIRE(valid_fmt(fmt) && repeats >= 1 && ctas >= 1 && ctas <= 65535, HIFA4_ERR_INVALID_ARG,
                "fp4_mma_probe: bad format/repeats/ctas");
  HIFA4_REQUIRE(aligned16(a_codes) && aligned16(a_scales) && aligned16(b_codes) && aligned16(b_scales),
                HIFA4_ERR_INVALID_ARG, "fp4_mma_probe: pointers must be 16-byte aligned");
  return fp4_mma_probe_launch(a_codes, a_scales, b_codes, b_scales, n, k, fmt, repeats, ctas, d_out,
                              static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_convert_probe(const float* x, int64_t count, uint8_t* e2m1_out, uint8_t* e4m3_out,
                                 hifa4_stream_t stream) {
  HIFA4_REQUIRE(x && e2m1_out && e4m3_out && count >= 0, HIFA4_ERR_INVALID_ARG, "convert_probe: bad args");
  if (count == 0) return HIFA4_OK;
  return convert_probe_launch(x, count, e2m1_out, e4m3_out, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_div6_probe(uint32_t lo_bits, uint32_t hi_bits, unsigned long long* mismatches,
                              uint32_t* first_bad, hifa4_stream_t stream) {
  HIFA4_REQUIRE(mismatches && first_bad && lo_bits <= hi_bits, HIFA4_ERR_INVALID_ARG, "div6_probe: bad args");
  return div6_probe_launch(lo_bits, hi_bits, mismatches, first_bad, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_bf16_attn_fwd(const void* q, const void* k, const void* vt, int B, int Hq, int Hkv, int N, int d,
                                 float softmax_scale, int causal, void* o, float* lse, hifa4_stream_t stream) {
  HIFA4_REQUIRE(q && k && vt && o, HIFA4_ERR_INVALID_ARG, "bf16_attn_fwd: null pointer");
  HIFA4_REQUIRE(B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && N > 0 && N % 8 == 0, HIFA4_ERR_INVALID_ARG,
                "bf16_attn_fwd: bad shape B=%d Hq=%d Hkv=%d N=%d (N a multiple of 8)", B, Hq, Hkv, N);
  HIFA4_REQUIRE(d == 64 || d == 128 || d == 256, HIFA4_ERR_UNSUPPORTED, "bf16_attn_fwd: d=%d not in {64,128,256}", d);
  HIFA4_REQUIRE(softmax_scale > 0.0f, HIFA4_ERR_INVALID_ARG, "bf16_attn_fwd: softmax_scale must be > 0");
  HIFA4_REQUIRE(aligned16(q) && aligned16(k) && aligned16(vt) && aligned16(o), HIFA4_ERR_INVALID_ARG,
                "bf16_attn_fwd: pointers must be 16-byte aligned");
  HIFA4_REQUIRE(static_cast<int64_t>(B) * Hq * N < (int64_t(1) << 31), HIFA4_ERR_UNSUPPORTED,
                "bf16_attn_fwd: problem too large");
  return bf16_attn_launch(q, k, vt, B, Hq, Hkv, N, d, softmax_scale, causal, o, lse, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_bf16_transpose_v(const void* v, int B, int Hkv, int N, int d, void* vt, hifa4_stream_t stream) {
  HIFA4_REQUIRE(v && vt && B >= 0 && Hkv > 0 && N >= 0 && d > 0, HIFA4_ERR_INVALID_ARG, "bf16_transpose_v: bad args");
  return transpose_v_bf16_launch(v, B, Hkv, N, d, vt, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_wait_timeout_probe(unsigned int* status, hifa4_stream_t stream) {
  HIFA4_REQUIRE(status != nullptr, HIFA4_ERR_INVALID_ARG, "wait_timeout_probe: null status");
  return wait_timeout_probe_launch(status, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_exp2_poly_probe(const float* y, int64_t count, float* out, hifa4_stream_t stream) {
  HIFA4_REQUIRE(count >= 0 && (count == 0 || (y && out)), HIFA4_ERR_INVALID_ARG, "exp2_poly_probe: bad args");
  return exp2_poly_probe_launch(y, count, out, static_cast<cudaStream_t>(stream));
}

hifa4_status hifa4_e2m1_map_probe(const float* y, int64_t count, uint8_t* codes_map, uint8_t* codes_ex2,
                                   hifa4_stream_t stream) {
  HIFA4_REQUIRE(count >= 0 && (count == 0 || (y && codes_map && codes_ex2)), HIFA4_ERR_INVALID_ARG,
                "e2m1_map_probe: bad args");
  return e2m1_map_probe_launch(y, count, codes_map, codes_ex2, static_cast<cudaStream_t>(stream));
}

const char* hifa4_status_string(hifa4_status st) {
  switch (st) {
    case HIFA4_OK: return "ok";
    case HIFA4_ERR_INVALID_ARG: return "invalid argument";
    case HIFA4_ERR_UNSUPPORTED: return "unsupported configuration";
    case HIFA4_ERR_CUDA: return "CUDA error";
    case HIFA4_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* hifa4_last_error(void) { return g_last_error; }

unsigned int hifa4_device_error(void) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return 0xFFFFFFFFu;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  const unsigned int zero = 0;
  cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  return v;
}

}  // extern "C"
