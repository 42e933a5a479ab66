// common.cuh -- shared host/device helpers of the CUDA library (layouts,
// launch checks).  Nothing here is shared with the CPU oracle.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/hifa4.h"

namespace hifa4 {

// P-hat global prescale of NVFP4: g_P = 2^kPPrescaleLog2.
constexpr int kPPrescaleLog2 = HIFA4_NVFP4_P_PRESCALE_LOG2;

__host__ __device__ constexpr int beta_of(int fmt) { return fmt == HIFA4_NVFP4 ? 16 : 32; }
__host__ __device__ constexpr int64_t pad128(int64_t n) { return (n + 127) / 128 * 128; }

// Byte offset of scale (row, block) inside the tiled scale layout of one
// matrix with `nkc` 4-block chunks per 128-row group: 512-byte chunks ordered
// (row group, block group); inside a chunk (row%32)*16 + ((row%128)/32)*4 +
// block%4.  Matches the 32x128b.warpx4 TMEM copy used by the MMAs.
__host__ __device__ __forceinline__ int64_t sf_word_offset(int64_t row, int block4, int nkc) {
  // offset of the 4-byte word that holds blocks [4*block4, 4*block4+4) of `row`
  return ((row >> 7) * nkc + block4) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
}

// Optional dump of the quantized attention weights of the prefill kernel
// (hifa4_attn_fwd_dump): per query row and key tile, the P-hat codes and block
// scale codes, the running max after the tile, and the tile's sum of P.
struct AttnDump {
  uint8_t* codes;    // [B][Hq][N][nkt][BN/2]
  uint8_t* scales;   // [B][Hq][N][nkt][BN/beta]
  float* m;          // [B][Hq][N][nkt]
  float* sum_p;      // [B][Hq][N][nkt] or null
};

// Error helpers of the C ABI (api.cu).
void set_last_error(const char* fmt, ...);
hifa4_status launch_status(const char* what);

}  // namespace hifa4
