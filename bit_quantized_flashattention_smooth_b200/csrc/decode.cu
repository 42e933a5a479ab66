// decode.cu -- split-KV decode over the 4-bit KV cache (placeholder until the
// swap-AB tcgen05 decode kernel lands).
#include <cstdint>
#include "common.cuh"

namespace hifa4 {

int decode_default_splits(int B, int Hkv, int kv_len, int block_n) {
  const int tiles = (kv_len + block_n - 1) / block_n;
  int splits = 1;
  while (static_cast<int64_t>(B) * Hkv * splits < 2 * 148 && splits * 2 <= tiles) splits *= 2;
  return splits;
}

hifa4_status decode_launch(const void*, int, const float*, const uint8_t*, const uint8_t*, const uint8_t*,
                           const uint8_t*, int, int, int, int, int, int, float, int, int, int, int*, void*, size_t,
                           void*, int, cudaStream_t) {
  set_last_error("attn_decode: not built yet");
  return HIFA4_ERR_UNSUPPORTED;
}

}  // namespace hifa4
