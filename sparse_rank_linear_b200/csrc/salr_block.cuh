// salr_block.cuh - the 128 x 64 block of the SALR weight format and the warp-level
// prefix sums its encoder and decoders share.
#pragma once
#include <cstdint>

namespace salr {

constexpr int kBlockRows = 128;
constexpr int kBlockCols = 64;
constexpr int kBitmapBytes = kBlockRows * kBlockCols / 8;  // 1024
constexpr int kEncThreads = 256;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace salr
