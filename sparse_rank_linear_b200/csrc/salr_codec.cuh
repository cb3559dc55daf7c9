// salr_codec.cuh - GPU encoder and decoder of the SALR bitmap block format.
//
// Encoding (SALR technical summary, Methodology 1 and 4): each row of W keeps its
// `keep` entries of largest magnitude (ties to the lower column), the mask is stored as a
// bitmap and the kept values as a compact array, both cut into 128 x 64 blocks that are
// located through a per-block offset table.  The byte layout is the one written out in
// include/salr.h.
#pragma once
#include <cstdint>
#include "sm100.cuh"

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

// Exclusive prefix sum over the threads of the block (blockDim.x a multiple of 32,
// at most 1024).  `sh` holds one slot per warp plus one for the total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const uint32_t inc = warp_incl_scan(v);
  if (lane == 31) sh[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < nw ? sh[lane] : 0u;
    const uint32_t xi = warp_incl_scan(x);
    if (lane < nw) sh[lane] = xi - x;
    if (lane == nw - 1) sh[32] = xi;
  }
  __syncthreads();
  const uint32_t r = sh[warp] + inc - v;
  if (total) *total = sh[32];
  __syncthreads();
  return r;
}

// One CTA per row: find the per-row threshold key by a two-level radix select on the
// 15-bit magnitude key (bf16 bits & 0x7FFF, which orders non-NaN |w| exactly), then
// apply the tie rule and write the row's bitmap words (row-major, K/64 words per row).
__global__ void __launch_bounds__(kEncThreads) encode_mask_kernel(const uint16_t* __restrict__ W,
                                                                  int K, int keep,
                                                                  uint64_t* __restrict__ bits,
                                                                  int* status) {
  extern __shared__ uint16_t keys[];  // K entries
  __shared__ uint32_t hist[256];
  __shared__ uint32_t scan_sh[33];
  __shared__ uint32_t s_hi, s_need, s_thr, s_eqkeep;
  const int row = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(W + static_cast<size_t>(row) * K);
  bool nan = false;
  for (int v = threadIdx.x; v < K / 8; v += blockDim.x) {
    const uint4 q = src[v];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint16_t k0 = static_cast<uint16_t>(w[h] & 0x7FFFu);
      const uint16_t k1 = static_cast<uint16_t>((w[h] >> 16) & 0x7FFFu);
      nan |= (k0 > 0x7F80u) | (k1 > 0x7F80u);
      keys[8 * v + 2 * h] = k0;
      keys[8 * v + 2 * h + 1] = k1;
    }
  }
  if (nan) atomicOr(status, DEV_ERR_NAN);
  for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  // level 1: top 8 bits of the key
  for (int c = threadIdx.x; c < K; c += blockDim.x) atomicAdd(&hist[keys[c] >> 7], 1u);
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t above = 0;
    int b = 255;
    for (; b > 0; --b) {
      if (above + hist[b] >= static_cast<uint32_t>(keep)) break;
      above += hist[b];
    }
    s_hi = b;
    s_need = keep - above;
  }
  __syncthreads();
  for (int b = threadIdx.x; b < 128; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  // level 2: low 7 bits among keys in the selected top bin
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    const uint32_t k = keys[c];
    if ((k >> 7) == s_hi) atomicAdd(&hist[k & 127u], 1u);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t above = 0;
    int b = 127;
    for (; b > 0; --b) {
      if (above + hist[b] >= s_need) break;
      above += hist[b];
    }
    s_thr = (s_hi << 7) | static_cast<uint32_t>(b);
    s_eqkeep = s_need - above;  // how many entries equal to the threshold are kept
  }
  __syncthreads();
  const uint32_t thr = s_thr, eqkeep = s_eqkeep;
  const int nwords = K / 64;
  const int wpt = (nwords + blockDim.x - 1) / blockDim.x;  // words per thread, contiguous
  const int w0 = threadIdx.x * wpt;
  uint32_t eq = 0;
  for (int w = w0; w < min(w0 + wpt, nwords); ++w)
    for (int c = 0; c < 64; ++c) eq += keys[64 * w + c] == thr;
  uint32_t eq_before = block_excl_scan(eq, scan_sh, nullptr);
  for (int w = w0; w < min(w0 + wpt, nwords); ++w) {
    uint64_t word = 0;
    for (int c = 0; c < 64; ++c) {
      const uint32_t k = keys[64 * w + c];
      bool kept = k > thr;
      if (k == thr) {
        kept = eq_before < eqkeep;
        ++eq_before;
      }
      word |= static_cast<uint64_t>(kept) << c;
    }
    bits[static_cast<size_t>(row) * nwords + w] = word;
  }
}

// One warp per block: number of kept entries and the block's size in 16-byte units.
__global__ void encode_count_kernel(const uint64_t* __restrict__ bits, int nwords, int nblocks,
                                    uint32_t* __restrict__ size16,
                                    unsigned long long* __restrict__ nnz_total,
                                    unsigned int* __restrict__ max16) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= nblocks) return;
  const int i = b / nwords, j = b % nwords;
  uint32_t c = 0;
  for (int r = lane; r < kBlockRows; r += 32)
    c += __popcll(bits[static_cast<size_t>(i * kBlockRows + r) * nwords + j]);
  c = warp_sum(c);
  if (lane == 0) {
    size16[b] = (kBitmapBytes + 2 * c + 15) / 16;
    atomicAdd(nnz_total, static_cast<unsigned long long>(c));
    atomicMax(max16, (kBitmapBytes + 2 * c + 15) / 16);
  }
}

// Single CTA: offsets[b] = sum of size16 before b; offsets[nblocks] = total.
__global__ void __launch_bounds__(1024) encode_scan_kernel(const uint32_t* __restrict__ size16,
                                                           int nblocks,
                                                           uint32_t* __restrict__ offsets,
                                                           int* status) {
  __shared__ uint32_t sh[33];
  unsigned long long carry = 0;
  for (int base = 0; base < nblocks; base += blockDim.x) {
    const int b = base + threadIdx.x;
    const uint32_t v = b < nblocks ? size16[b] : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl_scan(v, sh, &tot);
    if (b < nblocks) offsets[b] = static_cast<uint32_t>(carry + ex);
    carry += tot;
  }
  if (threadIdx.x == 0) {
    offsets[nblocks] = static_cast<uint32_t>(carry);
    if (carry >= (1ull << 32)) atomicOr(status, DEV_ERR_RANGE);
  }
}

// One CTA of 128 threads per block: thread r writes the block's row word r, its kept
// values (row-major after the bitmap) and thread 0 the zero padding.
__global__ void __launch_bounds__(kBlockRows) encode_scatter_kernel(
    const uint16_t* __restrict__ W, int K, const uint64_t* __restrict__ bits,
    const uint32_t* __restrict__ offsets, uint8_t* __restrict__ blob) {
  __shared__ uint32_t sh[33];
  const int b = blockIdx.x, nwords = K / 64;
  const int i = b / nwords, j = b % nwords, r = threadIdx.x;
  const int grow = i * kBlockRows + r;
  const uint64_t word = bits[static_cast<size_t>(grow) * nwords + j];
  uint32_t nnz;
  const uint32_t rstart = block_excl_scan(__popcll(word), sh, &nnz);
  uint8_t* base = blob + static_cast<size_t>(offsets[b]) * 16;
  reinterpret_cast<uint64_t*>(base)[r] = word;
  uint16_t* vals = reinterpret_cast<uint16_t*>(base + kBitmapBytes) + rstart;
  const uint16_t* wrow = W + static_cast<size_t>(grow) * K + j * kBlockCols;
  int k = 0;
  for (uint64_t m = word; m; m &= m - 1) vals[k++] = wrow[__ffsll(static_cast<long long>(m)) - 1];
  if (r == 0) {
    const uint32_t end = (offsets[b + 1] - offsets[b]) * 16;
    for (uint32_t p = kBitmapBytes + 2 * nnz; p < end; ++p) base[p] = 0;
  }
}

// One CTA of 128 threads per block: expand to dense rows, pruned entries +0.0.
__global__ void __launch_bounds__(kBlockRows) decode_kernel(const uint8_t* __restrict__ blob,
                                                            const uint32_t* __restrict__ offsets,
                                                            int K, uint16_t* __restrict__ out) {
  __shared__ uint32_t sh[33];
  const int b = blockIdx.x, nwords = K / 64;
  const int i = b / nwords, j = b % nwords, r = threadIdx.x;
  const uint8_t* base = blob + static_cast<size_t>(offsets[b]) * 16;
  const uint64_t word = reinterpret_cast<const uint64_t*>(base)[r];
  const uint32_t rstart = block_excl_scan(__popcll(word), sh, nullptr);
  const uint16_t* vals = reinterpret_cast<const uint16_t*>(base + kBitmapBytes) + rstart;
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(i * kBlockRows + r) * K +
                                        j * kBlockCols);
  int k = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 8 * q + 2 * e;
      uint32_t lo = 0, hi = 0;
      if ((word >> c) & 1) lo = vals[k++];
      if ((word >> (c + 1)) & 1) hi = vals[k++];
      o[e] = lo | (hi << 16);
    }
    dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace salr
