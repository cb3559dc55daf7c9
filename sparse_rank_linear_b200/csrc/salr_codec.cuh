// salr_codec.cuh - GPU encoder of the SALR bitmap block format, and the checks of a
// serialised image.
//
// Encoding (SALR technical summary, Methodology 1 and 4): each row of W keeps its
// `keep` entries of largest magnitude (ties to the lower column), the mask is stored as a
// bitmap and the kept values as a compact array, both cut into 128 x 64 blocks that are
// located through a per-block offset table.  The byte layout is the one written out in
// include/salr.h.  The scatter places each value where the decoders of salr_decode.cuh
// look for it; the dense expansion (salr_decode) lives with the layer kernels
// (expand_dense_kernel).
#pragma once
#include <cstdint>
#include "salr_block.cuh"
#include "salr_decode.cuh"
#include "sm100.cuh"

namespace salr {

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
// The bins are searched from the top by a prefix sum over the CTA, and each warp builds
// whole words with two ballots (columns lane and 32 + lane).
constexpr int kMaxWords = 512;  // K <= 32768
__global__ void __launch_bounds__(kEncThreads) encode_mask_kernel(const uint16_t* __restrict__ W,
                                                                  int K, int keep,
                                                                  uint64_t* __restrict__ bits,
                                                                  int* status) {
  extern __shared__ uint4 keys4[];  // K 16-bit keys
  uint16_t* keys = reinterpret_cast<uint16_t*>(keys4);
  __shared__ uint32_t hist[256];
  __shared__ uint32_t eqw[kMaxWords];
  __shared__ uint32_t scan_sh[33];
  __shared__ uint32_t s_hi, s_need, s_thr, s_eqkeep;
  const int row = blockIdx.x, t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int nwords = K / 64;
  const uint4* src = reinterpret_cast<const uint4*>(W + static_cast<size_t>(row) * K);
  hist[t] = 0;
  bool nan = false;
  for (int v = t; v < K / 8; v += kEncThreads) {
    uint4 q = src[v];
    q.x &= 0x7FFF7FFFu;
    q.y &= 0x7FFF7FFFu;
    q.z &= 0x7FFF7FFFu;
    q.w &= 0x7FFF7FFFu;
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) nan |= ((w4[h] & 0xFFFFu) > 0x7F80u) | ((w4[h] >> 16) > 0x7F80u);
    keys4[v] = q;
  }
  if (nan) atomicOr(status, DEV_ERR_NAN);
  __syncthreads();
  // level 1: top 8 bits of the key; thread t owns bin 255 - t
  for (int c = t; c < K; c += kEncThreads) atomicAdd(&hist[keys[c] >> 7], 1u);
  __syncthreads();
  {
    const uint32_t hb = hist[255 - t];
    const uint32_t above = block_excl_scan(hb, scan_sh, nullptr);
    if (above < static_cast<uint32_t>(keep) && static_cast<uint32_t>(keep) <= above + hb) {
      s_hi = 255 - t;
      s_need = keep - above;
    }
  }
  __syncthreads();
  if (t < 128) hist[t] = 0;
  __syncthreads();
  // level 2: low 7 bits among keys in the selected top bin; thread t < 128 owns bin 127 - t
  const uint32_t hi = s_hi;
  for (int c = t; c < K; c += kEncThreads) {
    const uint32_t k = keys[c];
    if ((k >> 7) == hi) atomicAdd(&hist[k & 127u], 1u);
  }
  __syncthreads();
  {
    const uint32_t hb = t < 128 ? hist[127 - t] : 0u;
    const uint32_t need = s_need;
    const uint32_t above = block_excl_scan(hb, scan_sh, nullptr);
    if (t < 128 && above < need && need <= above + hb) {
      s_thr = (hi << 7) | static_cast<uint32_t>(127 - t);
      s_eqkeep = need - above;  // how many entries equal to the threshold are kept
    }
  }
  __syncthreads();
  const uint32_t thr = s_thr, eqkeep = s_eqkeep;
  // entries equal to the threshold in each word, then their count before each word
  for (int wd = warp; wd < nwords; wd += kEncThreads / 32) {
    const uint32_t e0 = __ballot_sync(0xffffffffu, keys[64 * wd + lane] == thr);
    const uint32_t e1 = __ballot_sync(0xffffffffu, keys[64 * wd + 32 + lane] == thr);
    if (lane == 0) eqw[wd] = __popc(e0) + __popc(e1);
  }
  __syncthreads();
  {
    const int a = 2 * t, b = 2 * t + 1;
    const uint32_t ea = a < nwords ? eqw[a] : 0u, eb = b < nwords ? eqw[b] : 0u;
    const uint32_t ex = block_excl_scan(ea + eb, scan_sh, nullptr);
    if (a < nwords) eqw[a] = ex;
    if (b < nwords) eqw[b] = ex + ea;
  }
  __syncthreads();
  const uint32_t below = (1u << lane) - 1u;
  for (int wd = warp; wd < nwords; wd += kEncThreads / 32) {
    const uint32_t k0 = keys[64 * wd + lane], k1 = keys[64 * wd + 32 + lane];
    const uint32_t e0 = __ballot_sync(0xffffffffu, k0 == thr);
    const uint32_t e1 = __ballot_sync(0xffffffffu, k1 == thr);
    const uint32_t r0 = eqw[wd] + __popc(e0 & below);
    const uint32_t r1 = eqw[wd] + __popc(e0) + __popc(e1 & below);
    const uint32_t m0 = __ballot_sync(0xffffffffu, k0 > thr || (k0 == thr && r0 < eqkeep));
    const uint32_t m1 = __ballot_sync(0xffffffffu, k1 > thr || (k1 == thr && r1 < eqkeep));
    if (lane == 0)
      bits[static_cast<size_t>(row) * nwords + wd] = static_cast<uint64_t>(m0) |
                                                     (static_cast<uint64_t>(m1) << 32);
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

// Single CTA: offsets[b] = sum of size16 before b; offsets[nblocks] = total.  A total
// past the blob's capacity (cap16, in 16-byte units) is flagged, and the scatter then
// writes nothing past it.
__global__ void __launch_bounds__(1024) encode_scan_kernel(const uint32_t* __restrict__ size16,
                                                           int nblocks, unsigned long long cap16,
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
    if (carry >= (1ull << 32) || carry > cap16) atomicOr(status, DEV_ERR_RANGE);
  }
}

// One CTA of 128 threads per block.  Thread r (warp = row quarter, lane = row within it)
// writes its row's bitmap word, then its kept values, nibble by nibble, at the positions
// the decoders compute for them (values ordered by quarter, nibble, row, column; see
// salr_decode.cuh).  Thread 0 writes the zero padding.
__global__ void __launch_bounds__(kBlockRows) encode_scatter_kernel(
    const uint16_t* __restrict__ W, int K, const uint64_t* __restrict__ bits,
    const uint32_t* __restrict__ offsets, unsigned long long cap16, uint8_t* __restrict__ blob,
    int* status) {
  __shared__ uint64_t bm[kBlockRows];
  const int b = blockIdx.x, nwords = K / 64;
  if (offsets[b + 1] > cap16 || offsets[b] > offsets[b + 1]) return;
  const int i = b / nwords, j = b % nwords, r = threadIdx.x;
  const int warp = r >> 5, lane = r & 31;
  const uint64_t word = bits[static_cast<size_t>(i * kBlockRows + r) * nwords + j];
  bm[r] = word;
  uint8_t* base = blob + static_cast<size_t>(offsets[b]) * 16;
  reinterpret_cast<uint64_t*>(base)[r] = word;
  __syncthreads();
  const QuarterRuns qr = quarter_runs(bm, warp, lane);
  uint16_t* vals = reinterpret_cast<uint16_t*>(base + kBitmapBytes);
  const uint32_t cap_vals = ((offsets[b + 1] - offsets[b]) * 16 - kBitmapBytes) / 2;
  (void)cap_vals;
  (void)status;
  const uint4* src = reinterpret_cast<const uint4*>(W + static_cast<size_t>(i * kBlockRows + r) * K +
                                                    j * kBlockCols);
  uint32_t pos = qr.first;
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {  // 8 columns: two nibbles
    const uint4 q4 = src[c8];
    const uint32_t w4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = 2 * c8 + h;
      uint32_t at = pos;
      pos += nib_byte(qr.gap, n);
      const uint32_t nib = static_cast<uint32_t>(word >> (4 * n)) & 15u;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if ((nib >> c) & 1u) {
          if (SALR_CHECK(at < cap_vals, status))
            vals[at] = static_cast<uint16_t>(w4[2 * h + (c >> 1)] >> (16 * (c & 1)));
          ++at;
        }
    }
  }
  if (r == 0) {
    uint32_t nnz = 0;
    for (int rr = 0; rr < kBlockRows; ++rr) nnz += __popcll(bm[rr]);
    const uint32_t end = (offsets[b + 1] - offsets[b]) * 16;
    for (uint32_t q = kBitmapBytes + 2 * nnz; q < end; ++q) base[q] = 0;
  }
}

// Checks of an image read back by salr_load; the host has already checked that the offsets
// rise from 0 to the blob's end by at least one bitmap and at most one dense block each,
// so every read below stays inside its block.  One warp per block: the bitmap's population
// must give the block's stored size, every kept value must be a number, the padding must be
// zero, and each row's kept entries are added up for the row check.
__global__ void load_check_blocks_kernel(const uint8_t* __restrict__ blob,
                                         const uint32_t* __restrict__ offsets, int nwords,
                                         int nblocks, uint32_t* __restrict__ row_keep,
                                         unsigned long long* __restrict__ nnz_total,
                                         int* status) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= nblocks) return;
  const int i = b / nwords;
  const uint8_t* base = blob + static_cast<size_t>(offsets[b]) * 16;
  const uint32_t size = (offsets[b + 1] - offsets[b]) * 16;
  uint32_t c = 0;
  for (int r = lane; r < kBlockRows; r += 32) {
    const uint32_t n = __popcll(reinterpret_cast<const uint64_t*>(base)[r]);
    atomicAdd(&row_keep[i * kBlockRows + r], n);
    c += n;
  }
  c = warp_sum(c);
  if ((kBitmapBytes + 2 * c + 15) / 16 * 16 != size) {
    if (lane == 0) atomicOr(status, DEV_ERR_FORMAT);
    return;
  }
  // values then zero padding, 8 halves per 16-byte word
  const uint4* v = reinterpret_cast<const uint4*>(base + kBitmapBytes);
  bool nan = false, pad = false;
  for (uint32_t q = lane; q < (size - kBitmapBytes) / 16; q += 32) {
    const uint4 w = v[q];
    const uint32_t h2[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t val = (h2[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      if (8 * q + e < c) nan |= (val & 0x7FFFu) > 0x7F80u;
      else pad |= val != 0;
    }
  }
  nan = __any_sync(0xffffffffu, nan);
  pad = __any_sync(0xffffffffu, pad);
  if (lane == 0) {
    if (nan) atomicOr(status, DEV_ERR_NAN);
    if (pad) atomicOr(status, DEV_ERR_FORMAT);
    atomicAdd(nnz_total, static_cast<unsigned long long>(c));
  }
}

// One thread per row: every row keeps exactly `keep` entries.
__global__ void load_check_rows_kernel(const uint32_t* __restrict__ row_keep, int N,
                                       uint32_t keep, int* status) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N && row_keep[n] != keep) atomicOr(status, DEV_ERR_FORMAT);
}

}  // namespace salr
