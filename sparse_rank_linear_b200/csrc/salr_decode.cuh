// salr_decode.cuh - Stage 1 of the SALR layer (technical summary, Methodology 4): a
// 128 x 64 block of the pruned weight rebuilt from its bitmap and its compact values.
//
// Block layout (include/salr.h): 128 uint64 bitmap words (word r, bit c marks row r,
// column c as kept), then the kept values as bf16, ordered by row quarter (rows 32q ..
// 32q + 31), then by 4-column group ("nibble" n: columns 4n .. 4n + 3), then by row, then
// by column.  One warp rebuilds one quarter with one thread per row:
//
// * Positions: the thread counts the kept entries of each of its row's 16 nibbles (a
//   SWAR popcount, 4 bits per nibble, spread to bytes), and four warp scans of those
//   byte-packed counts give, for every nibble column, how many values the quarter's
//   earlier rows hold there and how many the whole column holds.  With the values of the
//   block's earlier quarters (the popcount of their bitmap words) that gives the start
//   of every (row, nibble) run: the lookup the pages' decoder reads beside the bitmap.
// * Expansion, per nibble: the three 32-bit words from the 4-byte boundary at or below
//   the run's first value, shifted by a halfword when that value is odd, are spread over
//   the nibble's four columns by byte permutes whose selectors come from a 16-entry table
//   (one 8-byte entry per bitmap nibble).  Columns whose mask bit is clear come out +0.
//
// A warp's nibble-n runs lie side by side (about 2 values a row), so its 32 window loads
// touch about 32 consecutive words: few bank conflicts.  And a thread holding a whole row
// is the fragment tcgen05.st 32x32b writes to one TMEM lane, so the small-M kernel puts
// the rebuilt block straight into tensor memory as the MMA's A operand.
#pragma once
#include <cstdint>
#include "salr_block.cuh"
#include "sm100.cuh"

namespace salr {

// Selectors of one nibble's expansion.  A nibble whose kept values v0, v1, ... sit, in
// order, in the window (L0, L1) expands as
//   columns 0, 1 = prmt(L0, 0, PAT(n & 3))
//   columns 2, 3 = prmt(prmt(L0, L1, PAIR(popc(n & 3))), 0, PAT(n >> 2))
// where PAT(v), v the 2-bit mask of two columns, is 0x4444 / 0x4410 / 0x1044 / 0x3210
// (both zero, first value low, first value high, both values; selector 4 reads the zero
// operand) and PAIR(s) = 0x3210 + 0x2222 s brings values s, s + 1 to the bottom.  Entry
// n of the table: {PAT(n & 3) | PAT(n >> 2) << 16, PAIR(popc(n & 3))}.
__device__ __forceinline__ uint32_t pat2(uint32_t v) {
  return v == 0 ? 0x4444u : v == 1 ? 0x4410u : v == 2 ? 0x1044u : 0x3210u;
}
__device__ __forceinline__ uint2 nibble_entry(uint32_t n) {
  return make_uint2(pat2(n & 3u) | (pat2(n >> 2) << 16), 0x3210u + 0x2222u * __popc(n & 3u));
}

// Where one thread's row of a block quarter finds its values.
struct QuarterPos {
  uint64_t word;    // the row's bitmap word
  uint32_t ex[4];   // nibble n's values in the quarter's earlier rows (byte-packed)
  uint32_t tot[4];  // nibble n's values in the whole quarter (byte-packed)
  uint32_t qb;      // the block's values in rows before the quarter
};

// byte of nibble n in a byte-packed count: word (n & 1) + 2 (n >> 3), byte (n >> 1) & 3
__device__ __forceinline__ uint32_t nib_field(const uint32_t (&e)[4], int n) {
  return (e[(n & 1) + 2 * (n >> 3)] >> (8 * ((n >> 1) & 3))) & 0xFFu;
}

// Positions of lane `lane`'s row 32q + lane.  bm: the block's 128 bitmap words.  Called
// by all 32 lanes of a warp.
__device__ __forceinline__ QuarterPos quarter_pos(const uint64_t* bm, int q, int lane) {
  QuarterPos qp;
  qp.word = bm[32 * q + lane];
  uint32_t qb = 0;
  for (int rr = lane; rr < 32 * q; rr += 32) qb += __popcll(bm[rr]);
  qp.qb = warp_sum(qb);
  // 4-bit kept counts of the 16 nibbles, then spread to bytes (a quarter's column sum is
  // at most 128 and fits a byte)
  uint64_t x = qp.word - ((qp.word >> 1) & 0x5555555555555555ull);
  x = (x & 0x3333333333333333ull) + ((x >> 2) & 0x3333333333333333ull);
  const uint32_t lo = static_cast<uint32_t>(x), hi = static_cast<uint32_t>(x >> 32);
  const uint32_t e[4] = {lo & 0x0F0F0F0Fu, (lo >> 4) & 0x0F0F0F0Fu, hi & 0x0F0F0F0Fu,
                         (hi >> 4) & 0x0F0F0F0Fu};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t s = warp_incl_scan(e[k]);
    qp.tot[k] = __shfl_sync(0xffffffffu, s, 31);
    qp.ex[k] = s - e[k];
  }
  return qp;
}

// Position (in values from the start of the block's value array) of the first value of
// nibble n of this thread's row, for n = 0 .. 15 in order: start with base = qp.qb and
// call once per nibble.
__device__ __forceinline__ uint32_t nib_pos(const QuarterPos& qp, int n, uint32_t& base) {
  const uint32_t p = base + nib_field(qp.ex, n);
  base += nib_field(qp.tot, n);
  return p;
}

// Expansion of this thread's row: sink(n, w0, w1) receives columns 4n, 4n+1 (w0) and
// 4n+2, 4n+3 (w1) as bf16 pairs, low half the lower column, for n = 0 .. 15.  The value
// array must be readable 12 bytes past its last value (the windows of the last runs);
// bytes read there only meet columns whose mask bit is clear.
// status / vals_bytes: the status word and the bytes readable from vals (the block, its
// padding and whatever the caller's buffer holds after it), for the checks of debug
// builds: a window that would reach past vals_bytes is flagged and read from the start.
template <class Sink>
__device__ __forceinline__ void expand_quarter(const QuarterPos& qp, const uint8_t* vals,
                                               const uint2* nt, Sink&& sink,
                                               int* status = nullptr,
                                               uint32_t vals_bytes = 0xFFFFFFFFu) {
  const uint32_t* v32 = reinterpret_cast<const uint32_t*>(vals);
  uint32_t base = qp.qb;
  (void)status;
  (void)vals_bytes;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
#ifdef SALR_CHECKS
    uint32_t p = nib_pos(qp, n, base);
    if (!SALR_CHECK(((p >> 1) + 3) * 4 <= vals_bytes, status)) p = 0;
#else
    const uint32_t p = nib_pos(qp, n, base);
#endif
    const uint32_t nib = static_cast<uint32_t>(qp.word >> (4 * n)) & 15u;
    const uint32_t* w = v32 + (p >> 1);
    const uint32_t a0 = w[0], a1 = w[1], a2 = w[2];
    const uint32_t sh = (p & 1u) << 4;
    const uint32_t L0 = __funnelshift_r(a0, a1, sh), L1 = __funnelshift_r(a1, a2, sh);
    const uint2 en = nt[nib];
    sink(n, __byte_perm(L0, 0u, en.x), __byte_perm(__byte_perm(L0, L1, en.y), 0u, en.x >> 16));
  }
}

// Rebuild quarter q of a block (positions qp, from quarter_pos on the block's bitmap)
// into the 128-byte-swizzled K-major tile the MMA reads: row r at r * 128, 16-byte chunk
// c at position c ^ (r & 7).  A warp's 8 consecutive rows put a chunk into 8 different
// bank groups, so the stores are conflict-free.
__device__ __forceinline__ void expand_quarter_to_tile(const QuarterPos& qp, const uint8_t* blk,
                                                       int q, int lane, const uint2* nt,
                                                       uint8_t* tile, int* status = nullptr,
                                                       uint32_t blk_bytes = 0xFFFFFFFFu) {
  const int row = 32 * q + lane;
  uint8_t* dst = tile + row * 128;
  uint32_t r[4];
  expand_quarter(
      qp, blk + kBitmapBytes, nt,
      [&](int n, uint32_t w0, uint32_t w1) {
        r[2 * (n & 1)] = w0;
        r[2 * (n & 1) + 1] = w1;
        if (n & 1)
          *reinterpret_cast<uint4*>(dst + ((((n >> 1) ^ (row & 7))) << 4)) =
              make_uint4(r[0], r[1], r[2], r[3]);
      },
      status, blk_bytes - kBitmapBytes);
}

}  // namespace salr
