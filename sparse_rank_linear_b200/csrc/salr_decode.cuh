// salr_decode.cuh - Stage 1 of the SALR layer (technical summary, Methodology 4): a
// 128 x 64 block of the pruned weight rebuilt from its bitmap and its compact values.
//
// Block layout (include/salr.h): 128 uint64 bitmap words (word r, bit c marks row r,
// column c as kept), then the kept values as bf16, ordered by row quarter (rows 32q ..
// 32q + 31), then by 4-column group ("nibble" n: columns 4n .. 4n + 3), then by row, then
// by column.  One warp rebuilds one quarter with one thread per row:
//
// * Runs: the thread counts the kept entries of each of its row's 16 nibbles (a SWAR
//   popcount, 4 bits per nibble, spread to bytes), and four warp scans of those
//   byte-packed counts give, for every nibble column, how many values the quarter's
//   earlier rows hold there and how many the whole column holds.  From these the thread
//   forms where its nibble-0 run starts and, byte-packed, the gap in values from each of
//   its runs to its next one (the column's values at and after its row plus the next
//   column's values before its row, at most 128): the lookup the pages' decoder reads
//   beside the bitmap, rebuilt in registers.
// * Expansion, per nibble: one pointer (shared-memory byte address of the run) gives the
//   4-byte-aligned window of three words and, in its low bits, the halfword shift that a
//   byte-funnel permute applies to it; the nibble's four columns then come out of byte
//   permutes whose selectors sit in a 16-entry table (8 bytes per bitmap nibble, the
//   table 256-byte aligned so that one byte permute forms an entry's address).  Columns
//   whose mask bit is clear come out +0.  The pointer then moves on by the run's gap.
//
// The rebuild is bound by the SM's integer pipe (about 10 integer instructions per nibble
// and 70 per row for the runs); the window loads of a warp's nibble-n runs lie side by
// side (about 2 values a row), so they touch about 32 consecutive words.  A thread holding
// a whole row is the fragment tcgen05.st 32x32b writes to one TMEM lane, so the small-M
// kernel puts the rebuilt block straight into tensor memory as the MMA's A operand.
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
struct QuarterRuns {
  uint64_t word;    // the row's bitmap word
  uint32_t gap[4];  // values from nibble n's run to nibble n + 1's (byte-packed, see nib_byte)
  uint32_t first;   // position of the nibble-0 run, in values from the block's first value
};

// byte of nibble n in a byte-packed set of four words: word (n & 1) + 2 (n >> 3), byte
// (n >> 1) & 3 (the order in which the SWAR popcount leaves the nibble counts)
__device__ __forceinline__ uint32_t nib_byte(const uint32_t (&e)[4], int n) {
  return __byte_perm(e[(n & 1) + 2 * (n >> 3)], 0u, 0x4440u | ((n >> 1) & 3));
}

__device__ __forceinline__ uint32_t mad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Runs of lane `lane`'s row 32q + lane.  bm: the block's 128 bitmap words.  Called by all
// 32 lanes of a warp.
__device__ __forceinline__ QuarterRuns quarter_runs(const uint64_t* bm, int q, int lane) {
  QuarterRuns qr;
  qr.word = bm[32 * q + lane];
  uint32_t qb = 0;  // the block's values in rows before the quarter
  for (int rr = lane; rr < 32 * q; rr += 32) qb += __popcll(bm[rr]);
  qb = __reduce_add_sync(0xffffffffu, qb);
  // 4-bit kept counts of the 16 nibbles, then spread to bytes (a quarter's column sum is
  // at most 128 and fits a byte)
  uint64_t x = qr.word - ((qr.word >> 1) & 0x5555555555555555ull);
  x = (x & 0x3333333333333333ull) + ((x >> 2) & 0x3333333333333333ull);
  const uint32_t lo = static_cast<uint32_t>(x), hi = static_cast<uint32_t>(x >> 32);
  const uint32_t e[4] = {lo & 0x0F0F0F0Fu, (lo >> 4) & 0x0F0F0F0Fu, hi & 0x0F0F0F0Fu,
                         (hi >> 4) & 0x0F0F0F0Fu};
  // four inclusive warp scans side by side; each step adds the value from `o` lanes down
  // as a multiply-add by a 0/1 lane mask (on the FMA pipe: the integer pipe is the
  // decoder's bottleneck)
  uint32_t s[4] = {e[0], e[1], e[2], e[3]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t m = lane >= o ? 1u : 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) s[k] = mad_u32(__shfl_up_sync(0xffffffffu, s[k], o), m, s[k]);
  }
  uint32_t ex[4], rest[4];  // per nibble: values in earlier rows / in this and later rows
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    ex[k] = s[k] - e[k];
    rest[k] = __shfl_sync(0xffffffffu, s[k], 31) - ex[k];  // no borrow: the total >= ex, bytewise
  }
  // gap(n) = rest(n) + ex(n + 1) <= 4 (32 - lane) + 4 lane: no carry between bytes.  The
  // next nibble of an even one is the same byte of the next word; of an odd one, the next
  // byte of the previous word (nibble 7's next, nibble 8, is byte 0 of word 2).
  qr.gap[0] = rest[0] + ex[1];
  qr.gap[1] = rest[1] + __funnelshift_r(ex[0], ex[2], 8);
  qr.gap[2] = rest[2] + ex[3];
  qr.gap[3] = rest[3] + (ex[2] >> 8);
  qr.first = qb + (ex[0] & 0xFFu);
  return qr;
}

// bytes c[1:0] .. c[1:0] + 3 of the 8-byte value {b, a}
__device__ __forceinline__ uint32_t byte_funnel(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32.f4e %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Expansion of this thread's row: sink(n, w0, w1) receives columns 4n, 4n+1 (w0) and
// 4n+2, 4n+3 (w1) as bf16 pairs, low half the lower column, for n = 0 .. 15.
// vals_sa: shared-memory address of the block's value array (4-byte aligned), which must
// be readable 12 bytes past its last value (the windows of the last runs; bytes read
// there only meet columns whose mask bit is clear).  tab_sa: shared-memory address of the
// 16 nibble_entry values, 256-byte aligned.  status / vals_bytes: the status word and
// the bytes readable from vals_sa, for the checks of debug builds: a window that would
// reach past vals_bytes is flagged and read from the start instead.
template <class Sink>
__device__ __forceinline__ void expand_runs(const QuarterRuns& qr, uint32_t vals_sa,
                                            uint32_t tab_sa, Sink&& sink, int* status = nullptr,
                                            uint32_t vals_bytes = 0xFFFFFFFFu) {
  (void)status;
  (void)vals_bytes;
  const uint32_t lo = static_cast<uint32_t>(qr.word), hi = static_cast<uint32_t>(qr.word >> 32);
  // table offsets (nibble value x 8), byte-packed like the counts
  const uint32_t ti[4] = {(lo << 3) & 0x78787878u, (lo >> 1) & 0x78787878u,
                          (hi << 3) & 0x78787878u, (hi >> 1) & 0x78787878u};
  uint32_t ptr = vals_sa + 2u * qr.first;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    uint32_t a = ptr & ~3u;
    if (!SALR_CHECK(a + 12u - vals_sa <= vals_bytes, status)) a = vals_sa;
    uint32_t a0, a1, a2;
    asm("ld.shared.u32 %0, [%3];\n\tld.shared.u32 %1, [%3+4];\n\tld.shared.u32 %2, [%3+8];"
        : "=r"(a0), "=r"(a1), "=r"(a2)
        : "r"(a));
    const uint32_t L0 = byte_funnel(a0, a1, ptr), L1 = byte_funnel(a1, a2, ptr);
    const uint32_t ea = __byte_perm(ti[(n & 1) + 2 * (n >> 3)], tab_sa, 0x7650u | ((n >> 1) & 3));
    uint32_t s01, pr;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(s01), "=r"(pr) : "r"(ea));
    sink(n, __byte_perm(L0, 0u, s01), __byte_perm(__byte_perm(L0, L1, pr), 0u, s01 >> 16));
    if (n < 15) ptr += 2u * nib_byte(qr.gap, n);
  }
}

// Rebuild quarter q of a block (runs qr, from quarter_runs on the block's bitmap) into the
// 128-byte-swizzled K-major tile the MMA reads: row r at r * 128, 16-byte chunk c at
// position c ^ (r & 7).  A warp's 8 consecutive rows put a chunk into 8 different bank
// groups, so the stores are conflict-free.
__device__ __forceinline__ void expand_runs_to_tile(const QuarterRuns& qr, uint32_t vals_sa,
                                                    int q, int lane, uint32_t tab_sa,
                                                    uint8_t* tile, int* status = nullptr,
                                                    uint32_t vals_bytes = 0xFFFFFFFFu) {
  const int row = 32 * q + lane;
  uint8_t* dst = tile + row * 128;
  uint32_t r[4];
  expand_runs(
      qr, vals_sa, tab_sa,
      [&](int n, uint32_t w0, uint32_t w1) {
        r[2 * (n & 1)] = w0;
        r[2 * (n & 1) + 1] = w1;
        if (n & 1)
          *reinterpret_cast<uint4*>(dst + ((((n >> 1) ^ (row & 7))) << 4)) =
              make_uint4(r[0], r[1], r[2], r[3]);
      },
      status, vals_bytes);
}

}  // namespace salr
