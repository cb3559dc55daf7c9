// salr_stream.cuh - persistent SALR layer kernel for small token counts (decode shapes).
//
// The layer salr_linear computes, Y = X (M (.) W)^T + (X A_cat) B_cat, organised for the
// HBM-bound regime (M <= 64) where decoding the bitmap blocks is the whole cost:
//
// * Work split: the weight's 128 x 64 blocks, in storage order, are cut into one
//   contiguous range per CTA (one CTA per SM, every SM the same number of blocks unless
//   the skew of stream_split is set).  A range covers one or more row-tile segments.  A
//   segment that does not cover a whole row tile adds its fp32 partial into the tile's
//   fp32 accumulator with vector reductions performed in L2, fences, and adds the number
//   of K blocks it covers to its 32-row quarter's count; the warp whose addition
//   completes the tile (no waiting) reads its sum, writes the bf16 output and clears the
//   accumulator and the count for the next call.
// * Stage 1 decode (SALR technical summary, Methodology 4): decoder warps work in
//   groups, each group on a different block so that several blocks are in flight.  Each
//   warp of a group rebuilds one 32-row quarter of the block, one row per thread
//   (salr_decode.cuh), and writes it with tcgen05.st into a TMEM slot: the rebuilt block
//   never passes through shared memory.
// * Stage 2: tcgen05 bf16 MMAs with A (the rebuilt block, 128 weight rows x 64) read from
//   that TMEM slot and B (the X tile) from shared memory, into a double-buffered TMEM
//   accumulator, pipelined against the decode through a ring of TMEM slots.
// * Concatenated adapter (Methodology 3): t = X A_cat is computed once per call.  The
//   lowest CTAs multiply a share of the K dimension each on the tensor cores and add
//   their parts into an fp32 buffer; when all parts have arrived every row tile reads t
//   back, rounds it to bf16 once and adds B_cat^T t^T to its accumulator with one more
//   MMA.  The CTAs that read t count themselves out; the last one clears the buffer and
//   both counts, so the scratch is zero again when the kernel ends, whatever the host
//   did in between (a replayed graph included).
// * Consecutive calls overlap (programmatic dependent launch): a CTA fetches its first
//   compact blocks and rebuilds its first blocks before waiting for the previous kernel
//   of the stream, and touches X, the adapters, the scratch and Y only after that wait.
//
// The only cross-CTA wait is for t, on the t-share CTAs, which finish their share without
// waiting on anything.  Every wait is bounded.
//
// Warp roles: 0 TMA producer, 1 TMEM allocator + adapter MMAs, 2-5 epilogue (also the
// adapter's t share), 6-25 decoders (a warp may only reach the TMEM lanes
// 32 (warp % 4) .. + 31, so the four warps of a decoder group, consecutive, cover the
// four quarters), 26-30 the MMA issuers of the five decoder groups.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "salr_codec.cuh"
#include "salr_decode.cuh"
#include "sm100.cuh"

namespace salr {

constexpr int kStreamFixedWarps = 6;  // producer, MMA, 4 epilogue warps
constexpr int kStreamGroups = 5;  // decoder groups, each decodes a different block
constexpr int kStreamMaxUnitsPerCta = 4096;
constexpr int kStreamMaxA = 16;  // rebuilt-block ring (TMEM slots)
constexpr int kStreamMaxC = 16;  // compact-block ring (super-slots of up to 4 blocks)
constexpr int kStreamMaxBpc = 4;  // blocks per bulk copy
constexpr int kStreamCtrlBytes = 2048;

struct StreamParams {
  const uint16_t* X;     // M x K bf16 activations (X tiles are read with ordinary loads)
  const uint8_t* blob;
  const uint32_t* offsets;
  uint16_t* Y;
  float* acc;            // [RT x 128 x BNT] fp32 sums of split row tiles, zero between calls
  uint32_t* counters;    // [RT x 4] segments arrived per split tile and 32-row quarter, zero between calls
  float* tacc;           // [R16 x BNT] fp32 accumulator of t = X A_cat (rank-major), zero between calls
  uint32_t* tflag;       // [2]: t parts arrived, CTAs done reading t; zero between calls
  int* status;
  int N, K, M, R, R16;
  int kblocks;  // K / 64
  int RT;       // N / 128
  int units;    // RT * kblocks
  int tshare;   // CTAs 0 .. tshare-1 compute a share of t (tshare = min(grid, kblocks))
  int treaders;  // CTAs that start a row tile (and read t): see stream_t_readers
  int skew;      // S of stream_split (0: equal ranges)
  int twant;     // t parts the readers wait for: tshare (more only in failure tests)
  int cbuf;     // bytes of a super-slot: bpc compact blocks + 32, multiple of 1024
  int bpc;      // compact blocks per bulk copy (1 .. 4)
  int bcbuf;    // bytes of the B_cat^T tile / t-share buffer (0 without adapter), x1024
  int sa;       // entries of the decoded-tile ring (tile + X tile each)
  int sc;       // entries of the compact-block ring
};

template <int BNT>
struct StreamLayout {
  static constexpr int kXbuf = BNT * 128;
  static constexpr int kAent = kXbuf;                  // one ring entry: the block's X tile
  static constexpr int kTbuf = BNT * 256;              // t as [BNT x 128] bf16, two chunks
  // TMEM columns: two accumulators and the t share (BNT each), then, from a multiple of
  // 32, the ring of rebuilt blocks (32 columns each: 64 bf16 per lane)
  __host__ __device__ static constexpr uint32_t a_col() { return (3 * BNT + 31) / 32 * 32; }
  __host__ __device__ static constexpr uint32_t tmem_cols(int sa) {
    const uint32_t need = a_col() + 32u * static_cast<uint32_t>(sa);
    return need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
  }
  // B_cat^T tile [128 x R16] and, at kernel start, the t-share stage (A_cat block + X)
  __host__ __device__ static int bcat_bytes(int R16) {
    if (R16 == 0) return 0;
    const int a = 256 * R16, b = 16384 + kXbuf;
    return ((a > b ? a : b) + 1023) / 1024 * 1024;
  }
  // layout: [X ring: sa x X tile] [C ring: sc x cbuf] [t] [B_cat] [ctrl] [nibble table]
  __host__ __device__ static int c_off(int sa) { return sa * kAent; }
  __host__ __device__ static int fixed_off(int cbuf, int sa, int sc) { return c_off(sa) + sc * cbuf; }
  __host__ __device__ static int smem_bytes(int cbuf, int bcbuf, int sa, int sc) {
    return fixed_off(cbuf, sa, sc) + kTbuf + bcbuf + kStreamCtrlBytes + 128 /*nibbles*/ +
           1024 /*align*/;
  }
};

struct StreamCtrl {
  uint64_t cfull[kStreamMaxC], cempty[kStreamMaxC];
  uint64_t dec[kStreamMaxA], aempty[kStreamMaxA];
  uint64_t gdone[kStreamGroups][2];  // a group's MMAs of a segment on accumulator x done
  uint64_t gfin[kStreamGroups];      // a group's last MMAs done (before TMEM is freed)
  uint64_t adone[2];                 // the adapter MMAs of a segment on accumulator x done
  uint64_t accempty[2];              // accumulator x drained and zeroed by the epilogue
  uint64_t bcfull, bcempty, tready, tsfull, tsfree, tsdone, fin;
  uint32_t tmem;
  int abort;
  int flag[2];
  uint32_t boff[kStreamMaxC][4];  // byte offset of each block of a super-slot's copy
};

static_assert(sizeof(StreamCtrl) <= kStreamCtrlBytes, "control block");

__device__ __forceinline__ void stream_timeout(const StreamParams& p, StreamCtrl* c) {
  atomicOr(p.status, DEV_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c->abort) = 1;
}
__device__ __forceinline__ bool stream_aborted(StreamCtrl* c) {
  return *reinterpret_cast<volatile int*>(&c->abort) != 0;
}

// Bounded wait for a global flag written by another CTA (acquire at gpu scope).
__device__ __forceinline__ bool wait_global_flag(const uint32_t* flag, uint32_t want) {
  const long long t0 = clock64();
  for (;;) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == want) return true;
    if (clock64() - t0 > wait_limit()) return false;
    __nanosleep(64);
  }
}

// First block of CTA c when U blocks in storage order are cut into one contiguous range
// per CTA of a grid of G.  S = 0: equal ranges, c U / G.  S > 0: the ranges shrink
// linearly with the CTA index, CTA G - 1 taking about (1 - S / 256) of CTA 0's share
// (F(c) = U c (512 G - S c) / (G (512 G - S G)), S < 256): with programmatic launch the
// CTAs of a call start in index order as the SMs of the previous call free up, so the
// later ones have less time.
__host__ __device__ inline long long stream_split(long long U, int G, int S, int c) {
  if (S == 0) return (static_cast<long long>(c) * U) / G;
  return (U * c * (512ll * G - static_cast<long long>(S) * c)) /
         (static_cast<long long>(G) * (512ll * G - static_cast<long long>(S) * G));
}

// CTAs whose range holds the first block of some row tile (K blocks of KB per row tile):
// the CTAs that apply the adapter and so read t.
__host__ __device__ inline int stream_t_readers(long long U, int G, int KB, int S) {
  int n = 0;
  for (int c = 0; c < G; ++c) {
    const long long a = stream_split(U, G, S, c), b = stream_split(U, G, S, c + 1);
    n += ((a + KB - 1) / KB) * KB < b;
  }
  return n;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}


// a * b / c rounded down, a * b < 2^32 when fits32 (32-bit division is several times
// cheaper than the 64-bit routine; the even split of U units over G CTAs fits whenever
// U * G < 2^32, about 29 M blocks on 148 SMs)
__device__ __forceinline__ int mul_div(long long a, long long b, long long c, bool fits32) {
  return fits32 ? static_cast<int>(static_cast<uint32_t>(a) * static_cast<uint32_t>(b) /
                                   static_cast<uint32_t>(c))
                : static_cast<int>((a * b) / c);
}

template <int BNT, int NDEC>
__global__ void __launch_bounds__(32 * (kStreamFixedWarps + NDEC + kStreamGroups), 1)
    salr_stream_kernel(const __grid_constant__ StreamParams p,
                       const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB) {
  using L = StreamLayout<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SA = p.sa, SC = p.sc;
  auto xbuf = [&](int s) { return smem + s * L::kAent; };
  auto cbuf = [&](int s) { return smem + L::c_off(SA) + s * p.cbuf; };
  uint8_t* tbuf = smem + L::fixed_off(p.cbuf, SA, SC);
  uint8_t* bcbuf = tbuf + L::kTbuf;  // B_cat^T tile; at kernel start, the t-share stage
  StreamCtrl* ctrl = reinterpret_cast<StreamCtrl*>(bcbuf + p.bcbuf);
  uint2* ntab = reinterpret_cast<uint2*>(bcbuf + p.bcbuf + kStreamCtrlBytes);  // 16 x 8 B, 1 KB aligned

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool adapter = p.R > 0;
  const int G = gridDim.x, cta = blockIdx.x;
  const long long U = p.units;
  const bool fits32 = U * G < (1ll << 32);
  const int u0 = p.skew ? static_cast<int>(stream_split(U, G, p.skew, cta)) : mul_div(cta, U, G, fits32);
  const int u1 = p.skew ? static_cast<int>(stream_split(U, G, p.skew, cta + 1))
                        : mul_div(cta + 1, U, G, fits32);
  const int KB = p.kblocks;
  // t share of this CTA: K blocks cta, cta + tshare, ... (only CTAs below tshare)
  const int nts = (adapter && cta < p.tshare) ? (KB - cta + p.tshare - 1) / p.tshare : 0;
  const uint32_t kCols = L::tmem_cols(SA);  // 2 accumulators, t share, rebuilt-block ring
  // the producer's first batch of block offsets is requested before the set-up below
  uint32_t offv = 0, offx = 0;
  if (warp == 0) {
    offv = (u0 + lane <= p.units) ? __ldg(p.offsets + u0 + lane) : 0u;
    offx = (u0 + 32 <= p.units) ? __ldg(p.offsets + u0 + 32) : 0u;
  }

  if (warp >= 2 && warp < kStreamFixedWarps) {
    // one barrier per thread of the epilogue warps: the init fence waits for the thread's
    // earlier memory operations, so it is kept away from the producer's offset loads
    constexpr int WPG = NDEC / kStreamGroups;
    int i = threadIdx.x - 64;
    uint64_t* b = nullptr;
    uint32_t cnt = 1;
    if (i < SC) {
      b = &ctrl->cfull[i];
    } else if ((i -= SC) < SC) {
      b = &ctrl->cempty[i];
      cnt = p.bpc * WPG;  // every warp of its blocks
    } else if ((i -= SC) < SA) {
      b = &ctrl->dec[i];
      cnt = WPG;
    } else if ((i -= SA) < SA) {
      b = &ctrl->aempty[i];
    } else if ((i -= SA) < 2 * kStreamGroups) {
      b = &ctrl->gdone[i >> 1][i & 1];
    } else if ((i -= 2 * kStreamGroups) < kStreamGroups) {
      b = &ctrl->gfin[i];
    } else if ((i -= kStreamGroups) < 2) {
      b = &ctrl->adone[i];
    } else if ((i -= 2) < 2) {
      b = &ctrl->accempty[i];
      cnt = 4;
    } else {
      switch (i - 2) {
        case 0: b = &ctrl->bcfull; break;
        case 1: b = &ctrl->bcempty; break;
        case 2: b = &ctrl->tready; cnt = 4; break;
        case 3: b = &ctrl->tsfull; break;
        case 4: b = &ctrl->tsfree; break;
        case 5: b = &ctrl->tsdone; break;
        case 6: b = &ctrl->fin; break;
        default: break;
      }
    }
    if (b) {
      mbar_init(b, cnt);
      fence_mbar_init();
    }
    if (threadIdx.x == 64) {
      ctrl->abort = 0;
      ctrl->flag[0] = ctrl->flag[1] = 0;
    }
  }
  if (threadIdx.x < 16) ntab[threadIdx.x] = nibble_entry(threadIdx.x);
  if (warp == 1) tmem_alloc(&ctrl->tmem, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;
  const uint32_t tmem_ts = tmem + 2 * BNT;  // t^T share accumulator [128 ranks x BNT]
  const uint32_t tmem_a = tmem + L::a_col();  // rebuilt-block ring, 32 columns per slot

  if (warp == 0) {
    // ================================================================ TMA producer
    // Warp-uniform loop; lane 0 issues.  Block offsets are fetched 32 at a time by the
    // whole warp so that no copy waits on a dependent global load.  The t-share rounds
    // share their buffer with the B_cat tile, so round r+1 is issued once round r has
    // been consumed and the B_cat tile of a segment only after its last block.
    const uint32_t xbytes = BNT * 128;
    int ts_next = 0;  // next t-share round to issue (lane 0)
    bool dep = false;  // lane 0 has waited for the preceding kernel
    auto issue_ts = [&](int r) {
      const int kb = cta + r * p.tshare;
      mbar_arrive_expect_tx(&ctrl->tsfull, (p.R > 64 ? 16384u : 8192u) + xbytes);
      tma_load_2d(bcbuf, &tmA, 0, kb * 64, &ctrl->tsfull);
      if (p.R > 64) tma_load_2d(bcbuf + 8192, &tmA, 64, kb * 64, &ctrl->tsfull);
      tma_load_2d(bcbuf + 16384, &tmX, kb * 64, 0, &ctrl->tsfull);
    };
    // blocking: issue every remaining round, then wait until the last one is consumed
    // X, the adapters and everything after are touched only after the preceding kernel
    // of the stream has completed; the compact blocks before that need no wait
    auto dep_wait = [&]() {
      if (!dep) {
        griddep_wait();
        dep = true;
        if (nts > 0) issue_ts(ts_next++);
      }
    };
    auto finish_ts = [&]() -> bool {
      while (ts_next < nts) {
        if (!mbar_wait(&ctrl->tsfree, (ts_next - 1) & 1)) return false;
        issue_ts(ts_next++);
      }
      return nts == 0 || mbar_wait(&ctrl->tsfree, (nts - 1) & 1);
    };
    if (lane == 0) {
      prefetch_tmap(&tmX);
      if (adapter) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
      }
    }
    // Copies of `bpc` consecutive blocks at a time (one bulk copy costs the SM's copy
    // engine about the same time whatever its size, so few large copies stream faster
    // than many small ones).  Copy j lands in super-slot j % SC; the byte offset of each
    // of its blocks is written to boff[slot][k] before the copy's barrier arrival.
    const int nunits = u1 - u0, bpc = p.bpc;
    int nad = 0, obase = u0, ncopies = 0;
    uint32_t ps = 0, pph = 0;  // super-slot and phase of the next copy (lane 0)
    // segment cursor of the B_cat tiles: row tile si holds CTA positions [.., send)
    int si = u0 / KB, send = min(u1, (u0 / KB + 1) * KB) - u0;
    bool sfirst = u0 % KB == 0, sleft = nunits > 0;
    bool stop = false, bc_pending = false;
    for (int it0 = 0; it0 < nunits && !stop; it0 += bpc) {
      const int nb = min(bpc, nunits - it0);
      if (u0 + it0 + nb > obase + 32) {
        obase = u0 + it0;
        offv = (obase + lane <= p.units) ? __ldg(p.offsets + obase + lane) : 0u;
        offx = (obase + 32 <= p.units) ? __ldg(p.offsets + obase + 32) : 0u;
      }
      const int k0 = u0 + it0 - obase;  // 0 .. 31; k0 + nb <= 32
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t v = __shfl_sync(0xffffffffu, offv, (k0 + k) & 31);
        o[k] = (k0 + k < 32) ? v : offx;
      }
      const uint32_t oe = __shfl_sync(0xffffffffu, offv, (k0 + nb) & 31);
      const uint32_t o_end = (k0 + nb < 32) ? oe : offx;  // the copy's end
      int fail = 0;
      if (lane == 0) {
        if (ncopies >= SC) dep_wait();
        if (ts_next < nts && ts_next > 0 && mbar_test_wait(smem_u32(&ctrl->tsfree), (ts_next - 1) & 1))
          issue_ts(ts_next++);
        const int s = static_cast<int>(ps);
        if (!SALR_CHECK(o_end >= o[0] && (o_end - o[0]) * 16u + 32u <= static_cast<uint32_t>(p.cbuf),
                        p.status)) {
          *reinterpret_cast<volatile int*>(&ctrl->abort) = 1;
          fail = 1;
        } else if (!mbar_wait(&ctrl->cempty[s], pph ^ 1) || stream_aborted(ctrl)) {
          stream_timeout(p, ctrl);
          fail = 1;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < nb) ctrl->boff[s][k] = (o[k] - o[0]) * 16u;
          const uint32_t cb = (o_end - o[0]) * 16u;
          mbar_arrive_expect_tx(&ctrl->cfull[s], cb);
          bulk_g2s(cbuf(s), p.blob + static_cast<size_t>(o[0]) * 16, cb, &ctrl->cfull[s]);
          if (++ncopies == SC) dep_wait();
        }
        if (++ps == static_cast<uint32_t>(SC)) {
          ps = 0;
          pph ^= 1u;
        }
      }
      if (__shfl_sync(0xffffffffu, fail, 0)) {
        stop = true;
        break;
      }
      // B_cat tiles of the row tiles whose last block of this CTA has now been requested
      while (!stop && sleft && send <= it0 + nb) {
        if (adapter && sfirst) {
          int bfail = 0;
          if (lane == 0) {
            dep_wait();
            if (!finish_ts() || !mbar_wait(&ctrl->bcempty, (nad & 1) ^ 1)) {
              stream_timeout(p, ctrl);
              bfail = 1;
            } else {
              mbar_arrive_expect_tx(&ctrl->bcfull, 256u * p.R16);
              tma_load_2d(bcbuf, &tmB, si * 128, 0, &ctrl->bcfull);
              tma_load_2d(bcbuf + p.R16 * 128, &tmB, si * 128 + 64, 0, &ctrl->bcfull);
              bc_pending = true;
            }
          }
          ++nad;
          if (__shfl_sync(0xffffffffu, bfail, 0)) stop = true;
        }
        sleft = send < nunits;
        ++si;
        sfirst = true;
        send = min(send + KB, nunits);
      }
    }
    if (lane == 0) {
      dep_wait();
      if (!stop && !finish_ts()) stream_timeout(p, ctrl);
      if (stream_aborted(ctrl)) {
        // let copies this thread started land before the CTA may exit
        for (int s = 0; s < SC; ++s)
          if (ncopies > s) mbar_wait(&ctrl->cfull[(ncopies - 1 - s) % SC], ((ncopies - 1 - s) / SC) & 1);
        if (bc_pending) mbar_wait(&ctrl->bcfull, (nad - 1) & 1);
        if (ts_next > 0) mbar_wait(&ctrl->tsfull, (ts_next - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ adapter MMAs
    // The blocks' MMAs are issued by the decoder groups themselves (one issuing thread
    // per group: a thread takes ~40 cycles to issue one tcgen05.mma, so one thread for
    // all of them would cap the block rate).  This thread multiplies this CTA's t shares
    // as they land, then adds B_cat^T t^T into the accumulator of every segment that
    // starts a row tile.  All MMAs into an accumulator accumulate; the epilogue zeroes it
    // after draining it.
    if (lane == 0) {
      constexpr uint32_t idesc_mn = idesc_bf16(128, BNT, 1, 0);
      bool ok = true;
      int ts_done = 0;  // t-share rounds multiplied so far
      while (ok && ts_done < nts) {
        if (!mbar_wait(&ctrl->tsfull, ts_done & 1) || stream_aborted(ctrl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(bcbuf), x0 = smem_u32(bcbuf + 16384);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem_ts, smem_desc_sw128(a0 + 2048 * k, 8192, 1024),
                      smem_desc_sw128(x0 + 32 * k, 16, 1024), idesc_mn, (ts_done | k) != 0);
        mma_commit(&ctrl->tsfree);
        if (++ts_done == nts) mma_commit(&ctrl->tsdone);
      }
      int seg = 0, nad = 0;
      for (int u = u0; u < u1 && ok && adapter; ++seg) {
        const int i = u / KB, kba = u % KB;
        const int kbb = min(KB, kba + (u1 - u));
        if (kba == 0) {
          const int x = seg & 1;
          if (!mbar_wait(&ctrl->accempty[x], (seg >> 1) & 1) || !mbar_wait(&ctrl->tready, 0) ||
              !mbar_wait(&ctrl->bcfull, nad & 1) || stream_aborted(ctrl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + x * BNT;
          const uint32_t b0 = smem_u32(bcbuf), t0 = smem_u32(tbuf);
          for (int k = 0; k < p.R16 / 16; ++k)
            mma_bf16_ss(acc, smem_desc_sw128(b0 + 2048 * k, p.R16 * 128, 1024),
                        smem_desc_sw128(t0 + (k >> 2) * (BNT * 128) + (k & 3) * 32, 16, 1024),
                        idesc_mn, 1);
          mma_commit(&ctrl->bcempty);
          mma_commit(&ctrl->adone[x]);
          ++nad;
        }
        u = i * KB + kbb;
      }
      if (!ok) stream_timeout(p, ctrl);
      mma_commit(&ctrl->fin);
      if (!mbar_wait_idle(&ctrl->fin, 0, 200)) stream_timeout(p, ctrl);
    }
  } else if (warp < kStreamFixedWarps) {
    // ================================================================ epilogue
    // Four warps (2-5): this CTA's part of the shared t first, then the accumulators of
    // the CTA's segments in order (two TMEM accumulators alternate, so the MMAs of the
    // next segment run while one is drained).
    const int eg = 0;                             // epilogue group
    const int bar_id = 1 + eg;                    // named barrier of the group
    const bool lead = threadIdx.x == 64 + 128 * eg;
    const int q = warp & 3;                       // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;  // weight row within the tile; rank index for t
    bool t_read = false;          // this CTA has read t (it is one of t's readers)
    __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(p.Y);
    volatile int* gflag = &ctrl->flag[eg];
    // ---- 0. both accumulators start at zero (every MMA into them accumulates); their
    //         accempty phase 0 lets the first two segments' MMAs in
    auto zero_acc = [&](int x) {
#pragma unroll
      for (int c = 0; c < BNT; c += 8)
        tmem_st8(tmem + x * BNT + lane_base + c, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->accempty[x]);
    };
    zero_acc(0);
    zero_acc(1);
    griddep_wait();
    if (eg == 0) {
      bool ok = true;
      // ---- 1. this CTA's share of t = X A_cat: drain t^T from TMEM into the fp32 buffer
      if (nts > 0) {
        ok = mbar_wait(&ctrl->tsdone, 0);
        if (!ok) stream_timeout(p, ctrl);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          for (int c = 0; c < BNT; c += 16) {
            uint32_t v[16];
            tmem_ld16(tmem_ts + lane_base + c, v);
            tmem_ld_wait();
            if (r < p.R) {  // t is kept rank-major, [R16 x BNT]
#pragma unroll
              for (int e = 0; e < 16; e += 4)
                if (c + e < p.M)
                  red_add_v4f32(p.tacc + r * BNT + c + e, __uint_as_float(v[e]),
                                __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                                __uint_as_float(v[e + 3]));
            }
          }
        }
        // publish: the group's adds happen before the arrival (release, cumulative over
        // the barrier)
        named_bar(bar_id, 128);
        if (lead) {
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.tflag) : "memory");
        }
      }
      // ---- 2. if this CTA starts some row tile it applies the adapter: wait for every
      //         share of t and round it to bf16 into shared memory
      bool has_adapter_seg = false;
      for (int u = u0; u < u1; u = (u / KB + 1) * KB)
        if (u % KB == 0) has_adapter_seg = true;
      if (adapter && has_adapter_seg) {
        if (lead) *gflag = wait_global_flag(p.tflag, static_cast<uint32_t>(p.twant)) ? 1 : 0;
        named_bar(bar_id, 128);
        if (*gflag == 0) {
          if (lead) stream_timeout(p, ctrl);
        } else {
          // four tokens of one rank per 16-byte load, 4 loads per thread per L2 round
          // trip: a batch's loads go out before its shared-memory stores
          constexpr int kPerRank = BNT / 4;
          for (int f0 = r; f0 < kPerRank * p.R16; f0 += 128 * 4) {
            float4 v[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int f = f0 + 128 * g, j = f / kPerRank, m = 4 * (f % kPerRank);
              v[g] = (f < kPerRank * p.R16 && m < p.M && j < p.R)
                         ? __ldcg(reinterpret_cast<const float4*>(p.tacc + j * BNT + m))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int f = f0 + 128 * g, j = f / kPerRank, m0 = 4 * (f % kPerRank);
              if (f >= kPerRank * p.R16) continue;
              const int chunk = j >> 6, cc = j & 63;
              const float tv[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int m = m0 + e;
                uint8_t* dst = tbuf + chunk * (BNT * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                               (((cc >> 3) ^ (m & 7)) << 4) + (cc & 7) * 2;
                *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(tv[e]);
              }
            }
          }
          fence_proxy_async_smem();
        }
        t_read = *gflag != 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->tready);
      }
    }
    // ---- 3. the CTA's segments in order: wait until every decoder group with blocks in
    //         the segment (and the adapter, if the segment applies it) has seen its MMAs
    //         complete, drain the accumulator, zero it for its next segment, then write Y
    //         or, for a split tile, add the partial into the tile's fp32 sum in L2; the
    //         last of the tile's segments to count itself in writes Y and clears the sum
    int seg = 0;
    uint32_t gph = 0, aph = 0;  // phase parities of gdone[g][x] (bit 2g + x), adone[x] (bit x)
    for (int u = u0; u < u1; ++seg) {
      const int i = u / KB, kba = u % KB;
      const int kbb = min(KB, kba + (u1 - u));
      const int x = seg & 1;
      {
        const int itA = u - u0, nb = kbb - kba;  // the segment's blocks, by CTA position
        bool okw = true;
#pragma unroll
        for (int g = 0; g < kStreamGroups; ++g) {
          const int gg = (itA + g) % kStreamGroups;  // groups of blocks itA, itA + 1, ...
          if (g < nb) {
            const uint32_t bit = 1u << (2 * gg + x);
            okw = okw && mbar_wait_idle(&ctrl->gdone[gg][x], (gph & bit) ? 1u : 0u, 64);
            gph ^= bit;
          }
        }
        if (adapter && kba == 0) {
          okw = okw && mbar_wait_idle(&ctrl->adone[x], (aph >> x) & 1u, 64);
          aph ^= 1u << x;
        }
        if (!okw) stream_timeout(p, ctrl);
        okw = __all_sync(0xffffffffu, okw) && !stream_aborted(ctrl);
        named_bar(bar_id, 128);
        if (lead) *gflag = okw ? 2 : 0;
        named_bar(bar_id, 128);
        if (*gflag != 2) break;
        tc_fence_after();
        const size_t n = static_cast<size_t>(i) * 128 + r;
        if (!SALR_CHECK(n < static_cast<size_t>(p.N), p.status)) break;
        const bool whole = kba == 0 && kbb == KB;
        float* sum = p.acc + n * BNT;
#pragma unroll
        for (int c = 0; c < BNT; c += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + x * BNT + lane_base + c, v);
          tmem_ld_wait();
          if (whole) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c + e < p.M)
                Y[(c + e) * static_cast<size_t>(p.N) + n] =
                    __float2bfloat16_rn(__uint_as_float(v[e]));
          } else {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              if (c + e < p.M)
                red_add_v4f32(sum + c + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                              __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
        zero_acc(x);
        if (!whole) {
          // Each warp counts its 32 rows of the tile in on its own, by the K blocks its
          // segment covers: its additions are performed first (fence), and the warp whose
          // count completes the tile's K blocks reads the sum of these rows, writes Y and
          // clears the sum and the count for the next call.
          __threadfence();
          __syncwarp();
          uint32_t last = 0;
          if (lane == 0) {
            const uint32_t nb = static_cast<uint32_t>(kbb - kba);
            last = atomicAdd(p.counters + 4 * i + q, nb) + nb == static_cast<uint32_t>(KB);
          }
          if (__shfl_sync(0xffffffffu, last, 0)) {
#pragma unroll
            for (int c0 = 0; c0 < BNT; c0 += 16) {
              if (c0 < p.M) {
                float4 t4[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                  if (c0 + 4 * q4 < p.M)
                    t4[q4] = __ldcg(reinterpret_cast<const float4*>(sum + c0 + 4 * q4));
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                  const int c = c0 + 4 * q4;
                  if (c < p.M) {
                    const float tv[4] = {t4[q4].x, t4[q4].y, t4[q4].z, t4[q4].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                      if (c + e < p.M)
                        Y[(c + e) * static_cast<size_t>(p.N) + n] = __float2bfloat16_rn(tv[e]);
                    __stcg(reinterpret_cast<float4*>(sum + c), make_float4(0.f, 0.f, 0.f, 0.f));
                  }
                }
              }
            }
            if (lane == 0) p.counters[4 * i + q] = 0u;
          }
        }
      }
      u = i * KB + kbb;
    }
    // ---- 4. count this CTA out of t's readers; the last one clears t and both counts.
    //      Every warp's loads of t completed before its tready arrival, which the adapter
    //      MMAs and so the drain of the adapter segment above waited for.
    if (t_read && warp == 2 + 4 * eg) {
      uint32_t last = 0;
      if (lane == 0) {
        __threadfence();
        last = atomicAdd(p.tflag + 1, 1u) + 1u == static_cast<uint32_t>(p.treaders);
      }
      if (__shfl_sync(0xffffffffu, last, 0)) {
        __threadfence();
        float4* z = reinterpret_cast<float4*>(p.tacc);
        for (int e = lane; e < BNT * p.R16 / 4; e += 32) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0) {
          p.tflag[0] = 0u;
          p.tflag[1] = 0u;
        }
      }
    }
  } else {
    // ================================================================ decoders
    // NDEC warps in kStreamGroups groups of four consecutive warps; group g decodes blocks
    // g, g + groups, ... so that several blocks are in flight.  Warp w of a group rebuilds
    // rows 32 (w % 4) .. + 31 of its block, one row per thread, into the TMEM lanes of
    // the same numbers (the only lanes a warp may write).
    static_assert(NDEC == 4 * kStreamGroups, "four warps, one per row quarter, in each group");
    const int dw = warp - kStreamFixedWarps;
    const int nunits = u1 - u0;
    // ring slots and phases of group g's blocks it = g, g + groups, ...: both rings hold a
    // multiple of `groups` slots, so the slot advances by `groups` and wraps (with a phase
    // flip) exactly when it crosses a multiple of the ring size
    if (dw < NDEC) {
      const int g = dw >> 2, q = warp & 3;
      const uint32_t tab_sa = smem_u32(ntab);
      const uint32_t tlane = tmem_a + (static_cast<uint32_t>(32 * q) << 16);
      // block it lives in copy it / bpc (super-slot sc, phase phc) at block kc of it
      const int bpc = p.bpc;
      uint32_t sc = 0, phc = 0, sa = g, pha = 0;
      int kc = g;
      for (; kc >= bpc; kc -= bpc)
        if (++sc == static_cast<uint32_t>(SC)) {
          sc = 0;
          phc ^= 1u;
        }
      // no wait for the preceding kernel here: the decoders read only the compact blocks
      // (which no kernel that lets this one start early writes) and this CTA's TMEM, so
      // the first blocks are rebuilt while that kernel finishes
      for (int it = g; it < nunits && !stream_aborted(ctrl); it += kStreamGroups) {
        // (waiting warps sleep between tests, leaving the issue slots to the warps at work;
        // the first wait lasts until the first copies land)
        if (!mbar_wait_idle(&ctrl->cfull[sc], phc, it == g ? 32 : 20)) {
          stream_timeout(p, ctrl);
          break;
        }
        const uint8_t* cb = cbuf(sc) + ctrl->boff[sc][kc];
        const QuarterRuns qr = quarter_runs(reinterpret_cast<const uint64_t*>(cb), q, lane);
        // ---- the TMEM slot must be free: the MMAs of its previous block have completed
        if (!mbar_wait_idle(&ctrl->aempty[sa], pha ^ 1, 20)) {
          stream_timeout(p, ctrl);
          break;
        }
        tc_fence_after();
        const uint32_t ts = tlane + 32u * sa;
        uint32_t r[8];
        expand_runs(
            qr, smem_u32(cb + kBitmapBytes), tab_sa,
            [&](int n, uint32_t w0, uint32_t w1) {
              r[2 * (n & 3)] = w0;
              r[2 * (n & 3) + 1] = w1;
              if ((n & 3) == 3)
                tmem_st8(ts + 8 * (n >> 2), r[0], r[1], r[2], r[3], r[4], r[5], r[6], r[7]);
            },
            p.status, static_cast<uint32_t>(p.cbuf) - ctrl->boff[sc][kc] - kBitmapBytes);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ctrl->dec[sa]);
          mbar_arrive(&ctrl->cempty[sc]);
        }
        for (kc += kStreamGroups; kc >= bpc; kc -= bpc)
          if (++sc == static_cast<uint32_t>(SC)) {
            sc = 0;
            phc ^= 1u;
          }
        if ((sa += kStreamGroups) >= static_cast<uint32_t>(SA)) {
          sa -= SA;
          pha ^= 1u;
        }
      }
    } else {
      // ============================================================== MMA issuers
      // One warp per decoder group (a thread needs ~40 cycles to issue one tcgen05.mma,
      // and warps issue in parallel).  For each of its group's blocks, once the TMEM slot
      // is free: the warp loads the block's X tile (BNT tokens x 64, rows past M zero)
      // with ordinary loads into the slot's 128-byte-swizzled X buffer (a TMA per block
      // would cost the SM's copy engine as much as a compact-block copy); then lane 0,
      // once the four quarters are in TMEM, issues the block's four MMAs into the
      // accumulator of the block's segment.  Every MMA accumulates (the epilogue zeroes an
      // accumulator after draining it).  After the group's last block of a segment, lane 0
      // commits gdone[g][x] for the epilogue.
      const int g = dw - NDEC;
      uint32_t sa = g, pha = 0;
      int kbx = (u0 + g) % KB;  // the block's K block, for its X tile
      int seg = 0, seg_waited = -1;  // segment `seg` holds CTA positions [.., segEnd)
      int segEnd = min(u1, (u0 / KB + 1) * KB) - u0;
      constexpr uint32_t idesc = idesc_bf16(128, BNT, 0, 0);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xbuf(0)), 16, 1024);
      constexpr uint32_t kSlotStep = L::kAent >> 4;  // X descriptors differ in the address only
      constexpr int kXChunks = BNT * 8 / 32;  // 16-byte chunks of an X tile per lane
      static_assert(kXChunks % 4 == 0, "X chunks per lane in fours");
      bool issued = false;
      griddep_wait();
      for (int it = g; it < nunits; it += kStreamGroups) {
        while (it >= segEnd) {
          ++seg;
          segEnd = min(segEnd + KB, nunits);
        }
        const int x = seg & 1;
        int ok = 1;
        if (lane == 0) ok = mbar_wait_idle(&ctrl->aempty[sa], pha ^ 1, 20) && !stream_aborted(ctrl);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          if (lane == 0) stream_timeout(p, ctrl);
          break;
        }
        // ---- X tile of the block: row m (token) at m * 128, chunk c at (c ^ (m & 7)) * 16
        uint8_t* xb = xbuf(sa);
        if (!SALR_CHECK(kbx >= 0 && kbx < KB && sa < static_cast<uint32_t>(SA), p.status)) kbx = 0;
#pragma unroll
        for (int t0 = 0; t0 < kXChunks; t0 += 4) {  // 4 loads in flight per lane at a time
          uint4 v[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int e = lane + 32 * (t0 + t), m = e >> 3, c = e & 7;
            v[t] = m < p.M ? __ldg(reinterpret_cast<const uint4*>(
                                 p.X + static_cast<size_t>(m) * p.K + kbx * 64) + c)
                           : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int e = lane + 32 * (t0 + t), m = e >> 3, c = e & 7;
            *reinterpret_cast<uint4*>(xb + m * 128 + ((c ^ (m & 7)) << 4)) = v[t];
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (seg_waited != seg) {
            ok = mbar_wait(&ctrl->accempty[x], (seg >> 1) & 1);
            seg_waited = seg;
          }
          ok = ok && mbar_wait_idle(&ctrl->dec[sa], pha, 100);
          if (!ok) {
            stream_timeout(p, ctrl);
          } else {
            tc_fence_after();
            const uint32_t acc = tmem + x * BNT, ta = tmem_a + 32u * sa;
            const uint64_t dx = xdesc0 + sa * kSlotStep;
            mma_bf16_ts(acc, ta, dx, idesc, 1u);
            mma_bf16_ts(acc, ta + 8, dx + 2, idesc, 1u);
            mma_bf16_ts(acc, ta + 16, dx + 4, idesc, 1u);
            mma_bf16_ts(acc, ta + 24, dx + 6, idesc, 1u);
            mma_commit(&ctrl->aempty[sa]);
            if (it + kStreamGroups >= segEnd) mma_commit(&ctrl->gdone[g][x]);
            issued = true;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if ((sa += kStreamGroups) >= static_cast<uint32_t>(SA)) {
          sa -= SA;
          pha ^= 1u;
        }
        for (kbx += kStreamGroups; kbx >= KB;) kbx -= KB;
      }
      // every MMA this thread issued has completed before the TMEM can be freed
      if (lane == 0 && issued) {
        mma_commit(&ctrl->gfin[g]);
        if (!mbar_wait(&ctrl->gfin[g], 0)) stream_timeout(p, ctrl);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace salr
