// salr_stream.cuh - persistent SALR layer kernel for small token counts (decode shapes).
//
// The layer salr_linear computes, Y = X (M (.) W)^T + (X A_cat) B_cat, organised for the
// HBM-bound regime (M <= 64) where decoding the bitmap blocks is the whole cost:
//
// * Work split: the weight's 128 x 64 blocks, in storage order, are cut into one
//   contiguous range per CTA (one CTA per SM, every SM the same number of blocks).  A
//   range covers one or more row-tile segments.  A segment that does not cover a whole
//   row tile adds its fp32 partial into the tile's fp32 accumulator with vector
//   reductions performed in L2, fences, and counts itself in per 32-row quarter; the last
//   warp to arrive for a quarter (no waiting) reads its sum, writes the bf16 output and
//   clears the accumulator and the count for the next call.
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
//   compact blocks before waiting for the previous kernel of the stream, and touches X,
//   the adapters, the scratch and Y only after that wait.
//
// The only cross-CTA wait is for t, on the t-share CTAs, which finish their share without
// waiting on anything.  Every wait is bounded.
//
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2-5 epilogue (also the
// adapter's t share), 6.. decoders (a warp may only reach the TMEM lanes
// 32 (warp % 4) .. + 31, so the four warps of a decoder group, consecutive, cover the
// four quarters).
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
constexpr int kStreamMaxC = 16;  // compact-block ring

struct StreamParams {
  const uint8_t* blob;
  const uint32_t* offsets;
  uint16_t* Y;
  float* acc;            // [RT x 128 x BNT] fp32 sums of split row tiles, zero between calls
  uint32_t* counters;    // [RT x 4] segments arrived per split tile and 32-row quarter, zero between calls
  float* tacc;           // [BNT x R16] fp32 accumulator of t = X A_cat, zero between calls
  uint32_t* tflag;       // [2]: t parts arrived, CTAs done reading t; zero between calls
  int* status;
  int N, K, M, R, R16;
  int kblocks;  // K / 64
  int RT;       // N / 128
  int units;    // RT * kblocks
  int tshare;   // CTAs 0 .. tshare-1 compute a share of t (tshare = min(grid, kblocks))
  int treaders;  // CTAs that start a row tile (and read t): see stream_t_readers
  int cbuf;     // per-stage bytes for one compact block (bitmap + values), multiple of 1024
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
    return fixed_off(cbuf, sa, sc) + kTbuf + bcbuf + 1024 /*ctrl*/ + 128 /*nibbles*/ +
           1024 /*align*/;
  }
};

struct StreamCtrl {
  uint64_t cfull[kStreamMaxC], cempty[kStreamMaxC];
  uint64_t dec[kStreamMaxA], xfull[kStreamMaxA], aempty[kStreamMaxA];
  uint64_t accfull[2], accempty[2];
  uint64_t bcfull, bcempty, tready, tsfull, tsfree, tsdone, fin;
  uint32_t tmem;
  int abort;
  int flag[2];
};

static_assert(sizeof(StreamCtrl) <= 1024, "control block");

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
    if (clock64() - t0 > kWaitLimitCycles) return false;
    __nanosleep(64);
  }
}

// CTAs of a grid of G over U blocks in storage order (K blocks of KB per row tile) whose
// contiguous range [c U / G, (c + 1) U / G) holds the first block of some row tile: the
// CTAs that apply the adapter and so read t.
__host__ __device__ inline int stream_t_readers(long long U, int G, int KB) {
  int n = 0;
  for (int c = 0; c < G; ++c) {
    const long long a = (static_cast<long long>(c) * U) / G;
    const long long b = (static_cast<long long>(c + 1) * U) / G;
    n += ((a + KB - 1) / KB) * KB < b;
  }
  return n;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}


// CTA that owns unit u (block u in storage order) under the even split of U units.
__device__ __forceinline__ int owner_of(long long u, long long U, int G) {
  int c = static_cast<int>((u * G) / U);
  while (c + 1 < G && ((c + 1) * U) / G <= u) ++c;
  while (c > 0 && (c * U) / G > u) --c;
  return c;
}

template <int BNT, int NDEC>
__global__ void __launch_bounds__(32 * (kStreamFixedWarps + NDEC), 1)
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
  uint2* ntab = reinterpret_cast<uint2*>(bcbuf + p.bcbuf + 1024);  // 16 x 8 B nibble table

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool adapter = p.R > 0;
  const int G = gridDim.x, cta = blockIdx.x;
  const long long U = p.units;
  const int u0 = static_cast<int>((static_cast<long long>(cta) * U) / G);
  const int u1 = static_cast<int>((static_cast<long long>(cta + 1) * U) / G);
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      mbar_init(&ctrl->cfull[s], 1);
      mbar_init(&ctrl->cempty[s], NDEC / kStreamGroups);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&ctrl->dec[s], NDEC / kStreamGroups);
      mbar_init(&ctrl->xfull[s], 1);
      mbar_init(&ctrl->aempty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&ctrl->accfull[x], 1);
      mbar_init(&ctrl->accempty[x], 4);
    }
    mbar_init(&ctrl->bcfull, 1);
    mbar_init(&ctrl->bcempty, 1);
    mbar_init(&ctrl->tready, 4);
    mbar_init(&ctrl->tsfull, 1);
    mbar_init(&ctrl->tsfree, 1);
    mbar_init(&ctrl->tsdone, 1);
    mbar_init(&ctrl->fin, 1);
    ctrl->abort = 0;
    ctrl->flag[0] = ctrl->flag[1] = 0;
    fence_mbar_init();
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
    int it = 0, nad = 0, obase = u0;
    uint32_t ps = 0, pph = 0;  // compact-ring slot and phase of block `it` (lane 0)
    bool stop = false, bc_pending = false;
    for (int u = u0; u < u1 && !stop;) {
      const int i = u / KB, kba = u % KB;
      const int kbb = min(KB, kba + (u1 - u));
      for (int kb = kba; kb < kbb; ++kb, ++it) {
        const int unit = i * KB + kb;
        if (unit >= obase + 32) {
          obase = unit;
          offv = (obase + lane <= p.units) ? __ldg(p.offsets + obase + lane) : 0u;
          offx = (obase + 32 <= p.units) ? __ldg(p.offsets + obase + 32) : 0u;
        }
        const int k = unit - obase;
        const uint32_t o0 = __shfl_sync(0xffffffffu, offv, k);
        const uint32_t o1n = __shfl_sync(0xffffffffu, offv, (k + 1) & 31);
        const uint32_t o1 = (k + 1 < 32) ? o1n : offx;
        int fail = 0;
        if (lane == 0) {
          if (it >= SC) dep_wait();
          if (ts_next < nts && ts_next > 0 && mbar_test_wait(smem_u32(&ctrl->tsfree), (ts_next - 1) & 1))
            issue_ts(ts_next++);
          const int s = static_cast<int>(ps);
          if (!mbar_wait(&ctrl->cempty[s], pph ^ 1) || stream_aborted(ctrl)) {
            stream_timeout(p, ctrl);
            fail = 1;
          } else {
            const uint32_t cb = (o1 - o0) * 16u;
            mbar_arrive_expect_tx(&ctrl->cfull[s], cb);
            bulk_g2s(cbuf(s), p.blob + static_cast<size_t>(o0) * 16, cb, &ctrl->cfull[s]);
            if (it == SC - 1) dep_wait();
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
      }
      if (!stop && adapter && kba == 0) {
        int fail = 0;
        if (lane == 0) {
          dep_wait();
          if (!finish_ts() || !mbar_wait(&ctrl->bcempty, (nad & 1) ^ 1)) {
            stream_timeout(p, ctrl);
            fail = 1;
          } else {
            mbar_arrive_expect_tx(&ctrl->bcfull, 256u * p.R16);
            tma_load_2d(bcbuf, &tmB, i * 128, 0, &ctrl->bcfull);
            tma_load_2d(bcbuf + p.R16 * 128, &tmB, i * 128 + 64, 0, &ctrl->bcfull);
            bc_pending = true;
          }
        }
        ++nad;
        if (__shfl_sync(0xffffffffu, fail, 0)) stop = true;
      }
      u = i * KB + kbb;
    }
    if (lane == 0) {
      dep_wait();
      if (!stop && !finish_ts()) stream_timeout(p, ctrl);
      if (stream_aborted(ctrl)) {
        // let copies this thread started land before the CTA may exit
        for (int s = 0; s < SC; ++s)
          if (it > s) mbar_wait(&ctrl->cfull[(it - 1 - s) % SC], ((it - 1 - s) / SC) & 1);
        if (bc_pending) mbar_wait(&ctrl->bcfull, (nad - 1) & 1);
        if (ts_next > 0) mbar_wait(&ctrl->tsfull, (ts_next - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BNT, 0, 0);
      constexpr uint32_t idesc_mn = idesc_bf16(128, BNT, 1, 0);
      bool ok = true;
      int ts_done = 0;  // t-share rounds multiplied so far
      auto mma_ts = [&]() {
        tc_fence_after();
        const uint32_t a0 = smem_u32(bcbuf), x0 = smem_u32(bcbuf + 16384);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem_ts, smem_desc_sw128(a0 + 2048 * k, 8192, 1024),
                      smem_desc_sw128(x0 + 32 * k, 16, 1024), idesc_mn, (ts_done | k) != 0);
        mma_commit(&ctrl->tsfree);
        if (++ts_done == nts) mma_commit(&ctrl->tsdone);
      };
      // the t share is multiplied as soon as its data has landed (polled between blocks),
      // never ahead of decoded blocks: it is fetched only after the dependency wait
      // The block loop runs on one thread that shares its SM sub-partition with decoder
      // warps, so it is kept short: X descriptors differ from slot 0's only in the
      // start-address field (address >> 4, which never carries past its 14 bits in shared
      // memory), slot s's A operand is TMEM columns 32 s .. of the ring, and the slot index
      // and its phase parity advance without division.
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xbuf(0)), 16, 1024);
      constexpr uint32_t kSlotStep = L::kAent >> 4;
      uint32_t dec0 = smem_u32(&ctrl->dec[0]), xf0 = smem_u32(&ctrl->xfull[0]);
      int s = 0;
      uint32_t ph = 0;
      int seg = 0, nad = 0;
      for (int u = u0; u < u1 && ok && !stream_aborted(ctrl); ++seg) {
        const int i = u / KB, kba = u % KB;
        const int kbb = min(KB, kba + (u1 - u));
        const int x = seg & 1;
        if (!mbar_wait(&ctrl->accempty[x], ((seg >> 1) & 1) ^ 1)) {
          stream_timeout(p, ctrl);
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + x * BNT;
        for (int kb = kba; kb < kbb; ++kb) {
          if (ts_done < nts && mbar_test_wait(smem_u32(&ctrl->tsfull), ts_done & 1)) mma_ts();
          if (ts_done < nts) {
            // while the block is still being decoded, take the t share once it has landed
            const long long t0 = clock64();
            while (!mbar_test_wait(dec0 + 8 * s, ph)) {
              if (ts_done < nts && mbar_test_wait(smem_u32(&ctrl->tsfull), ts_done & 1)) mma_ts();
              if (clock64() - t0 > kWaitLimitCycles || stream_aborted(ctrl)) {
                ok = false;
                break;
              }
              __nanosleep(32);
            }
            if (!ok) {
              stream_timeout(p, ctrl);
              break;
            }
          } else if (!mbar_try_wait(dec0 + 8 * s, ph) && !mbar_wait(&ctrl->dec[s], ph)) {
            stream_timeout(p, ctrl);
            ok = false;
            break;
          }
          if (!mbar_try_wait(xf0 + 8 * s, ph) && !mbar_wait(&ctrl->xfull[s], ph)) {
            stream_timeout(p, ctrl);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ta = tmem_a + 32u * s;
          const uint64_t dx = xdesc0 + s * kSlotStep;
          mma_bf16_ts(acc, ta, dx, idesc, kb != kba);
          mma_bf16_ts(acc, ta + 8, dx + 2, idesc, 1u);
          mma_bf16_ts(acc, ta + 16, dx + 4, idesc, 1u);
          mma_bf16_ts(acc, ta + 24, dx + 6, idesc, 1u);
          mma_commit(&ctrl->aempty[s]);
          if (++s == SA) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (adapter && kba == 0) {
          while (ok && ts_done < nts) {
            if (!mbar_wait(&ctrl->tsfull, ts_done & 1)) {
              ok = false;
              break;
            }
            mma_ts();
          }
          if (!ok || !mbar_wait(&ctrl->tready, 0) || !mbar_wait(&ctrl->bcfull, nad & 1)) {
            stream_timeout(p, ctrl);
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_u32(bcbuf), t0 = smem_u32(tbuf);
          for (int k = 0; k < p.R16 / 16; ++k)
            mma_bf16_ss(acc, smem_desc_sw128(b0 + 2048 * k, p.R16 * 128, 1024),
                        smem_desc_sw128(t0 + (k >> 2) * (BNT * 128) + (k & 3) * 32, 16, 1024),
                        idesc_mn, 1);
          mma_commit(&ctrl->bcempty);
          ++nad;
        }
        mma_commit(&ctrl->accfull[x]);
        u = i * KB + kbb;
      }
      while (ok && !stream_aborted(ctrl) && ts_done < nts) {
        if (!mbar_wait(&ctrl->tsfull, ts_done & 1)) {
          stream_timeout(p, ctrl);
          break;
        }
        mma_ts();
      }
      mma_commit(&ctrl->fin);
      if (!mbar_wait(&ctrl->fin, 0)) stream_timeout(p, ctrl);
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
    __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(p.Y);
    volatile int* gflag = &ctrl->flag[eg];
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
            if (r < p.R) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (c + e < p.M) atomicAdd(&p.tacc[(c + e) * p.R16 + r], __uint_as_float(v[e]));
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
        if (lead) *gflag = wait_global_flag(p.tflag, static_cast<uint32_t>(p.tshare)) ? 1 : 0;
        named_bar(bar_id, 128);
        if (*gflag == 0) {
          if (lead) stream_timeout(p, ctrl);
        } else {
          // 8 entries per thread per L2 round trip: a batch's loads go out before its
          // shared-memory stores
          for (int e0 = r; e0 < BNT * p.R16; e0 += 128 * 8) {
            float v[8];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const int e = e0 + 128 * g;
              const int m = e / p.R16, j = e % p.R16;
              v[g] = (e < BNT * p.R16 && m < p.M && j < p.R) ? __ldcg(&p.tacc[m * p.R16 + j])
                                                            : 0.0f;
            }
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const int e = e0 + 128 * g;
              if (e >= BNT * p.R16) continue;
              const int m = e / p.R16, j = e % p.R16;
              const int chunk = j >> 6, cc = j & 63;
              uint8_t* dst = tbuf + chunk * (BNT * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                             (((cc >> 3) ^ (m & 7)) << 4) + (cc & 7) * 2;
              *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(v[g]);
            }
          }
          fence_proxy_async_smem();
        }
        const bool tok = *gflag != 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->tready);
        if (tok) {
          // ---- count this CTA out of t's readers; the last one clears t and both counts
          //      (every reader's loads of t are complete before its count: the values
          //      are already in shared memory)
          __threadfence();
          named_bar(bar_id, 128);
          if (lead) {
            const uint32_t done = atomicAdd(p.tflag + 1, 1u) + 1u;
            *gflag = done == static_cast<uint32_t>(p.treaders) ? 3 : 1;
          }
          named_bar(bar_id, 128);
          if (*gflag == 3) {
            __threadfence();
            float4* z = reinterpret_cast<float4*>(p.tacc);
            for (int e = r; e < p.M * p.R16 / 4; e += 128) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lead) {
              p.tflag[0] = 0u;
              p.tflag[1] = 0u;
            }
          }
        }
      }
    }
    // ---- 3. segments of this group's parity: drain the accumulator, then write Y or, for
    //         a split tile, add the partial into the tile's fp32 sum in L2; the last of
    //         the tile's segments to count itself in writes Y and clears the sum
    int seg = 0;
    for (int u = u0; u < u1; ++seg) {
      const int i = u / KB, kba = u % KB;
      const int kbb = min(KB, kba + (u1 - u));
      const int x = seg & 1;
      {
        bool okw = mbar_wait(&ctrl->accfull[x], (seg >> 1) & 1);
        if (!okw) stream_timeout(p, ctrl);
        okw = __all_sync(0xffffffffu, okw) && !stream_aborted(ctrl);
        named_bar(bar_id, 128);
        if (lead) *gflag = okw ? 2 : 0;
        named_bar(bar_id, 128);
        if (*gflag != 2) break;
        tc_fence_after();
        const size_t n = static_cast<size_t>(i) * 128 + r;
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
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->accempty[x]);
        if (!whole) {
          // Each warp counts its 32 rows of the tile in on its own: its additions are
          // performed first (fence), and the warp that arrives last for these rows reads
          // their sum, writes Y and clears the sum and the count for the next call.
          __threadfence();
          __syncwarp();
          uint32_t last = 0;
          if (lane == 0) {
            const int c_first = owner_of(static_cast<long long>(i) * KB, U, G);
            const int segs =
                owner_of(static_cast<long long>(i) * KB + KB - 1, U, G) - c_first + 1;
            last = atomicAdd(p.counters + 4 * i + q, 1u) == static_cast<uint32_t>(segs - 1);
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
  } else {
    // ================================================================ decoders
    // NDEC warps in kStreamGroups groups of four consecutive warps; group g decodes blocks
    // g, g + groups, ... so that several blocks are in flight.  Warp w of a group rebuilds
    // rows 32 (w % 4) .. + 31 of its block, one row per thread, into the TMEM lanes of
    // the same numbers (the only lanes a warp may write).
    static_assert(NDEC == 4 * kStreamGroups, "four warps, one per row quarter, in each group");
    const int dw = warp - kStreamFixedWarps;
    const int g = dw >> 2, q = warp & 3;
    const int nunits = u1 - u0;
    const bool leader = (dw & 3) == 0 && lane == 0;  // issues the group's X-tile copies
    const uint32_t tlane = tmem_a + (static_cast<uint32_t>(32 * q) << 16);
    int last_x = -1;
    // ring slots and phases of this group's blocks it = g, g + groups, ...: both rings
    // hold a multiple of `groups` slots, so the slot advances by `groups` and wraps (with
    // a phase flip) exactly when it crosses a multiple of the ring size
    uint32_t sc = g, phc = 0, sa = g, pha = 0;
    int kbx = (u0 + g) % KB;  // the block's K block, for its X tile
    griddep_wait();
    for (int it = g; it < nunits && !stream_aborted(ctrl); it += kStreamGroups) {
      if (!mbar_wait(&ctrl->cfull[sc], phc)) {
        stream_timeout(p, ctrl);
        break;
      }
      const uint8_t* cb = cbuf(sc);
      const QuarterPos qp = quarter_pos(reinterpret_cast<const uint64_t*>(cb), q, lane);
      // ---- the TMEM slot must be free (its last MMAs complete); the group leader fetches X
      if (!mbar_wait(&ctrl->aempty[sa], pha ^ 1)) {
        stream_timeout(p, ctrl);
        break;
      }
      tc_fence_after();
      if (leader) {
        mbar_arrive_expect_tx(&ctrl->xfull[sa], BNT * 128);
        tma_load_2d(xbuf(sa), &tmX, kbx * 64, 0, &ctrl->xfull[sa]);
        last_x = it;
      }
      const uint32_t ts = tlane + 32u * sa;
      uint32_t r[8];
      expand_quarter(qp, cb + kBitmapBytes, ntab, [&](int n, uint32_t w0, uint32_t w1) {
        r[2 * (n & 3)] = w0;
        r[2 * (n & 3) + 1] = w1;
        if ((n & 3) == 3) tmem_st8(ts + 8 * (n >> 2), r[0], r[1], r[2], r[3], r[4], r[5], r[6], r[7]);
      });
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctrl->dec[sa]);
        mbar_arrive(&ctrl->cempty[sc]);
      }
      if ((sc += kStreamGroups) >= static_cast<uint32_t>(SC)) {
        sc -= SC;
        phc ^= 1u;
      }
      if ((sa += kStreamGroups) >= static_cast<uint32_t>(SA)) {
        sa -= SA;
        pha ^= 1u;
      }
      for (kbx += kStreamGroups; kbx >= KB;) kbx -= KB;
    }
    if (leader && last_x >= 0 && stream_aborted(ctrl))
      mbar_wait(&ctrl->xfull[last_x % SA], (last_x / SA) & 1);  // own copy lands first
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace salr
