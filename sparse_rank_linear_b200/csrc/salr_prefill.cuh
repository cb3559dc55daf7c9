// salr_prefill.cuh - the SALR layer for token counts above 64 (prefill shapes), where the
// tensor-core contraction dominates.  Up to three kernels per call:
//
// * expand_dense_kernel (from two token tiles on): the weight expanded once into a dense
//   bf16 N x K scratch, so that the layer kernel need not decode every block once per
//   token tile.  Persistent CTAs walk the blocks, staging the next by cp.async while
//   expanding the current.
// * salr_t_kernel: t = X A_cat, the concatenated adapter's down projection (SALR
//   technical summary, Methodology 3), computed once per call on the tensor cores and
//   rounded once to bf16 into a [M x 128] scratch.  Grid: token tiles x K splits.  With
//   several splits, each adds its fp32 part into a token-major sum in L2 (coalesced
//   reductions), and the last split of a token tile to count itself in converts the sum
//   and clears it.
// * salr_prefill_kernel: persistent, one CTA per SM over the work units (128-row weight
//   tile, token tile, K split).  Tiles are whole while every CTA gets one; the tiles of a
//   last, partial round are split along K so that their parts even out over the CTAs.
//   Tiles go token tile first or, when X outgrows about half the L2, in groups of row
//   tiles, token tile by token tile, so that the tiles in flight share few weight and X
//   tiles (pre_unit).
//   Fused mode: each 128 x 64 bitmap block arrives by one bulk copy and the matching X
//   tile by tensor TMA; decoder warps expand the block into the 128-byte-swizzled tile
//   (stage 1, Methodology 4) with the same device functions as the small-M kernel, and
//   tcgen05 MMAs multiply it (stage 2).  Dense mode: warp 0 copies the weight tiles from
//   the dense scratch by TMA into the same slots, and the decoders stay idle.  Wide dense
//   mode takes 256 weight rows per unit: each slot holds two 128-row tiles, two MMAs (one
//   TMEM accumulator each) share every X tile, and the two accumulators then serve one
//   unit instead of alternating between units.  The
//   adapter's up projection B_cat^T t^T runs as extra iterations of the same pipeline
//   after a unit's K blocks (on split 0).  The epilogue writes Y; a split unit adds into
//   a token-major fp32 sum in L2 whose last contributor writes Y.
//
// Orientation as in the small-M kernel: D[128 weight rows x BNT tokens] in TMEM, two
// accumulators used by alternate units.  Rings: compact blocks (producer -> decoders),
// decoded tiles (decoders or the dense loads -> MMA) and X tiles (X loader -> MMA), so
// that the copy latency and the decode of a block overlap the MMAs of earlier blocks;
// four decoder groups each work on a different block.  Warp roles (736 threads): 0
// compact-block or dense-tile producer, 1 TMEM allocator + MMA issuer, 2-5 epilogue, 6
// X-tile producer, 7-22 decoders.  Every wait is bounded; a timeout is recorded in the
// status word.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "salr_codec.cuh"
#include "salr_stream.cuh"
#include "sm100.cuh"

namespace salr {

constexpr int kPreDecoders = 16;
constexpr int kPreGroups = 4;                             // decoder groups (blocks in flight)
static_assert((kPreGroups & (kPreGroups - 1)) == 0, "group of iteration g is g & (groups - 1)");
constexpr int kPreThreads = 32 * (7 + kPreDecoders);      // + producer, MMA, 4 epilogue, X loader
constexpr int kPreMaxC = 8, kPreMaxA = 6, kPreMaxX = 4;    // ring depths
constexpr int kPreMaxKBlocks = 512;  // K <= 32768
constexpr int kPreCtrlBytes = 5120;
constexpr int kPreTileBytes = 16384;

struct PrefillParams {
  const uint8_t* blob;
  const uint32_t* offsets;
  uint16_t* Y;
  float* acc;          // [split tiles][BNT tokens][rows] fp32 sums, zero between calls
  uint32_t* counters;  // [split tiles][4] split arrivals per 32-row quarter, zero between calls
  int* status;
  int N, K, M, R16;
  int kblocks;         // K / 64
  int TT;              // token tiles
  int full;            // tiles 0 .. full - 1 are whole units
  int splits;          // K splits of each tile from `full` on (the split tiles)
  int units;           // split tiles x splits + full (split units first)
  int dense;           // 1: weight tiles come dense from tmW by TMA (no decoding)
  int wide;            // dense mode with 256-row tiles: each unit is two 128-row halves
                       // that share the X tiles, one TMEM accumulator per half
  int atile;           // bytes of a decoded-tile ring slot: 16 KB, or 32 KB when wide
  int rtiles;          // weight row tiles (of 128 or 256 rows)
  int group_rows;      // 0: tile t is (row tile t / TT, token tile t % TT).  Otherwise the
                       // tiles go in groups of group_rows row tiles, token tile by token
                       // tile, so that the tiles in flight share a few weight and X tiles
                       // that stay in L2
  int cbuf;            // bytes of a compact-block slot, multiple of 1024
  int sc, sa, sx;      // ring depths: compact blocks, decoded tiles, X tiles
};

struct PrefillCtrl {
  uint64_t cfull[kPreMaxC], cempty[kPreMaxC];
  uint64_t dec[kPreMaxA], aempty[kPreMaxA];
  uint64_t xfull[kPreMaxX], xempty[kPreMaxX];
  uint64_t accfull[2], accempty[2];  // the two TMEM accumulators: MMA -> epilogue -> MMA
  uint64_t adfull[kPreGroups];       // per decoder group: the B_cat^T copy it requested
  uint64_t fin;
  uint32_t tmem;
  int abort;
  uint32_t off[2][kPreMaxKBlocks + 1];  // block offsets of the current and the next unit
};
static_assert(sizeof(PrefillCtrl) <= kPreCtrlBytes, "control block");

// Shared-memory layout: [decoded tiles: sa x 16 KB][X tiles: sx x BNT*128][compact blocks:
// sc x cbuf][nibble table][control].
template <int BNT>
struct PrefillLayout {
  static constexpr int kXbuf = BNT * 128;
  // `sa` counts 16 KB units: ring slots x (atile / 16 KB)
  __host__ __device__ static int x_off(int sa) { return sa * kPreTileBytes; }
  __host__ __device__ static int c_off(int sa, int sx) { return x_off(sa) + sx * kXbuf; }
  __host__ __device__ static int table_off(int sa, int sx, int sc, int cbuf) {
    return c_off(sa, sx) + sc * cbuf;
  }
  __host__ __device__ static int smem_bytes(int sa, int sx, int sc, int cbuf) {
    return table_off(sa, sx, sc, cbuf) + 128 /*nibbles*/ + kPreCtrlBytes + 1024 /*align*/;
  }
};

__device__ __forceinline__ void pre_timeout(int* status, PrefillCtrl* c) {
  atomicOr(status, DEV_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c->abort) = 1;
}
__device__ __forceinline__ bool pre_aborted(PrefillCtrl* c) {
  return *reinterpret_cast<volatile int*>(&c->abort) != 0;
}

// Slot and phase of a ring walked in order (cheaper than dividing the iteration count).
struct RingCursor {
  uint32_t s = 0, ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++s == static_cast<uint32_t>(n)) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// One work unit: output tile t = (weight row tile i, token tile j), K split sidx of ns,
// and its K-block range.  Tiles below p.full are whole; each later tile is cut into
// p.splits consecutive units (the parts of one tile go to neighbouring CTAs).  The split
// units come first, so that their partial sums meet while the whole tiles that follow
// keep the tensor cores busy.
struct PreUnit {
  int t, i, j, sidx, ns, kb0, nk, nad;  // nad: adapter iterations (64 ranks each) after the K blocks
};
__device__ __forceinline__ PreUnit pre_unit(const PrefillParams& p, int u) {
  PreUnit w;
  const int nsu = p.units - p.full;  // split units
  if (u >= nsu) {
    w.t = u - nsu;
    w.sidx = 0;
    w.ns = 1;
  } else {
    w.t = p.full + u / p.splits;
    w.sidx = u % p.splits;
    w.ns = p.splits;
  }
  if (p.group_rows > 0) {
    const int per = p.group_rows * p.TT, g = w.t / per, r = w.t - g * per;
    const int rows = min(p.group_rows, p.rtiles - g * p.group_rows);  // the last group's
    w.i = g * p.group_rows + r % rows;
    w.j = r / rows;
  } else {
    w.j = w.t % p.TT;
    w.i = w.t / p.TT;
  }
  w.kb0 = static_cast<int>(static_cast<long long>(w.sidx) * p.kblocks / w.ns);
  const int kb1 = static_cast<int>(static_cast<long long>(w.sidx + 1) * p.kblocks / w.ns);
  w.nk = kb1 - w.kb0;
  w.nad = (p.R16 > 0 && w.sidx == 0) ? (p.R16 + 63) / 64 : 0;
  return w;
}

// Persistent: one CTA per SM takes units blockIdx.x, blockIdx.x + gridDim.x, ...  Every
// role walks the same sequence of iterations g (the K blocks of each unit, then its
// adapter chunks), so ring slot g % S and phase (g / S) & 1 agree between roles across
// units, and the rings run on from one unit into the next.  An adapter chunk is one more
// iteration: its decoder group copies 64 ranks of B_cat^T (an MN-major 128 x 64 tile)
// into the decoded-tile slot instead of decoding, the X loader copies the matching 64
// ranks of t, and its compact-block slot turn carries no data.  Accumulators alternate
// between two TMEM column ranges, so that the epilogue of one unit overlaps the MMAs of
// the next.
template <int BNT, bool WIDE>
__global__ void __launch_bounds__(kPreThreads, 1)
    salr_prefill_kernel(const __grid_constant__ PrefillParams p,
                        const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmT,
                        const __grid_constant__ CUtensorMap tmW) {
  using L = PrefillLayout<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SC = p.sc, SA = p.sa, SX = p.sx;
  const int AU = SA * (p.atile / kPreTileBytes);  // 16 KB units of the decoded-tile ring
  auto abuf = [&](int s) { return smem + s * p.atile; };
  auto xbuf = [&](int s) { return smem + L::x_off(AU) + s * L::kXbuf; };
  auto cbuf = [&](int s) { return smem + L::c_off(AU, SX) + s * p.cbuf; };
  uint8_t* tables = smem + L::table_off(AU, SX, SC, p.cbuf);
  // weight rows per unit: 128, or 256 (taken from the parameters in the wide kernel, which
  // as a run-time value keeps that kernel's registers within bounds)
  const int ROWS = WIDE ? 128 * (1 + (p.wide & 1)) : 128;
  uint2* ntab = reinterpret_cast<uint2*>(tables);  // 1 KB aligned
  PrefillCtrl* ctrl = reinterpret_cast<PrefillCtrl*>(tables + 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  constexpr int WPG = kPreDecoders / kPreGroups;
  constexpr uint32_t kCols = 2 * BNT;  // two accumulators

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      mbar_init(&ctrl->cfull[s], 1);
      mbar_init(&ctrl->cempty[s], WPG);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&ctrl->dec[s], p.dense ? 1 : WPG);  // dense: the producer's copy completes it
      mbar_init(&ctrl->aempty[s], 1);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(&ctrl->xfull[s], 1);
      mbar_init(&ctrl->xempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->accfull[b], 1);
      mbar_init(&ctrl->accempty[b], 4);
    }
    for (int g = 0; g < kPreGroups; ++g) mbar_init(&ctrl->adfull[g], 1);
    mbar_init(&ctrl->fin, 1);
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) ntab[threadIdx.x] = nibble_entry(threadIdx.x);
  if (warp == 1) tmem_alloc(&ctrl->tmem, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;

  if (warp == 0 && p.dense) {
    // ================================================================ dense weight-tile producer
    // The weights were expanded to a dense [N x K] scratch before this kernel: each
    // iteration's 128 x 64 tile (or adapter chunk of B_cat^T) goes by TMA straight into
    // the decoded-tile slot, and its arrival completes the slot's barrier.
    if (lane == 0) {
      prefetch_tmap(&tmW);
      if (p.R16 > 0) prefetch_tmap(&tmB);
      RingCursor ac;
      uint32_t g = 0, gi = 0;
      bool ok = true;
      for (int u = cta; u < p.units && ok; u += G) {
        const PreUnit w = pre_unit(p, u);
        for (int it = 0; it < w.nk + w.nad; ++it, ++g, ac.next(SA)) {
          const uint32_t sa = ac.s;
          if (!mbar_wait(&ctrl->aempty[sa], ac.ph ^ 1) || pre_aborted(ctrl)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctrl->dec[sa], static_cast<uint32_t>(p.atile));
#pragma unroll 1
          for (int hf = 0; hf < ROWS / 128; ++hf) {  // 128-row halves, 16 KB apart
            uint8_t* dst = abuf(sa) + hf * kPreTileBytes;
            const int row = w.i * ROWS + hf * 128;
            if (it < w.nk) {
              tma_load_2d(dst, &tmW, (w.kb0 + it) * 64, row, &ctrl->dec[sa]);
            } else {
              const int c = it - w.nk;
              tma_load_2d(dst, &tmB, row, c * 64, &ctrl->dec[sa]);
              tma_load_2d(dst + 8192, &tmB, row + 64, c * 64, &ctrl->dec[sa]);
            }
          }
          gi = g + 1;
        }
      }
      if (pre_aborted(ctrl)) {
        for (uint32_t x = gi > static_cast<uint32_t>(SA) ? gi - SA : 0; x < gi; ++x)
          mbar_wait(&ctrl->dec[x % SA], (x / SA) & 1);
      }
    }
  } else if (warp == 0) {
    // ================================================================ compact-block producer
    // Each unit's block offsets sit in one of two shared buffers: the whole warp starts
    // the copy of the next unit's offsets (cp.async) before lane 0 issues this unit's
    // blocks, and waits for it after, so the next unit's first copy goes out at once.
    uint32_t g = 0, gi = 0;  // iterations walked / slot turns issued
    RingCursor cc;           // lane 0's compact-ring cursor
    bool ok = true;
    int ob = 0;
    if (cta < p.units) {
      const PreUnit w = pre_unit(p, cta);
      const uint32_t* src = p.offsets + static_cast<size_t>(w.i) * p.kblocks + w.kb0;
      for (int t = lane; t <= w.nk; t += 32) ctrl->off[0][t] = src[t];
    }
    __syncwarp();
    for (int u = cta; u < p.units && ok; u += G) {
      const PreUnit w = pre_unit(p, u);
      if (u + G < p.units) {
        const PreUnit wn = pre_unit(p, u + G);
        const uint32_t* src = p.offsets + static_cast<size_t>(wn.i) * p.kblocks + wn.kb0;
        for (int t = lane; t <= wn.nk; t += 32) cp_async4(&ctrl->off[ob ^ 1][t], src + t);
      }
      if (lane == 0) {
        const uint32_t* off = ctrl->off[ob];
        for (int it = 0; it < w.nk + w.nad; ++it, cc.next(SC)) {
          const uint32_t s = cc.s;
          if (!mbar_wait(&ctrl->cempty[s], cc.ph ^ 1) || pre_aborted(ctrl)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          if (it < w.nk) {
            const uint32_t o0 = off[it], o1 = off[it + 1];
            mbar_arrive_expect_tx(&ctrl->cfull[s], (o1 - o0) * 16u);
            bulk_g2s(cbuf(s), p.blob + static_cast<size_t>(o0) * 16, (o1 - o0) * 16u,
                     &ctrl->cfull[s]);
          } else {
            mbar_arrive(&ctrl->cfull[s]);  // an adapter iteration: the turn carries no data
          }
          gi = g + it + 1;
        }
      }
      cp_async_wait_all();
      __syncwarp();  // the next unit's offsets, copied by every lane, are visible to lane 0
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      g += w.nk + w.nad;
      ob ^= 1;
    }
    cp_async_wait_all();
    if (lane == 0 && pre_aborted(ctrl)) {
      // let every copy this thread started land before the CTA can exit
      for (uint32_t x = gi > static_cast<uint32_t>(SC) ? gi - SC : 0; x < gi; ++x)
        mbar_wait(&ctrl->cfull[x % SC], (x / SC) & 1);
    }
  } else if (warp == 6) {
    // ================================================================ X / t tile producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      if (p.R16 > 0) prefetch_tmap(&tmT);
      uint32_t g = 0, gi = 0;
      RingCursor xc;
      bool ok = true, t_ready = false;
      for (int u = cta; u < p.units && ok; u += G) {
        const PreUnit w = pre_unit(p, u);
        for (int it = 0; it < w.nk + w.nad; ++it, ++g, xc.next(SX)) {
          const uint32_t s = xc.s;
          if (!mbar_wait(&ctrl->xempty[s], xc.ph ^ 1) || pre_aborted(ctrl)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          if (it == w.nk && !t_ready) {
            // t comes from the kernel launched just before this one, which may still run
            griddep_wait();
            t_ready = true;
          }
          mbar_arrive_expect_tx(&ctrl->xfull[s], L::kXbuf);
          if (it < w.nk)
            tma_load_2d(xbuf(s), &tmX, (w.kb0 + it) * 64, w.j * BNT, &ctrl->xfull[s]);
          else
            tma_load_2d(xbuf(s), &tmT, (it - w.nk) * 64, w.j * BNT, &ctrl->xfull[s]);
          gi = g + 1;
        }
      }
      if (pre_aborted(ctrl)) {
        for (uint32_t x = gi > static_cast<uint32_t>(SX) ? gi - SX : 0; x < gi; ++x)
          mbar_wait(&ctrl->xfull[x % SX], (x / SX) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BNT, 0, 0);
      constexpr uint32_t idesc_mn = idesc_bf16(128, BNT, 1, 0);
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(abuf(0)), 16, 1024);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xbuf(0)), 16, 1024);
      const uint32_t astep = static_cast<uint32_t>(p.atile) >> 4;
      constexpr uint32_t xstep = L::kXbuf >> 4, hstep = kPreTileBytes >> 4;
      const int halves = ROWS / 128;
      bool ok = true;
      RingCursor ac, xc;
      int t = 0;
      for (int u = cta; u < p.units && ok; u += G, ++t) {
        const PreUnit w = pre_unit(p, u);
        // two accumulators used by alternate units, or (wide) by the two halves of every
        // unit: then the epilogue of a unit must drain both before the next one starts
        const int b = WIDE ? 0 : (t & 1);
        const uint32_t ph = WIDE ? (t & 1) : ((t >> 1) & 1);
        const uint32_t acc = tmem + static_cast<uint32_t>(b * BNT);
        if (!mbar_wait(&ctrl->accempty[b], ph ^ 1) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
          break;
        }
        tc_fence_after();
        for (int it = 0; it < w.nk + w.nad; ++it, ac.next(SA), xc.next(SX)) {
          const uint32_t sa = ac.s, sx = xc.s;
          if (!mbar_wait(&ctrl->dec[sa], ac.ph) || !mbar_wait(&ctrl->xfull[sx], xc.ph) ||
              pre_aborted(ctrl)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dx = xdesc0 + sx * xstep;
#pragma unroll 1
          for (int hf = 0; hf < halves; ++hf) {
            const uint32_t acch = acc + static_cast<uint32_t>(hf * BNT);
            if (it < w.nk) {
              const uint64_t da = adesc0 + sa * astep + hf * hstep;
              mma_bf16_ss(acch, da, dx, idesc, it != 0);
              mma_bf16_ss(acch, da + 2, dx + 2, idesc, 1u);
              mma_bf16_ss(acch, da + 4, dx + 4, idesc, 1u);
              mma_bf16_ss(acch, da + 6, dx + 6, idesc, 1u);
            } else {
              // B_cat^T chunk, MN-major: two 64-row halves 8 KB apart, 16 ranks = 2 KB
              const int c = it - w.nk;
              const int kk = min(4, (p.R16 - 64 * c) / 16);
              const uint32_t a0 = smem_u32(abuf(sa) + hf * kPreTileBytes);
              for (int k = 0; k < kk; ++k)
                mma_bf16_ss(acch, smem_desc_sw128(a0 + 2048 * k, 8192, 1024), dx + 2 * k,
                            idesc_mn, 1u);
            }
          }
          mma_commit(&ctrl->aempty[sa]);
          mma_commit(&ctrl->xempty[sx]);
        }
        if (ok) mma_commit(&ctrl->accfull[b]);
      }
      mma_commit(&ctrl->fin);
      // every MMA of this CTA has finished before TMEM can be released
      if (!mbar_wait(&ctrl->fin, 0)) pre_timeout(p.status, ctrl);
    }
  } else if (warp < 6) {
    // ================================================================ epilogue (warps 2-5)
    const int q = warp & 3;  // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;  // weight row within a 128-row half
    const int halves = ROWS / 128;
    __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(p.Y);
    int t = 0;
    for (int u = cta; u < p.units; u += G, ++t) {
      const PreUnit w = pre_unit(p, u);
      const int b = WIDE ? 0 : (t & 1);
      const uint32_t ph = WIDE ? (t & 1) : ((t >> 1) & 1);
      const uint32_t acc = tmem + static_cast<uint32_t>(b * BNT);
      bool ok = mbar_wait(&ctrl->accfull[b], ph) && !pre_aborted(ctrl);
      if (!ok) pre_timeout(p.status, ctrl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int mvalid = min(BNT, p.M - w.j * BNT);
      const size_t row0 = static_cast<size_t>(w.j) * BNT;
      if (w.ns == 1) {
#pragma unroll 1
        for (int hf = 0; hf < halves; ++hf) {
          const size_t n = static_cast<size_t>(w.i) * ROWS + hf * 128 + r;
          const uint32_t acch = acc + static_cast<uint32_t>(hf * BNT);
          for (int c = 0; c < BNT; c += 16) {
            uint32_t v[16];
            tmem_ld16(acch + lane_base + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c + e < mvalid)
                Y[(row0 + c + e) * p.N + n] = __float2bfloat16_rn(__uint_as_float(v[e]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->accempty[b]);
      } else {
        // split K: add into the tile's fp32 sum in L2, count in per warp; the warp that
        // arrives last for these rows writes Y and clears both.  The sum is token-major
        // ([token][ROWS rows]), so that every reduction, load and store of a warp covers
        // one 128-byte line.
        const size_t st = static_cast<size_t>(w.t - p.full);  // index among the split tiles
        float* sum = p.acc + st * ROWS * BNT + r;
#pragma unroll 1
        for (int hf = 0; hf < halves; ++hf) {
          const uint32_t acch = acc + static_cast<uint32_t>(hf * BNT);
          for (int c = 0; c < BNT; c += 16) {
            uint32_t v[16];
            tmem_ld16(acch + lane_base + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c + e < mvalid)
                red_add_f32(sum + hf * 128 + (c + e) * ROWS, __uint_as_float(v[e]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->accempty[b]);
        __threadfence();
        __syncwarp();
        uint32_t last = 0;
        const size_t cidx = st * 4 + q;
        if (lane == 0) last = atomicAdd(p.counters + cidx, 1u) == static_cast<uint32_t>(w.ns - 1);
        if (__shfl_sync(0xffffffffu, last, 0)) {
          __threadfence();
#pragma unroll 1
          for (int hf = 0; hf < halves; ++hf) {
            const size_t n = static_cast<size_t>(w.i) * ROWS + hf * 128 + r;
            float* sh = sum + hf * 128;
            // 32 tokens per L2 round trip: a chunk's loads all go out before its stores
            for (int c0 = 0; c0 < mvalid; c0 += 32) {
              float tv[32];
#pragma unroll
              for (int e = 0; e < 32; ++e)
                tv[e] = c0 + e < mvalid ? __ldcg(sh + (c0 + e) * ROWS) : 0.f;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < mvalid) {
                  Y[(row0 + c0 + e) * p.N + n] = __float2bfloat16_rn(tv[e]);
                  __stcg(sh + (c0 + e) * ROWS, 0.f);
                }
            }
          }
          if (lane == 0) p.counters[cidx] = 0u;
        }
      }
    }
  } else {
    // ================================================================ decoders (warps 7-22)
    // four groups of four warps; group x takes the iterations g = x mod 4, warp wg of the
    // group rebuilds rows 32 wg .. + 31 of a block, one row per thread (or, for an adapter
    // chunk, the group's leader copies B_cat^T)
    static_assert(WPG == 4, "one warp per 32-row quarter");
    const int dw = warp - 7;
    const int grp = dw / WPG, wg = dw % WPG;
    if (p.R16 > 0 && wg == 0 && lane == 0 && !p.dense) prefetch_tmap(&tmB);
    uint32_t g = 0, adn = 0;
    RingCursor cc, ac;  // walked on every iteration, this group's or not
    bool ok = !p.dense;  // dense weights need no decoding
    for (int u = cta; u < p.units && ok; u += G) {
      const PreUnit w = pre_unit(p, u);
      for (int it = 0; it < w.nk + w.nad; ++it, ++g, cc.next(SC), ac.next(SA)) {
        if (static_cast<int>(g & (kPreGroups - 1)) != grp) continue;
        const uint32_t sc = cc.s, sa = ac.s;
        if (!mbar_wait(&ctrl->cfull[sc], cc.ph) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
          ok = false;
          break;
        }
        if (it < w.nk) {
          const uint8_t* cb = cbuf(sc);
          const QuarterRuns qr = quarter_runs(reinterpret_cast<const uint64_t*>(cb), wg, lane);
          if (!mbar_wait(&ctrl->aempty[sa], ac.ph ^ 1)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          expand_runs_to_tile(qr, smem_u32(cb + kBitmapBytes), wg, lane, smem_u32(ntab), abuf(sa),
                              p.status, static_cast<uint32_t>(p.cbuf) - kBitmapBytes);
          fence_proxy_async_smem();
        } else {
          if (!mbar_wait(&ctrl->aempty[sa], ac.ph ^ 1)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          if (wg == 0 && lane == 0) {
            const int c = it - w.nk;
            mbar_arrive_expect_tx(&ctrl->adfull[grp], kPreTileBytes);
            tma_load_2d(abuf(sa), &tmB, w.i * 128, c * 64, &ctrl->adfull[grp]);
            tma_load_2d(abuf(sa) + 8192, &tmB, w.i * 128 + 64, c * 64, &ctrl->adfull[grp]);
          }
          // every warp of the group waits for the copy (a bounded wait also lets the
          // copy land before the CTA can exit)
          if (!mbar_wait(&ctrl->adfull[grp], adn & 1)) {
            pre_timeout(p.status, ctrl);
            ok = false;
            break;
          }
          ++adn;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ctrl->dec[sa]);
          mbar_arrive(&ctrl->cempty[sc]);
        }
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

// ------------------------------------------------------------------------------------
// Dense expansion of the whole encoded weight, [N x K] bf16 row-major with pruned entries
// +0 (the layer's dense-scratch path and salr_decode).  CTAs of four warps walk the
// 128 x 64 blocks blockIdx.x, blockIdx.x + gridDim.x, ...: each block is staged in shared
// memory by cp.async while the previous one is expanded (two buffers); each warp rebuilds
// one 32-row quarter with the layer kernels' device functions into a swizzled shared
// tile, and the tile then goes out row segment by row segment (8 lanes write one
// 128-byte row segment).  About 51 KB of shared memory, so four CTAs share an SM.
constexpr int kExpandMaxBlockBytes = kBitmapBytes + 2 * kBlockRows * kBlockCols;  // dense block
constexpr int kExpandBuf = kExpandMaxBlockBytes + 32;
constexpr int kExpandCtasPerSm = 4;
__global__ void __launch_bounds__(128) expand_dense_kernel(const uint8_t* __restrict__ blob,
                                                           const uint32_t* __restrict__ offsets,
                                                           int K, int nblocks,
                                                           uint16_t* __restrict__ out,
                                                           int* status) {
  extern __shared__ uint4 exp_smem[];
  uint8_t* const cb0 = reinterpret_cast<uint8_t*>(exp_smem);  // two staging buffers
  auto cb = [&](int buf) { return cb0 + buf * kExpandBuf; };
  uint8_t* tile = cb0 + 2 * kExpandBuf;
  uint2* nt = reinterpret_cast<uint2*>((reinterpret_cast<uintptr_t>(tile + kPreTileBytes) + 255) &
                                       ~static_cast<uintptr_t>(255));  // 256-byte aligned
  const int nwords = K / 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 16) nt[threadIdx.x] = nibble_entry(threadIdx.x);
  auto stage = [&](int b, int buf) {
    const uint32_t o0 = offsets[b];
    uint32_t n16 = offsets[b + 1] - o0;
    if (!SALR_CHECK(n16 * 16 + 32 <= static_cast<uint32_t>(kExpandBuf), status)) n16 = 0;
    const uint4* src = reinterpret_cast<const uint4*>(blob) + o0;
    for (uint32_t k = threadIdx.x; k < n16; k += 128)
      cp_async16(reinterpret_cast<uint4*>(cb(buf)) + k, src + k);
  };
  int buf = 0;
  if (static_cast<int>(blockIdx.x) < nblocks) stage(blockIdx.x, 0);
  cp_async_commit();
  for (int b = blockIdx.x; b < nblocks; b += gridDim.x, buf ^= 1) {
    const int bn = b + gridDim.x;
    if (bn < nblocks) stage(bn, buf ^ 1);
    cp_async_commit();
    cp_async_wait_one();  // this block's copies (the older group) have landed
    uint32_t n16 = offsets[b + 1] - offsets[b];
    if (n16 * 16 + 32 > static_cast<uint32_t>(kExpandBuf)) n16 = 0;  // flagged when staged
    if (threadIdx.x < 2) reinterpret_cast<uint4*>(cb(buf))[n16 + threadIdx.x] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const QuarterRuns qr = quarter_runs(reinterpret_cast<const uint64_t*>(cb(buf)), warp, lane);
    // readable: the block and the two zeroed 16-byte chunks after it
    const uint32_t readable = n16 * 16 + 32;
    expand_runs_to_tile(qr, smem_u32(cb(buf) + kBitmapBytes), warp, lane, smem_u32(nt), tile, status,
                        readable > kBitmapBytes ? readable - kBitmapBytes : 0u);
    __syncthreads();  // the tile is complete; this compact buffer is free for block b + 2 grid
    const int i = b / nwords, j = b % nwords;
    uint16_t* dst = out + static_cast<size_t>(i) * kBlockRows * K + j * kBlockCols;
    const int c = threadIdx.x & 7;
#pragma unroll 4
    for (int r = threadIdx.x >> 3; r < kBlockRows; r += 16)
      *reinterpret_cast<uint4*>(dst + static_cast<size_t>(r) * K + c * 8) =
          *reinterpret_cast<const uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
    __syncthreads();  // the tile is free for the next block
  }
}
constexpr int kExpandSmemBytes = 2 * kExpandBuf + kPreTileBytes + 256 + 128;  // table aligned up

// ------------------------------------------------------------------------------------
// t = X A_cat for all tokens, rounded once to bf16 into T [M x 128] (ranks past R16 are
// not written).  D[128 ranks x BNT tokens] = A_cat^T (MN-major) x X^T, as the small-M
// kernel's t shares.
constexpr int kTThreads = 192;
constexpr int kTStages = 4;

struct TParams {
  uint16_t* T;         // [M x 128] bf16
  float* T32;          // [tokens x 128 ranks] fp32 sums of K splits (token-major), zero between calls
  uint32_t* counters;  // [TT x 4] split arrivals per token tile and 32-rank quarter
  int* status;
  int M, R16, kblocks, TT, splits;
};

struct TCtrl {
  uint64_t full[kTStages], empty[kTStages], fin;
  uint32_t tmem;
  int abort;
};

template <int BNT>
struct TLayout {
  static constexpr int kStage = 16384 + BNT * 128;  // A_cat block [64 k x 128 ranks] + X tile
  static constexpr int kSmemBytes = kTStages * kStage + 1024 + 1024;
};

template <int BNT>
__global__ void __launch_bounds__(kTThreads, 1)
    salr_t_kernel(const __grid_constant__ TParams p, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmA) {
  using L = TLayout<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  TCtrl* ctrl = reinterpret_cast<TCtrl*>(smem + kTStages * L::kStage);
  // the layer kernel that follows may start now: it waits for this grid before reading t
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x % p.TT, sidx = blockIdx.x / p.TT;
  const int kb0 = static_cast<int>(static_cast<long long>(sidx) * p.kblocks / p.splits);
  const int kb1 = static_cast<int>(static_cast<long long>(sidx + 1) * p.kblocks / p.splits);
  const int nk = kb1 - kb0;
  constexpr uint32_t kCols = BNT < 32 ? 32 : BNT;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->fin, 1);
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&ctrl->tmem, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;
  volatile int* abort_flag = &ctrl->abort;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmA);
      const uint32_t abytes = (p.R16 > 64 ? 2u : 1u) * 8192u;
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % kTStages;
        if (!mbar_wait(&ctrl->empty[s], ((it / kTStages) & 1) ^ 1) || *abort_flag) {
          atomicOr(p.status, DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uint8_t* st = smem + s * L::kStage;
        const int kb = kb0 + it;
        mbar_arrive_expect_tx(&ctrl->full[s], abytes + BNT * 128);
        tma_load_2d(st, &tmA, 0, kb * 64, &ctrl->full[s]);
        if (p.R16 > 64) tma_load_2d(st + 8192, &tmA, 64, kb * 64, &ctrl->full[s]);
        tma_load_2d(st + 16384, &tmX, kb * 64, j * BNT, &ctrl->full[s]);
        issued = it + 1;
      }
      if (*abort_flag) {
        for (int it = issued - kTStages < 0 ? 0 : issued - kTStages; it < issued; ++it)
          mbar_wait(&ctrl->full[it % kTStages], (it / kTStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_mn = idesc_bf16(128, BNT, 1, 0);
      bool ok = true;
      for (int it = 0; it < nk && ok; ++it) {
        const int s = it % kTStages;
        if (!mbar_wait(&ctrl->full[s], (it / kTStages) & 1) || *abort_flag) {
          atomicOr(p.status, DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * L::kStage), x0 = a0 + 16384;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem, smem_desc_sw128(a0 + 2048 * k, 8192, 1024),
                      smem_desc_sw128(x0 + 32 * k, 16, 1024), idesc_mn, (it | k) != 0);
        mma_commit(&ctrl->empty[s]);
      }
      mma_commit(&ctrl->fin);
      if (!mbar_wait(&ctrl->fin, 0)) atomicOr(p.status, DEV_ERR_TIMEOUT);
    }
  } else {
    // epilogue warps 2-5: lane quarter q holds ranks 32q..32q+31
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;
    bool ok = mbar_wait(&ctrl->fin, 0) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int mvalid = min(BNT, p.M - j * BNT);
      const size_t row0 = static_cast<size_t>(j) * BNT;
      __nv_bfloat16* T = reinterpret_cast<__nv_bfloat16*>(p.T);
      if (p.splits == 1) {
        for (int c = 0; c < BNT; c += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + c, v);
          tmem_ld_wait();
          if (r < p.R16) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c + e < mvalid) T[(row0 + c + e) * 128 + r] = __float2bfloat16_rn(__uint_as_float(v[e]));
          }
        }
      } else {
        // token-major sums ([token][128 ranks]): a warp's 32 ranks of one token are one
        // 128-byte line for every reduction, load and store
        float* sum = p.T32 + row0 * 128 + r;
        for (int c = 0; c < BNT; c += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + c, v);
          tmem_ld_wait();
          if (r < p.R16) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c + e < mvalid) red_add_f32(sum + (c + e) * 128, __uint_as_float(v[e]));
          }
        }
        __threadfence();
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0) last = atomicAdd(p.counters + j * 4 + q, 1u) == static_cast<uint32_t>(p.splits - 1);
        if (__shfl_sync(0xffffffffu, last, 0)) {
          __threadfence();
          if (r < p.R16) {
            // 32 tokens per L2 round trip: a chunk's loads all go out before its stores
            for (int c0 = 0; c0 < mvalid; c0 += 32) {
              float tv[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) tv[e] = c0 + e < mvalid ? __ldcg(sum + (c0 + e) * 128) : 0.f;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < mvalid) {
                  T[(row0 + c0 + e) * 128 + r] = __float2bfloat16_rn(tv[e]);
                  __stcg(sum + (c0 + e) * 128, 0.f);
                }
            }
          }
          if (lane == 0) p.counters[j * 4 + q] = 0u;
        }
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
