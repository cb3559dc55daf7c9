// salr_prefill.cuh - the SALR layer for token counts above 64 (prefill shapes), where the
// tensor-core contraction dominates.  Two kernels per call:
//
// * salr_t_kernel: t = X A_cat, the concatenated adapter's down projection (SALR
//   technical summary, Methodology 3), computed once per call on the tensor cores and
//   rounded once to bf16 into a [M x 128] scratch.  Grid: token tiles x K splits.  With
//   several splits, each adds its fp32 part into a sum in L2 (vector reductions), and the
//   last split of a token tile to count itself in converts the sum and clears it.
// * salr_prefill_kernel: one CTA per (128-row weight tile, token tile, K split).  Each
//   128 x 64 bitmap block arrives by one bulk copy and the matching X tile by tensor TMA.
//   Decoder warps expand the block into the 128-byte-swizzled tile (stage 1, Methodology
//   4) with the same device functions as the small-M kernel; tcgen05 MMAs multiply it
//   (stage 2).  After the K blocks,
//   the CTA of split 0 adds B_cat^T t^T with R/16 more MMAs.  The epilogue writes Y; with
//   several K splits, each adds into an fp32 sum in L2 whose last contributor writes Y.
//
// Orientation as in the small-M kernel: D[128 weight rows x BNT tokens] in TMEM.
// Rings: compact blocks (producer -> decoders), decoded tiles (decoders -> MMA) and X
// tiles (X loader -> MMA), so that the copy latency and the decode of a block overlap the
// MMAs of earlier blocks; four decoder groups each work on a different block.
// Warp roles (736 threads): 0 compact-block producer, 1 TMEM allocator + MMA issuer, 2-5
// epilogue, 6 X-tile producer, 7-22 decoders.  Every wait is bounded; a timeout is
// recorded in the status word.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "salr_codec.cuh"
#include "salr_stream.cuh"
#include "sm100.cuh"

namespace salr {

constexpr int kPreDecoders = 16;
constexpr int kPreGroups = 4;                             // decoder groups (blocks in flight)
constexpr int kPreThreads = 32 * (7 + kPreDecoders);      // + producer, MMA, 4 epilogue, X loader
constexpr int kPreMaxC = 8, kPreMaxA = 6, kPreMaxX = 4;    // ring depths
constexpr int kPreMaxKBlocks = 512;  // K <= 32768
constexpr int kPreCtrlBytes = 3072;
constexpr int kPreTileBytes = 16384;

struct PrefillParams {
  const uint8_t* blob;
  const uint32_t* offsets;
  uint16_t* Y;
  float* acc;          // [N x Mp] fp32 sums of split-K tiles (token-contiguous), zero between calls
  uint32_t* counters;  // [RT x TT x 4] split arrivals per tile and 32-row quarter, zero between calls
  int* status;
  int N, K, M, R16;
  int Mp;              // M rounded up to 4: row stride of the fp32 sums
  int kblocks;         // K / 64
  int TT;              // token tiles
  int splits;          // K splits per output tile
  int cbuf;            // bytes of a compact-block slot, multiple of 1024
  int sc, sa, sx;      // ring depths: compact blocks, decoded tiles, X tiles
};

struct PrefillCtrl {
  uint64_t cfull[kPreMaxC], cempty[kPreMaxC];
  uint64_t dec[kPreMaxA], aempty[kPreMaxA];
  uint64_t xfull[kPreMaxX], xempty[kPreMaxX];
  uint64_t tfull, bcfull, fin;
  uint32_t tmem;
  int abort;
  int flag;
  uint32_t off[kPreMaxKBlocks + 1];
};
static_assert(sizeof(PrefillCtrl) <= kPreCtrlBytes, "control block");

// Shared-memory layout: [decoded tiles: sa x 16 KB][X tiles: sx x BNT*128][compact blocks:
// sc x cbuf][chunk tables: 4 x 4 KB][nibble table][control].  After the K loop the
// adapter's operands reuse the front: the B_cat^T tile [128 x R16] at offset 0 (<= 32 KB)
// and the t tile [BNT x 128] (two 64-rank chunks) at 32 KB.
template <int BNT>
struct PrefillLayout {
  static constexpr int kXbuf = BNT * 128;
  __host__ __device__ static int x_off(int sa) { return sa * kPreTileBytes; }
  __host__ __device__ static int c_off(int sa, int sx) { return x_off(sa) + sx * kXbuf; }
  __host__ __device__ static int table_off(int sa, int sx, int sc, int cbuf) {
    return c_off(sa, sx) + sc * cbuf;
  }
  __host__ __device__ static int smem_bytes(int sa, int sx, int sc, int cbuf) {
    return table_off(sa, sx, sc, cbuf) + kPreGroups * 4096 + 128 /*nibbles*/ + kPreCtrlBytes +
           1024 /*align*/;
  }
  static constexpr int kAdapterBytes = 32768 + 2 * kXbuf;  // B_cat^T tile + t tile
};

__device__ __forceinline__ void pre_timeout(int* status, PrefillCtrl* c) {
  atomicOr(status, DEV_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c->abort) = 1;
}
__device__ __forceinline__ bool pre_aborted(PrefillCtrl* c) {
  return *reinterpret_cast<volatile int*>(&c->abort) != 0;
}

template <int BNT>
__global__ void __launch_bounds__(kPreThreads, 1)
    salr_prefill_kernel(const __grid_constant__ PrefillParams p,
                        const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmT) {
  using L = PrefillLayout<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SC = p.sc, SA = p.sa, SX = p.sx;
  auto abuf = [&](int s) { return smem + s * kPreTileBytes; };
  auto xbuf = [&](int s) { return smem + L::x_off(SA) + s * L::kXbuf; };
  auto cbuf = [&](int s) { return smem + L::c_off(SA, SX) + s * p.cbuf; };
  uint8_t* tables = smem + L::table_off(SA, SX, SC, p.cbuf);
  uint2* ntab = reinterpret_cast<uint2*>(tables + kPreGroups * 4096);
  PrefillCtrl* ctrl = reinterpret_cast<PrefillCtrl*>(tables + kPreGroups * 4096 + 128);
  uint8_t* bcbuf = smem;           // after the K loop only
  uint8_t* tbuf = smem + 32768;    // after the K loop only

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool adapter = p.R16 > 0;
  // work unit: token tile j (fastest), K split s, weight row tile i
  const int cta = blockIdx.x;
  const int j = cta % p.TT;
  const int rest = cta / p.TT;
  const int sidx = rest % p.splits;
  const int i = rest / p.splits;
  const int kb0 = static_cast<int>(static_cast<long long>(sidx) * p.kblocks / p.splits);
  const int kb1 = static_cast<int>(static_cast<long long>(sidx + 1) * p.kblocks / p.splits);
  const int nk = kb1 - kb0;
  const bool add_adapter = adapter && sidx == 0;
  constexpr int WPG = kPreDecoders / kPreGroups;
  constexpr uint32_t kCols = BNT < 32 ? 32 : BNT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      mbar_init(&ctrl->cfull[s], 1);
      mbar_init(&ctrl->cempty[s], WPG);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&ctrl->dec[s], WPG);
      mbar_init(&ctrl->aempty[s], 1);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(&ctrl->xfull[s], 1);
      mbar_init(&ctrl->xempty[s], 1);
    }
    mbar_init(&ctrl->tfull, 1);
    mbar_init(&ctrl->bcfull, 1);
    mbar_init(&ctrl->fin, 1);
    ctrl->abort = 0;
    ctrl->flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) ntab[threadIdx.x] = nibble_entry(threadIdx.x);
  if (warp == 0) {
    const uint32_t* src = p.offsets + static_cast<size_t>(i) * p.kblocks + kb0;
    for (int t = lane; t <= nk; t += 32) ctrl->off[t] = src[t];
  }
  if (warp == 1) tmem_alloc(&ctrl->tmem, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;

  if (warp == 0) {
    // ================================================================ compact-block producer
    if (lane == 0) {
      int issued = 0;
      bool bc_issued = false;
      for (int it = 0; it < nk; ++it) {
        const int s = it % SC;
        if (!mbar_wait(&ctrl->cempty[s], ((it / SC) & 1) ^ 1) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
          break;
        }
        const uint32_t o0 = ctrl->off[it], o1 = ctrl->off[it + 1];
        mbar_arrive_expect_tx(&ctrl->cfull[s], (o1 - o0) * 16u);
        bulk_g2s(cbuf(s), p.blob + static_cast<size_t>(o0) * 16, (o1 - o0) * 16u, &ctrl->cfull[s]);
        issued = it + 1;
      }
      if (add_adapter && !pre_aborted(ctrl)) {
        // the adapter operands go where the rings were: wait until every MMA read them
        if (!mbar_wait(&ctrl->tfull, 0)) {
          pre_timeout(p.status, ctrl);
        } else {
          prefetch_tmap(&tmB);
          prefetch_tmap(&tmT);
          const int nch = (p.R16 + 63) / 64;
          mbar_arrive_expect_tx(&ctrl->bcfull, 256u * p.R16 + nch * L::kXbuf);
          tma_load_2d(bcbuf, &tmB, i * 128, 0, &ctrl->bcfull);
          tma_load_2d(bcbuf + p.R16 * 128, &tmB, i * 128 + 64, 0, &ctrl->bcfull);
          for (int c = 0; c < nch; ++c) tma_load_2d(tbuf + c * L::kXbuf, &tmT, c * 64, j * BNT, &ctrl->bcfull);
          bc_issued = true;
        }
      }
      if (pre_aborted(ctrl)) {
        // let every copy this thread started land before the CTA can exit
        for (int it = issued - SC < 0 ? 0 : issued - SC; it < issued; ++it)
          mbar_wait(&ctrl->cfull[it % SC], (it / SC) & 1);
        if (bc_issued) mbar_wait(&ctrl->bcfull, 0);
      }
    }
  } else if (warp == 6) {
    // ================================================================ X-tile producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % SX;
        if (!mbar_wait(&ctrl->xempty[s], ((it / SX) & 1) ^ 1) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
          break;
        }
        mbar_arrive_expect_tx(&ctrl->xfull[s], L::kXbuf);
        tma_load_2d(xbuf(s), &tmX, (kb0 + it) * 64, j * BNT, &ctrl->xfull[s]);
        issued = it + 1;
      }
      if (pre_aborted(ctrl)) {
        for (int it = issued - SX < 0 ? 0 : issued - SX; it < issued; ++it)
          mbar_wait(&ctrl->xfull[it % SX], (it / SX) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BNT, 0, 0);
      constexpr uint32_t idesc_mn = idesc_bf16(128, BNT, 1, 0);
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(abuf(0)), 16, 1024);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xbuf(0)), 16, 1024);
      constexpr uint32_t astep = kPreTileBytes >> 4, xstep = L::kXbuf >> 4;
      bool ok = true;
      int sa = 0, sx = 0;
      uint32_t pa = 0, px = 0;
      for (int it = 0; it < nk; ++it) {
        if (!mbar_wait(&ctrl->dec[sa], pa) || !mbar_wait(&ctrl->xfull[sx], px) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = adesc0 + sa * astep, dx = xdesc0 + sx * xstep;
        mma_bf16_ss(tmem, da, dx, idesc, it != 0);
        mma_bf16_ss(tmem, da + 2, dx + 2, idesc, 1u);
        mma_bf16_ss(tmem, da + 4, dx + 4, idesc, 1u);
        mma_bf16_ss(tmem, da + 6, dx + 6, idesc, 1u);
        mma_commit(&ctrl->aempty[sa]);
        mma_commit(&ctrl->xempty[sx]);
        if (++sa == SA) {
          sa = 0;
          pa ^= 1u;
        }
        if (++sx == SX) {
          sx = 0;
          px ^= 1u;
        }
      }
      mma_commit(&ctrl->tfull);
      if (ok && add_adapter) {
        if (!mbar_wait(&ctrl->bcfull, 0) || pre_aborted(ctrl)) {
          pre_timeout(p.status, ctrl);
        } else {
          tc_fence_after();
          const uint32_t b0 = smem_u32(bcbuf), t0 = smem_u32(tbuf);
          for (int k = 0; k < p.R16 / 16; ++k)
            mma_bf16_ss(tmem, smem_desc_sw128(b0 + 2048 * k, p.R16 * 128, 1024),
                        smem_desc_sw128(t0 + (k >> 2) * (BNT * 128) + (k & 3) * 32, 16, 1024),
                        idesc_mn, 1u);
        }
      }
      mma_commit(&ctrl->fin);
      // every MMA of this CTA has finished before TMEM can be released
      if (!mbar_wait(&ctrl->fin, 0)) pre_timeout(p.status, ctrl);
    }
  } else if (warp < 6) {
    // ================================================================ epilogue (warps 2-5)
    // Decisions guarding warp-collective instructions or the group barrier are made
    // uniform first (a vote, then one shared flag).
    const int q = warp & 3;  // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;  // weight row within the tile
    bool ok = mbar_wait(&ctrl->fin, 0);
    if (!ok) pre_timeout(p.status, ctrl);
    ok = __all_sync(0xffffffffu, ok);
    named_bar(1, 128);
    if (threadIdx.x == 64) ctrl->flag = (ok && !pre_aborted(ctrl)) ? 2 : 0;
    named_bar(1, 128);
    const bool go = *reinterpret_cast<volatile int*>(&ctrl->flag) == 2;
    tc_fence_after();
    const int mvalid = min(BNT, p.M - j * BNT);
    const size_t n = static_cast<size_t>(i) * 128 + r;
    const size_t row0 = static_cast<size_t>(j) * BNT;
    __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(p.Y);
    if (go && p.splits == 1) {
      for (int c = 0; c < BNT; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (c + e < mvalid)
            Y[(row0 + c + e) * p.N + n] = __float2bfloat16_rn(__uint_as_float(v[e]));
      }
    } else if (go) {
      // split K: add into the tile's fp32 sum in L2 (row n, token-contiguous), count in
      // per warp; the warp that arrives last for these 32 rows writes Y and clears both
      float* sum = p.acc + n * p.Mp + row0;
      for (int c = 0; c < BNT; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          if (c + e < mvalid)
            red_add_v4f32(sum + c + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                          __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
      }
      __threadfence();
      __syncwarp();
      uint32_t last = 0;
      const size_t cidx = (static_cast<size_t>(i) * p.TT + j) * 4 + q;
      if (lane == 0) last = atomicAdd(p.counters + cidx, 1u) == static_cast<uint32_t>(p.splits - 1);
      if (__shfl_sync(0xffffffffu, last, 0)) {
        __threadfence();
        // 32 tokens per L2 round trip: a chunk's loads all go out before its stores
        for (int c0 = 0; c0 < mvalid; c0 += 32) {
          float4 t4[8];
#pragma unroll
          for (int g = 0; g < 8; ++g)
            t4[g] = c0 + 4 * g < mvalid ? __ldcg(reinterpret_cast<const float4*>(sum + c0 + 4 * g))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int c = c0 + 4 * g;
            if (c >= mvalid) continue;
            const float tv[4] = {t4[g].x, t4[g].y, t4[g].z, t4[g].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (c + e < mvalid) Y[(row0 + c + e) * p.N + n] = __float2bfloat16_rn(tv[e]);
            __stcg(reinterpret_cast<float4*>(sum + c), make_float4(0.f, 0.f, 0.f, 0.f));
          }
        }
        if (lane == 0) p.counters[cidx] = 0u;
      }
    }
  } else {
    // ================================================================ decoders (warps 7-22)
    // four groups of four warps, group g on blocks g, g + 4, ..., each warp on 32 rows
    constexpr int RPW = 128 / WPG;
    const int dw = warp - 7;
    const int g = dw / WPG, wg = dw % WPG;
    uint32_t* cs = reinterpret_cast<uint32_t*>(tables + g * 4096);
    for (int it = g; it < nk; it += kPreGroups) {
      const int sc = it % SC, sa = it % SA;
      if (!mbar_wait(&ctrl->cfull[sc], (it / SC) & 1) || pre_aborted(ctrl)) {
        pre_timeout(p.status, ctrl);
        break;
      }
      const uint8_t* cb = cbuf(sc);
      build_chunk_table<RPW>(reinterpret_cast<const uint64_t*>(cb), cs, wg, lane);
      __syncwarp();
      if (!mbar_wait(&ctrl->aempty[sa], ((it / SA) & 1) ^ 1)) {
        pre_timeout(p.status, ctrl);
        break;
      }
      expand_rows<RPW>(cb + kBitmapBytes, cs, abuf(sa), wg, lane, ntab);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctrl->dec[sa]);
        mbar_arrive(&ctrl->cempty[sc]);
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
// t = X A_cat for all tokens, rounded once to bf16 into T [M x 128] (ranks past R16 are
// not written).  D[128 ranks x BNT tokens] = A_cat^T (MN-major) x X^T, as the small-M
// kernel's t shares.
constexpr int kTThreads = 192;
constexpr int kTStages = 4;

struct TParams {
  uint16_t* T;         // [M x 128] bf16
  float* T32;          // [128 x Mp] fp32 sums of K splits (token-contiguous), zero between calls
  uint32_t* counters;  // [TT x 4] split arrivals per token tile and 32-rank quarter
  int* status;
  int M, Mp, R16, kblocks, TT, splits;
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
        float* sum = p.T32 + static_cast<size_t>(r) * p.Mp + row0;
        for (int c = 0; c < BNT; c += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + c, v);
          tmem_ld_wait();
          if (r < p.R16) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              if (c + e < mvalid)
                red_add_v4f32(sum + c + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                              __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
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
              float4 t4[8];
#pragma unroll
              for (int g = 0; g < 8; ++g)
                t4[g] = c0 + 4 * g < mvalid
                            ? __ldcg(reinterpret_cast<const float4*>(sum + c0 + 4 * g))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int g = 0; g < 8; ++g) {
                const int c = c0 + 4 * g;
                if (c >= mvalid) continue;
                const float tv[4] = {t4[g].x, t4[g].y, t4[g].z, t4[g].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (c + e < mvalid) T[(row0 + c + e) * 128 + r] = __float2bfloat16_rn(tv[e]);
                __stcg(reinterpret_cast<float4*>(sum + c), make_float4(0.f, 0.f, 0.f, 0.f));
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
