// salr_linear.cuh - the fused SALR layer Y = X (M (.) W)^T + (X A_cat) B_cat on sm_100a.
//
// Two-stage pipeline (SALR technical summary, Methodology 4): bitmap blocks and their
// compact values are streamed into shared memory by TMA, expanded on CUDA cores into a
// dense 128 x 64 bf16 tile (stage 1) and consumed by tcgen05 tensor-core MMAs that
// accumulate in tensor memory (stage 2), with the expansion of block k+1 overlapping
// the MMAs of block k.  The concatenated adapter (Methodology 3) runs in the same
// kernel: t^T = A_cat^T X^T accumulates beside the main product over the same K blocks,
// is rounded to bf16 into shared memory, and one more MMA adds B_cat^T t^T into the
// accumulator before the epilogue.
//
// Orientation: the MMA computes Y^T tiles, D[128 weight rows x BNT tokens] =
// Wtile[128 x K] * Xtile[BNT x K]^T, so the decoded weight tile is the 128-row operand
// and the token count (1 .. 256 per tile) is the MMA's N.  Small token counts split K
// across CTAs; partial sums meet in an fp32 workspace and the last CTA of a tile (an
// arrival counter, no waiting) writes Y.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer,
// warps 2-5 decoders and, after the K loop, the epilogue.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "salr_codec.cuh"
#include "sm100.cuh"

namespace salr {

constexpr int kLinThreads = 192;
constexpr int kCbufBytes = kBitmapBytes + kBlockRows * kBlockCols * 2;  // worst case: all kept
constexpr int kAbufBytes = kBlockRows * kBlockCols * 2;                 // 16 KB dense tile
constexpr int kAcatBytes = 2 * 64 * 128;                                // 64 K rows x 128 ranks
constexpr int kMaxKBlocks = 512;                                        // K <= 32768
constexpr int kCtrlBytes = 4096;
constexpr int kSmemLimit = 232448;  // B200 opt-in dynamic shared memory per CTA

template <int BNT>
struct LinLayout {
  static constexpr int kXbuf = BNT * 128;
  static constexpr int kStage = kCbufBytes + kAbufBytes + kXbuf + kAcatBytes;
  static constexpr int kStagesRaw = (kSmemLimit - 1024 - kCtrlBytes) / kStage;
  static constexpr int kStages = kStagesRaw > 6 ? 6 : kStagesRaw;
  static constexpr int kTbuf = BNT * 256;          // t as [BNT x 128] bf16, two 64-wide chunks
  static constexpr int kBcatMax = 2 * 128 * 128;   // B_cat^T tile, [128 x R<=128]
  static constexpr int kCtrlOff = kStages * kStage;
  static constexpr int kSmemBytes = kCtrlOff + kCtrlBytes + 1024;
  static_assert(kStages >= 2, "pipeline needs two stages");
  static_assert(kTbuf + kBcatMax <= kStages * kStage, "post-loop buffers alias the stages");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

struct LinParams {
  const uint8_t* blob;
  const uint32_t* offsets;
  uint16_t* Y;
  float* ws;            // split-K fp32 partial sums, [TT*BNT x N], zero between calls
  uint32_t* counters;   // split-K arrival counters, [RT x TT], zero between calls
  int* status;
  int N, K, M, R, R16;
  int kblocks;          // K / 64
  int TT;               // token tiles
  int splits;           // K splits per output tile
};

struct Ctrl {
  uint64_t full[8], dec[8], empty[8];
  uint64_t tfull, tready, bcfull, fin;
  uint32_t tmem;
  int abort;
  int last;
  uint32_t off[kMaxKBlocks + 1];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block");

__device__ __forceinline__ void record_timeout(const LinParams& p, Ctrl* c) {
  atomicOr(p.status, DEV_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&c->abort) = 1;
}

__device__ __forceinline__ bool aborted(Ctrl* c) {
  return *reinterpret_cast<volatile int*>(&c->abort) != 0;
}

template <int BNT>
__global__ void __launch_bounds__(kLinThreads, 1)
    salr_linear_kernel(const __grid_constant__ LinParams p, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB) {
  using L = LinLayout<BNT>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + L::kCtrlOff);
  auto cbuf = [&](int s) { return smem + s * L::kStage; };
  auto abuf = [&](int s) { return smem + s * L::kStage + kCbufBytes; };
  auto xbuf = [&](int s) { return smem + s * L::kStage + kCbufBytes + kAbufBytes; };
  auto acbuf = [&](int s) { return smem + s * L::kStage + kCbufBytes + kAbufBytes + L::kXbuf; };
  uint8_t* tbuf = smem;               // after the K loop only
  uint8_t* bcbuf = smem + L::kTbuf;   // after the K loop only

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool adapter = p.R > 0;

  // work unit: token tile j (fastest), K split s, weight row tile i
  const int cta = blockIdx.x;
  const int j = cta % p.TT;
  const int rest = cta / p.TT;
  const int s_idx = rest % p.splits;
  const int i = rest / p.splits;
  const int kb0 = static_cast<int>(static_cast<long long>(s_idx) * p.kblocks / p.splits);
  const int kb1 = static_cast<int>(static_cast<long long>(s_idx + 1) * p.kblocks / p.splits);
  const int nk = kb1 - kb0;
  const uint32_t ncols = adapter ? (2 * BNT < 32 ? 32 : 2 * BNT) : (BNT < 32 ? 32 : BNT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->dec[s], 4);
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->tfull, 1);
    mbar_init(&ctrl->tready, 4);
    mbar_init(&ctrl->bcfull, 1);
    mbar_init(&ctrl->fin, 1);
    ctrl->abort = 0;
    ctrl->last = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    const uint32_t* src = p.offsets + static_cast<size_t>(i) * p.kblocks + kb0;
    for (int t = lane; t <= nk; t += 32) ctrl->off[t] = src[t];
  }
  if (warp == 1) tmem_alloc(&ctrl->tmem, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;
  const uint32_t tmem_main = tmem;
  const uint32_t tmem_t = tmem + BNT;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      if (adapter) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
      }
      const uint32_t xbytes = BNT * 128;
      const uint32_t acbytes = adapter ? (p.R > 64 ? 2u : 1u) * 8192u : 0u;
      int issued = 0;
      bool bc_issued = false;
      for (int it = 0; it < nk; ++it) {
        const int s = it % S;
        const uint32_t round = static_cast<uint32_t>(it / S);
        if (!mbar_wait(&ctrl->empty[s], (round & 1u) ^ 1u)) {
          record_timeout(p, ctrl);
          break;
        }
        if (aborted(ctrl)) break;
        const int kb = kb0 + it;
        const uint32_t o0 = ctrl->off[it], o1 = ctrl->off[it + 1];
        const uint32_t cbytes = (o1 - o0) * 16u;
        mbar_arrive_expect_tx(&ctrl->full[s], cbytes + xbytes + acbytes);
        bulk_g2s(cbuf(s), p.blob + static_cast<size_t>(o0) * 16, cbytes, &ctrl->full[s]);
        tma_load_2d(xbuf(s), &tmX, kb * 64, j * BNT, &ctrl->full[s]);
        if (adapter) {
          tma_load_2d(acbuf(s), &tmA, 0, kb * 64, &ctrl->full[s]);
          if (p.R > 64) tma_load_2d(acbuf(s) + 8192, &tmA, 64, kb * 64, &ctrl->full[s]);
        }
        issued = it + 1;
      }
      if (adapter && !aborted(ctrl)) {
        // B_cat^T tile goes where the stages were: wait until every MMA has read them
        if (!mbar_wait(&ctrl->tfull, 0)) {
          record_timeout(p, ctrl);
        } else {
          mbar_arrive_expect_tx(&ctrl->bcfull, 256u * p.R16);
          tma_load_2d(bcbuf, &tmB, i * 128, 0, &ctrl->bcfull);
          tma_load_2d(bcbuf + p.R16 * 128, &tmB, i * 128 + 64, 0, &ctrl->bcfull);
          bc_issued = true;
        }
      }
      if (aborted(ctrl)) {
        // let every copy this thread started land before the CTA can exit
        for (int it = issued - S < 0 ? 0 : issued - S; it < issued; ++it)
          mbar_wait(&ctrl->full[it % S], static_cast<uint32_t>(it / S) & 1u);
        if (bc_issued) mbar_wait(&ctrl->bcfull, 0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = idesc_bf16(128, BNT, 0, 0);
      constexpr uint32_t idesc_mnA = idesc_bf16(128, BNT, 1, 0);
      bool ok = true;
      for (int it = 0; it < nk; ++it) {
        const int s = it % S;
        const uint32_t round = static_cast<uint32_t>(it / S);
        if (!mbar_wait(&ctrl->dec[s], round & 1u)) {
          record_timeout(p, ctrl);
          ok = false;
          break;
        }
        if (aborted(ctrl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(abuf(s)), x0 = smem_u32(xbuf(s)), c0 = smem_u32(acbuf(s));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bd = smem_desc_sw128(x0 + 32 * k, 16, 1024);
          const uint32_t acc = (it | k) != 0;
          mma_bf16_ss(tmem_main, smem_desc_sw128(a0 + 32 * k, 16, 1024), bd, idesc_main, acc);
          if (adapter)
            mma_bf16_ss(tmem_t, smem_desc_sw128(c0 + 2048 * k, 8192, 1024), bd, idesc_mnA, acc);
        }
        mma_commit(&ctrl->empty[s]);
      }
      mma_commit(&ctrl->tfull);
      if (ok && adapter) {
        if (!mbar_wait(&ctrl->tready, 0) || !mbar_wait(&ctrl->bcfull, 0)) {
          record_timeout(p, ctrl);
        } else if (!aborted(ctrl)) {
          tc_fence_after();
          const uint32_t b0 = smem_u32(bcbuf), t0 = smem_u32(tbuf);
          for (int k = 0; k < p.R16 / 16; ++k) {
            const uint64_t ad = smem_desc_sw128(b0 + 2048 * k, p.R16 * 128, 1024);
            const uint64_t bd = smem_desc_sw128(t0 + (k >> 2) * (BNT * 128) + (k & 3) * 32, 16, 1024);
            mma_bf16_ss(tmem_main, ad, bd, idesc_mnA, 1);
          }
        }
      }
      mma_commit(&ctrl->fin);
      // every MMA of this CTA has finished before TMEM can be released
      if (!mbar_wait(&ctrl->fin, 0)) record_timeout(p, ctrl);
    }
  } else {
    // ------------------------------------------------------------ decoders (warps 2-5)
    const int dw = warp - 2;           // rows 32 dw .. 32 dw + 31 of each block
    for (int it = 0; it < nk; ++it) {
      const int s = it % S;
      const uint32_t round = static_cast<uint32_t>(it / S);
      if (!mbar_wait(&ctrl->full[s], round & 1u)) {
        record_timeout(p, ctrl);
        break;
      }
      if (aborted(ctrl)) break;
      const uint8_t* cb = cbuf(s);
      const uint64_t* bm = reinterpret_cast<const uint64_t*>(cb);
      const uint16_t* vals = reinterpret_cast<const uint16_t*>(cb + kBitmapBytes);
      const uint64_t w = bm[32 * dw + lane];
      const uint32_t cnt = __popcll(w);
      const uint32_t inc = warp_incl_scan(cnt);
      uint32_t base = 0;
      for (int r = lane; r < 32 * dw; r += 32) base += __popcll(bm[r]);
      base = warp_sum(base);
      const uint32_t rstart = base + inc - cnt;
      uint8_t* ab = abuf(s);
#pragma unroll 2
      for (int q = 0; q < 8; ++q) {
        const int src = 4 * q + (lane >> 3);
        const int c = lane & 7;
        const uint64_t wr = __shfl_sync(0xffffffffu, w, src);
        const uint32_t rs = __shfl_sync(0xffffffffu, rstart, src);
        const uint32_t b = static_cast<uint32_t>(wr >> (8 * c)) & 0xFFu;
        uint32_t pos = rs + __popcll(wr & ((1ull << (8 * c)) - 1ull));
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t lo = 0, hi = 0;
          if ((b >> (2 * e)) & 1u) lo = vals[pos++];
          if ((b >> (2 * e + 1)) & 1u) hi = vals[pos++];
          o[e] = lo | (hi << 16);
        }
        const int row = 32 * dw + src;
        *reinterpret_cast<uint4*>(ab + row * 128 + ((c ^ (row & 7)) << 4)) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->dec[s]);
    }

    // ------------------------------------------------------------ epilogue (warps 2-5)
    // Every decision that guards a warp-collective instruction or a named barrier is
    // made uniform first (vote within a warp, one shared flag across the four warps).
    const int q = warp & 3;                        // TMEM lane quarter of this warp
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;                   // weight row within the tile / rank index
    bool ok = !aborted(ctrl);
    if (ok && !mbar_wait(&ctrl->tfull, 0)) {
      record_timeout(p, ctrl);
      ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && adapter) {
      tc_fence_after();
      for (int c = 0; c < BNT; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_t + lane_base + c, v);
        tmem_ld_wait();
        if (r < p.R16) {
          const int chunk = r >> 6, cc = r & 63;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int m = c + e;
            const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[e]));
            uint8_t* dst = tbuf + chunk * (BNT * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                           (((cc >> 3) ^ (m & 7)) << 4) + (cc & 7) * 2;
            *reinterpret_cast<__nv_bfloat16*>(dst) = h;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->tready);
      if (!mbar_wait(&ctrl->fin, 0)) {
        record_timeout(p, ctrl);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
    }
    named_bar(1, 128);
    if (threadIdx.x == 64) ctrl->last = (ok && !aborted(ctrl)) ? 2 : 0;
    named_bar(1, 128);
    const bool go = *reinterpret_cast<volatile int*>(&ctrl->last) == 2;
    tc_fence_after();
    const int mvalid = min(BNT, p.M - j * BNT);
    const size_t n = static_cast<size_t>(i) * 128 + r;
    const size_t row0 = static_cast<size_t>(j) * BNT;
    __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(p.Y);
    if (go && p.splits == 1) {
      for (int c = 0; c < BNT; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_main + lane_base + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int m = c + e;
          if (m < mvalid) Y[(row0 + m) * p.N + n] = __float2bfloat16_rn(__uint_as_float(v[e]));
        }
      }
    } else if (go) {
      for (int c = 0; c < BNT; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_main + lane_base + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int m = c + e;
          if (m < mvalid) atomicAdd(&p.ws[(row0 + m) * p.N + n], __uint_as_float(v[e]));
        }
      }
      __threadfence();
      named_bar(1, 128);
      if (threadIdx.x == 64) {
        const uint32_t tile = static_cast<uint32_t>(i) * p.TT + j;
        const uint32_t prev = atomicAdd(&p.counters[tile], 1u);
        ctrl->last = prev == static_cast<uint32_t>(p.splits - 1) ? 3 : 2;
      }
      named_bar(1, 128);
      if (*reinterpret_cast<volatile int*>(&ctrl->last) == 3) {
        __threadfence();
        for (int m = 0; m < mvalid; ++m) {
          float* slot = &p.ws[(row0 + m) * p.N + n];
          Y[(row0 + m) * p.N + n] = __float2bfloat16_rn(__ldcg(slot));
          *slot = 0.0f;
        }
        if (threadIdx.x == 64) p.counters[static_cast<uint32_t>(i) * p.TT + j] = 0u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace salr
