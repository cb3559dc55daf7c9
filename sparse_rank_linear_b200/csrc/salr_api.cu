// salr_api.cu - host side of the SALR C ABI declared in include/salr.h: argument checks,
// the weight handle and its device buffers, tensor maps, schedule choice and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>

#include "../../include/salr.h"
#include "salr_codec.cuh"
#include "salr_prefill.cuh"
#include "salr_stream.cuh"
#include "salr_svd.cuh"

using namespace salr;

namespace {

constexpr uint64_t kMagic = 0x53414c5257454754ull;  // "SALRWEGT"
constexpr int kSmemLimit = 232448;  // B200 opt-in dynamic shared memory per CTA
// Token tiles (of 256) from which salr_linear expands the weight once to a dense scratch
// instead of once per token tile.  Measured on B200 with both paths built: with one token
// tile the fused decode is faster (down_proj M = 128: 51.7 against 68.0 us; up_proj
// M = 256: 70.7 against 74.1 us; large M = 128: 167 against 258 us); from two the dense
// scratch wins (up_proj M = 512: 104 against 128 us; down_proj M = 512: 107 against
// 110 us; up_proj M = 1024: 134 against 183 us).
constexpr int kDenseMinTokenTiles = 2;
// Full rounds (256-row tiles per SM) from which the dense path takes 256-row weight tiles.
// SALR_WIDE_MIN_ROUNDS overrides it (tests reach the 256-row kernel on small shapes).
constexpr int kWideMinRounds = 8;
int wide_min_rounds() {
  const char* v = getenv("SALR_WIDE_MIN_ROUNDS");
  return v && v[0] >= '0' && v[0] <= '9' ? atoi(v) : kWideMinRounds;
}

// Split-K scratch of the prefill kernel: fp32 tile sums and arrival counts (grown on
// demand, left zeroed by every call).
struct Workspace {
  float* ws = nullptr;
  size_t ws_elems = 0;
  uint32_t* counters = nullptr;
  size_t n_counters = 0;
};

// Prefill adapter scratch: t = X A_cat as bf16 [M x 128], its fp32 split sums [128 x M]
// and their arrival counts (grown on demand; sums and counts left zeroed by every call).
struct TScratch {
  uint16_t* T = nullptr;
  float* T32 = nullptr;
  uint32_t* counters = nullptr;
  int64_t rows = 0;  // token capacity (multiple of 256)
};

// Scratch of the persistent small-M kernel: fp32 sums of split row tiles [N x 64] and
// their arrival counts [N/128 x 4 quarters], the fp32 t = X A_cat accumulator [64 x 128]
// and its two counts (parts arrived, readers done).  Every call leaves all of it zero:
// the last user of each piece clears it on the device.
struct StreamScratch {
  float* acc = nullptr;
  uint32_t* counters = nullptr;
  float* tacc = nullptr;       // kTBuf floats
  uint32_t* tflags = nullptr;  // 2 counts
};
constexpr int kTBuf = 64 * 128;

}  // namespace

struct salr_weight_s {
  uint64_t magic;
  int device;
  int64_t N, K, keep, nnz;
  float sparsity;
  uint8_t* mem;  // one device allocation: [status][offsets][blob]
  uint8_t* blob;
  int64_t blob_bytes;
  uint32_t* offsets;
  int64_t nblocks;
  int* status;  // device status word (DEV_ERR_* bits)
  uint32_t max16;  // largest encoded block, 16-byte units
  Workspace work;
  TScratch tscr;
  StreamScratch sscr;
  uint8_t* x_stage;  // salr_linear_host staging
  size_t x_cap;
  uint8_t* y_stage;
  size_t y_cap;
};

namespace {

std::mutex g_mu;
std::unordered_set<salr_weight_s*>& live() {
  static std::unordered_set<salr_weight_s*> s;
  return s;
}

bool valid_handle(salr_handle h) {
  std::lock_guard<std::mutex> g(g_mu);
  return h && live().count(h) && h->magic == kMagic;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SALR_OK;
  return e == cudaErrorMemoryAllocation ? SALR_ERR_OOM : SALR_ERR_CUDA;
}

#define SALR_TRY(expr)                      \
  do {                                      \
    const cudaError_t e_ = (expr);          \
    if (e_ != cudaSuccess) return cuda_status(e_); \
  } while (0)

bool fake_oom() {
  const char* v = getenv("SALR_FAKE_OOM");
  return v && v[0] == '1';
}

cudaError_t dev_alloc(void** p, size_t bytes) {
  if (fake_oom()) return cudaErrorMemoryAllocation;
  return cudaMalloc(p, bytes);
}

// The library's stream-ordered memory pool on each device.  Freed blocks stay reserved
// for reuse up to 1 GiB (the default pool would hand them back to the driver at every
// synchronisation, and mapping them again costs about as much as a cudaMalloc).
constexpr uint64_t kPoolKeepBytes = 1ull << 30;

cudaError_t library_pool(int dev, cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = kPoolKeepBytes;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    pools[dev] = pool;
  }
  *out = pools[dev];
  return cudaSuccess;
}

// Stream-ordered allocation from the library pool (freed with cudaFreeAsync).
cudaError_t dev_alloc_async(void** p, size_t bytes, cudaStream_t st) {
  if (fake_oom()) return cudaErrorMemoryAllocation;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaMemPool_t pool;
  if ((e = library_pool(dev, &pool)) != cudaSuccess) return e;
  return cudaMallocFromPoolAsync(p, bytes, pool, st);
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// The handle's device memory, [status word][offset table][blob], in one allocation from
// the library pool, ordered on `st` (the calls that make a handle synchronise `st`
// before returning it, so any stream may use it afterwards).
cudaError_t alloc_handle_memory(salr_weight_s* h, int64_t blob_capacity, cudaStream_t st) {
  const size_t offs = round256((h->nblocks + 1) * sizeof(uint32_t));
  const cudaError_t e =
      dev_alloc_async(reinterpret_cast<void**>(&h->mem), 256 + offs + blob_capacity, st);
  if (e != cudaSuccess) return e;
  h->status = reinterpret_cast<int*>(h->mem);
  h->offsets = reinterpret_cast<uint32_t*>(h->mem + 256);
  h->blob = h->mem + 256 + offs;
  return cudaSuccess;
}

int device_sms(int dev) {
  static std::atomic<int> cache[64];  // zero-initialised: not looked up yet
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n > 0 ? n : 1;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map with 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void release(salr_weight_s* h) {
  int cur = -1;
  const bool switched = cudaGetDevice(&cur) == cudaSuccess && cur != h->device &&
                        cudaSetDevice(h->device) == cudaSuccess;
  cudaFree(h->sscr.acc);
  cudaFree(h->sscr.counters);
  cudaFree(h->sscr.tacc);
  cudaFree(h->sscr.tflags);
  // pool memory: every caller of release() has synchronised the work that used it
  if (h->mem) cudaFreeAsync(h->mem, 0);
  cudaFree(h->work.ws);
  cudaFree(h->work.counters);
  cudaFree(h->tscr.T);
  cudaFree(h->tscr.T32);
  cudaFree(h->tscr.counters);
  cudaFree(h->x_stage);
  cudaFree(h->y_stage);
  if (switched) cudaSetDevice(cur);
  h->magic = 0;
  delete h;
}

// Grow the split-K workspace to hold `elems` floats and `ctrs` counters (both zeroed).
int ensure_workspace(salr_weight_s* h, size_t elems, size_t ctrs, cudaStream_t st) {
  if (elems > h->work.ws_elems) {
    if (h->work.ws) {
      SALR_TRY(cudaStreamSynchronize(st));
      cudaFree(h->work.ws);
      h->work.ws = nullptr;
      h->work.ws_elems = 0;
    }
    void* p = nullptr;
    SALR_TRY(dev_alloc(&p, elems * sizeof(float)));
    h->work.ws = static_cast<float*>(p);
    h->work.ws_elems = elems;
    SALR_TRY(cudaMemsetAsync(p, 0, elems * sizeof(float), st));
  }
  if (ctrs > h->work.n_counters) {
    if (h->work.counters) {
      SALR_TRY(cudaStreamSynchronize(st));
      cudaFree(h->work.counters);
      h->work.counters = nullptr;
      h->work.n_counters = 0;
    }
    void* p = nullptr;
    SALR_TRY(dev_alloc(&p, ctrs * sizeof(uint32_t)));
    h->work.counters = static_cast<uint32_t*>(p);
    h->work.n_counters = ctrs;
    SALR_TRY(cudaMemsetAsync(p, 0, ctrs * sizeof(uint32_t), st));
  }
  return SALR_OK;
}

int ensure_tscratch(salr_weight_s* h, int64_t M, cudaStream_t st) {
  const int64_t rows = (M + 255) / 256 * 256;
  if (rows <= h->tscr.rows) return SALR_OK;
  if (h->tscr.T) {
    SALR_TRY(cudaStreamSynchronize(st));
    cudaFree(h->tscr.T);
    cudaFree(h->tscr.T32);
    cudaFree(h->tscr.counters);
    h->tscr = TScratch{};
  }
  void *a = nullptr, *b = nullptr, *c = nullptr;
  const size_t tb = static_cast<size_t>(rows) * 128 * sizeof(uint16_t);
  const size_t t32b = static_cast<size_t>(rows) * 128 * sizeof(float);
  const size_t cb = static_cast<size_t>(rows / 128) * 4 * sizeof(uint32_t);
  cudaError_t e;
  if ((e = dev_alloc(&a, tb)) != cudaSuccess || (e = dev_alloc(&b, t32b)) != cudaSuccess ||
      (e = dev_alloc(&c, cb)) != cudaSuccess) {
    cudaFree(a);
    cudaFree(b);
    cudaFree(c);
    return cuda_status(e);
  }
  h->tscr.T = static_cast<uint16_t*>(a);
  h->tscr.T32 = static_cast<float*>(b);
  h->tscr.counters = static_cast<uint32_t*>(c);
  h->tscr.rows = rows;
  SALR_TRY(cudaMemsetAsync(a, 0, tb, st));
  SALR_TRY(cudaMemsetAsync(b, 0, t32b, st));
  SALR_TRY(cudaMemsetAsync(c, 0, cb, st));
  return SALR_OK;
}

// The dense expansion: as many CTAs as share the SMs (about 51 KB of shared memory each),
// each walking several blocks so that staging the next one overlaps expanding this one.
cudaError_t launch_expand(const salr_weight_s* h, uint16_t* out, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(expand_dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kExpandSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const long long g = std::min<long long>(h->nblocks, 1ll * kExpandCtasPerSm * device_sms(h->device));
  expand_dense_kernel<<<static_cast<unsigned>(g < 1 ? 1 : g), 128, kExpandSmemBytes, st>>>(
      h->blob, h->offsets, static_cast<int>(h->K), static_cast<int>(h->nblocks), out, h->status);
  return cudaGetLastError();
}

template <int BNT>
int launch_t(const TParams& p, const CUtensorMap& tx, const CUtensorMap& ta, int grid,
             cudaStream_t st) {
  constexpr int smem = TLayout<BNT>::kSmemBytes;
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return SALR_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    SALR_TRY(cudaFuncSetAttribute(salr_t_kernel<BNT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem));
    attr_set[dev] = true;
  }
  salr_t_kernel<BNT><<<grid, kTThreads, smem, st>>>(p, tx, ta);
  SALR_TRY(cudaGetLastError());
  return SALR_OK;
}

// Work split of the persistent layer kernel over `tiles` output tiles of `kb` K blocks
// on `sms` CTAs.
// * Fewer tiles than CTAs: every tile is split along K into as many parts as fit in one
//   round.
// * Otherwise the tiles of the full rounds stay whole, and each CTA takes the same number
//   of them.  The rem tiles of the last, partial round are split into s parts of at most
//   ceil(kb / s) blocks.  The parts run first, so a CTA takes at most ceil(rem s / sms)
//   of them.  s minimises that bound on a CTA's extra blocks, ceil(rem s / sms)
//   ceil(kb / s), against kb for one whole tile; ties go to fewer splits.  A part keeps
//   at least 4 K blocks, and s stays at most 8, since each part adds an fp32 partial sum
//   in L2.
struct TileSplit {
  int full, splits;
};
TileSplit tail_split(int tiles, int kb, int sms) {
  if (tiles < sms) return TileSplit{0, std::max(1, std::min(kb, sms / tiles))};
  const int full = tiles / sms * sms, rem = tiles - full;
  TileSplit r{tiles, 1};
  if (rem == 0) return r;
  r.full = full;
  const int smax = std::max(1, std::min(8, kb / 4));
  long long best = kb;  // one whole tile
  for (int s = 2; s <= smax; ++s) {
    const long long parts = (static_cast<long long>(rem) * s + sms - 1) / sms;
    const long long cost = parts * ((kb + s - 1) / s);
    if (cost < best) {
      best = cost;
      r.splits = s;
    }
  }
  return r;
}

// Bound on the K blocks the busiest CTA multiplies under a work split (see tail_split).
int64_t split_makespan(int tiles, int kb, int sms, TileSplit ts) {
  const int64_t s = ts.splits;
  const int64_t part = (kb + s - 1) / s;
  if (tiles < sms) return part;  // at most one part per CTA
  const int64_t whole = static_cast<int64_t>(tiles / sms) * kb;
  const int64_t rem = tiles - ts.full;
  if (rem == 0) return whole;
  return whole + (rem * s + sms - 1) / sms * part;
}

// The launch plan of salr_linear for M tokens on `sms` SMs: the call itself and
// salr_linear_plan both take their decisions from here.  N and K are valid shapes
// (check_shape); for M > 64, K stays within kPreMaxKBlocks blocks of 64.
// Order of the prefill kernel's output tiles.  Taken token tile first, the tiles in flight
// sweep all of X every few row tiles: harmless while X stays in L2, but with X larger than
// about half of it each sweep goes back to DRAM (large M = 8192: about 6 GB of reads per
// call for 0.6 GB of operands).  Taken in groups of g row tiles, token tile by token
// tile, the `grid` tiles in flight touch g weight row tiles and about grid / g X tiles,
// and a group reads X once; g = sqrt(grid * X tile / weight tile) makes the tiles in
// flight the fewest bytes.  0 keeps the plain order.
int tile_group_rows(int rtiles, int TT, int rows, int bnt, int64_t K, int grid) {
  const char* v = getenv("SALR_TILE_GROUP_ROWS");  // tests: a group size on small shapes
  if (v && v[0] >= '0' && v[0] <= '9') {
    const int g = atoi(v);
    return g > rtiles ? rtiles : g;
  }
  const double wtile = 2.0 * rows * K, xtile = 2.0 * bnt * K;
  if (TT * xtile <= 48.0 * (1 << 20) || TT < 2) return 0;
  int g = static_cast<int>(std::lround(std::sqrt(grid * xtile / wtile)));
  return g < 1 ? 1 : g > rtiles ? rtiles : g;
}

struct LinearPlan {
  int path;     // 0 small-M kernel, 1 t + fused decode/GEMM, 2 expansion + t + dense GEMM
  int kernels;  // launches per call
  int bnt;      // tokens per MMA tile
  int rows;     // weight rows per output tile: 128, or 256 (dense path, N % 256 == 0)
  int RT, KB, TT, tiles;
  int full, splits;  // whole tiles; K parts of each later tile
  int units, grid;
  int64_t sum_bytes, dense_bytes;
  int group_rows;  // prefill tile order (tile_group_rows)
};
LinearPlan plan_linear(int64_t N, int64_t K, int64_t M, int64_t R, int sms) {
  LinearPlan p{};
  p.RT = static_cast<int>(N / 128);
  p.KB = static_cast<int>(K / 64);
  if (M <= 64) {
    p.path = 0;
    p.kernels = 1;
    p.bnt = M <= 16 ? 16 : M <= 32 ? 32 : 64;
    p.units = p.RT * p.KB;  // 128 x 64 blocks, split evenly over the CTAs
    p.grid = std::min(p.units, sms);
    return p;
  }
  p.bnt = M <= 128 ? 128 : 256;
  p.TT = static_cast<int>((M + p.bnt - 1) / p.bnt);
  const bool dense = p.TT >= kDenseMinTokenTiles;
  // Dense weight tiles of 256 rows let two MMAs share every X tile: a third fewer operand
  // bytes through shared memory per MMA cycle.  Their two accumulators fill the TMEM, so
  // a unit's epilogue no longer overlaps the next unit's MMAs; that costs a few us per
  // unit.  Measured on B200 (256-row against 128-row tiles): large M = 8192 (3584 tiles,
  // 24 rounds) 3.42 against 4.23 ms; up_proj M = 2048 (344 tiles) 214 against 203 us;
  // down_proj M = 4096 (256 tiles) 379 against 364 us.  So they are taken from
  // kWideMinRounds full rounds of 256-row tiles on, and only if the busiest CTA then gets
  // no more 128-row block steps than with 128-row tiles.
  p.rows = 128;
  if (dense && p.bnt == 256 && N % 256 == 0) {
    const int t128 = p.RT * p.TT, t256 = static_cast<int>(N / 256) * p.TT;
    const int64_t m128 = split_makespan(t128, p.KB, sms, tail_split(t128, p.KB, sms));
    const int64_t m256 = 2 * split_makespan(t256, p.KB, sms, tail_split(t256, p.KB, sms));
    if (t256 >= static_cast<int64_t>(wide_min_rounds()) * sms && m256 <= m128) p.rows = 256;
  }
  p.tiles = static_cast<int>(N / p.rows) * p.TT;
  const TileSplit ts = tail_split(p.tiles, p.KB, sms);
  p.full = ts.full;
  p.splits = ts.splits;
  p.units = ts.full + (p.tiles - ts.full) * ts.splits;
  p.grid = std::min(p.units, sms);
  p.path = dense ? 2 : 1;
  p.kernels = 1 + (R > 0 ? 1 : 0) + (dense ? 1 : 0);
  p.sum_bytes = p.splits > 1 ? static_cast<int64_t>(p.tiles - p.full) * p.rows * p.bnt * 4 : 0;
  p.dense_bytes = dense ? N * K * 2 : 0;
  p.group_rows = tile_group_rows(static_cast<int>(N / p.rows), p.TT, p.rows, p.bnt, K, p.grid);
  return p;
}

template <int BNT, bool WIDE>
int launch_prefill(PrefillParams p, const CUtensorMap& tx, const CUtensorMap& tb,
                   const CUtensorMap& tt, const CUtensorMap& tw, int grid, bool after_t,
                   cudaStream_t st) {
  using L = PrefillLayout<BNT>;
  const auto kern = salr_prefill_kernel<BNT, WIDE>;
  p.wide = WIDE ? 1 : 0;
  // Ring sizes.  Among 5 or 4 decoded-tile slots and 4 to 2 X slots, take the layout
  // with the most compact-block slots (a multiple of the group count, at most kPreMaxC):
  // compact blocks come from HBM and need the deepest queue, X tiles mostly hit L2.  Ties
  // go to more X slots, then more decoded-tile slots.
  //   The compact-block slots come in a multiple of the group count, so that slot s only
  // ever holds blocks of group s mod 4: a group then never waits on a slot whose previous
  // fill it has not consumed itself, and a parity wait can never pass on a phase two
  // fills old.  The decoded-tile ring is safe for any count of at least the group count:
  // a group's wait for the consumption of block it - SA follows its own earlier wait, at
  // block it - 4, which saw block it - 4 - SA >= it - 2 SA consumed (the MMA consumes in
  // order), so the slot can never be two phases behind.
  int sa = 0, sx = 0, sc = 0;
  p.atile = p.wide ? 2 * kPreTileBytes : kPreTileBytes;
  const int au = p.atile / kPreTileBytes;  // 16 KB units per weight-tile slot
  if (p.dense) {
    // dense weight tiles: no compact-block ring.  Four weight-tile slots and as many X
    // slots as fit (up to four): measured against 6 + 3 and 3 + 5 slots on B200, 4 + 4
    // was the fastest (down_proj M = 4096: 380 against 404 and 393 us; up_proj M = 2048
    // even).  256-row tiles take 32 KB slots: three of them and three X slots.
    sa = p.wide ? 3 : 4;
    for (sx = kPreMaxX; sx >= 2; --sx)
      if (L::smem_bytes(sa * au, sx, 0, p.cbuf) <= kSmemLimit) break;
    if (sx < 2) return SALR_ERR_UNSUPPORTED;
    sc = kPreGroups;  // placeholder so the check below passes; no slot is used
  }
  for (int a = kPreGroups + 1; a >= kPreGroups && !p.dense; --a) {
    for (int x = kPreMaxX; x >= 2; --x) {
      int c = (kSmemLimit - L::smem_bytes(a, x, 0, p.cbuf)) / p.cbuf;
      if (c > kPreMaxC) c = kPreMaxC;
      c -= c % kPreGroups;
      if (c > sc || (c == sc && c > 0 && (x > sx || (x == sx && a > sa)))) {
        sa = a;
        sx = x;
        sc = c;
      }
    }
  }
  if (sc < kPreGroups) return SALR_ERR_UNSUPPORTED;
  p.sa = sa;
  p.sx = sx;
  p.sc = p.dense ? 0 : sc;
  const int smem = L::smem_bytes(p.sa * au, p.sx, p.sc, p.cbuf);
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return SALR_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    SALR_TRY(cudaFuncSetAttribute(kern,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    attr_set[dev] = true;
  }
  // Directly after the t kernel, the launch may overlap it (programmatic stream
  // serialization): the t kernel started only once everything before it had completed,
  // and the layer kernel waits for the t kernel itself before its first read of t.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPreThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_t ? 1 : 0;
  SALR_TRY(cudaLaunchKernelEx(&cfg, kern, p, tx, tb, tt, tw));
  return SALR_OK;
}

// Persistent small-M path: one CTA per SM, launched so that it may overlap the preceding
// kernel of the stream.
constexpr int kStreamDecoders = 4 * kStreamGroups;  // one warp per row quarter in each group

int ensure_stream_scratch(salr_weight_s* h, cudaStream_t st) {
  if (h->sscr.acc) return SALR_OK;
  void *a = nullptr, *b = nullptr, *c = nullptr, *d = nullptr;
  const size_t ab = static_cast<size_t>(h->N) * 64 * sizeof(float);
  const size_t cb = static_cast<size_t>(h->N / 128) * 4 * sizeof(uint32_t);
  const size_t tb = kTBuf * sizeof(float);
  cudaError_t e;
  if ((e = dev_alloc(&a, ab)) != cudaSuccess || (e = dev_alloc(&b, cb)) != cudaSuccess ||
      (e = dev_alloc(&c, tb)) != cudaSuccess || (e = dev_alloc(&d, 2 * sizeof(uint32_t))) != cudaSuccess) {
    cudaFree(a);
    cudaFree(b);
    cudaFree(c);
    cudaFree(d);
    return cuda_status(e);
  }
  h->sscr.acc = static_cast<float*>(a);
  h->sscr.counters = static_cast<uint32_t*>(b);
  h->sscr.tacc = static_cast<float*>(c);
  h->sscr.tflags = static_cast<uint32_t*>(d);
  SALR_TRY(cudaMemsetAsync(a, 0, ab, st));
  SALR_TRY(cudaMemsetAsync(b, 0, cb, st));
  SALR_TRY(cudaMemsetAsync(c, 0, tb, st));
  SALR_TRY(cudaMemsetAsync(d, 0, 2 * sizeof(uint32_t), st));
  return SALR_OK;
}

// Point the kernel at its scratch (all of it zero between calls).
void bind_call(StreamParams& sp, float* acc, uint32_t* counters, float* tacc, uint32_t* tflags) {
  sp.acc = acc;
  sp.counters = counters;
  sp.tacc = tacc;
  sp.tflag = tflags;
}

// The bound on device-side waits, in SM cycles: kWaitLimitCycles (about 1 s), or
// SALR_WAIT_LIMIT_CYCLES (failure tests make waits run out quickly with it).  Copied to
// the device on the call's stream whenever it differs from the value last sent there.
cudaError_t apply_wait_limit(cudaStream_t st) {
  static std::atomic<long long> sent[64];  // 0: the module's initial value
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e;
  const char* v = getenv("SALR_WAIT_LIMIT_CYCLES");
  long long want = v && v[0] >= '0' && v[0] <= '9' ? atoll(v) : kWaitLimitCycles;
  if (want < 1000) want = 1000;
  const long long have = sent[dev].load() == 0 ? kWaitLimitCycles : sent[dev].load();
  if (want == have) return cudaSuccess;
  static long long staged[64];  // stays valid while the copy is queued
  staged[dev] = want;
  e = cudaMemcpyToSymbolAsync(g_wait_limit, &staged[dev], sizeof(long long), 0,
                              cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) sent[dev] = want;
  return e;
}

// Compact blocks per bulk copy: as many as make about 40 KB (at most 4).  A bulk copy
// occupies the SM's copy engine for about 540 cycles whatever its size (measured on B200
// from L2: 2 to 32 KB per copy, 2 to 8 copies in flight, 1 or 148 CTAs), so copies of
// single ~9 KB blocks cap a CTA near 17 bytes per cycle, about 5 TB/s over 148 SMs, before
// anything else shares the engine.
int stream_blocks_per_copy(uint32_t max16) {
  const int blockb = static_cast<int>(max16) * 16;
  const int b = 40960 / (blockb > 0 ? blockb : 1);
  return b < 1 ? 1 : b > kStreamMaxBpc ? kStreamMaxBpc : b;
}

template <int BNT>
int launch_stream(StreamParams p, const CUtensorMap& tx, const CUtensorMap& ta,
                  const CUtensorMap& tb, int sms, cudaStream_t st) {
  using L = StreamLayout<BNT>;
  constexpr int kThreads = 32 * (kStreamFixedWarps + kStreamDecoders + kStreamGroups);
  p.bcbuf = L::bcat_bytes(p.R16);
  // rebuilt-block ring (TMEM slots, each with its X tile in shared memory): two per
  // decoder group, so that a group only ever waits for the MMAs of its own block before
  // last; the rest of shared memory becomes compact-block entries, which set how many
  // blocks are in flight from HBM
  p.sa = 2 * kStreamGroups;
  const int fixed = L::smem_bytes(p.cbuf, p.bcbuf, p.sa, 0);
  // The rest of shared memory becomes super-slots, one bulk copy of p.bpc blocks each.  A
  // super-slot is refilled only once every decoder warp of all its blocks has counted out,
  // so no warp can wait on a fill two phases old.
  int sc = (kSmemLimit - fixed) / p.cbuf;
  if (sc > kStreamMaxC) sc = kStreamMaxC;
  if (sc < 2) return SALR_ERR_UNSUPPORTED;
  p.sc = sc;
  const int smem = L::smem_bytes(p.cbuf, p.bcbuf, p.sa, p.sc);
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return SALR_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    SALR_TRY(cudaFuncSetAttribute(salr_stream_kernel<BNT, kStreamDecoders>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    attr_set[dev] = true;
  }
  const long long units = p.units;
  const int grid = static_cast<int>(units < sms ? units : sms);
  p.tshare = grid < p.kblocks ? grid : p.kblocks;
  // SALR_STREAM_SKEW=S (0 .. 255): ranges that shrink with the CTA index (stream_split)
  const char* sk = getenv("SALR_STREAM_SKEW");
  const int skew = sk && sk[0] >= '0' && sk[0] <= '9' ? atoi(sk) : 0;
  // (at most 192: the last CTA keeps at least a quarter of the first one's share; none
  // below 4 blocks a CTA)
  p.skew = units < 4ll * grid ? 0 : skew < 0 ? 0 : skew > 192 ? 192 : skew;
  p.treaders = stream_t_readers(units, grid, p.kblocks, p.skew);
  // SALR_FAIL_T_WAIT=1 (failure tests only): the readers of t wait for one part more
  // than are ever added, so their bounded wait runs out and the call reports a timeout
  const char* ft = getenv("SALR_FAIL_T_WAIT");
  p.twant = p.tshare + (ft && ft[0] == '1' ? 1 : 0);
  SALR_TRY(apply_wait_limit(st));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // One CTA per SM (the shared-memory footprint admits no second one); cross-CTA waits
  // go to lower-indexed CTAs or to the t-share CTAs, which wait on nothing before
  // finishing their share.  The launch may overlap the preceding kernel of the stream
  // (programmatic stream serialization): the kernel waits for it before touching
  // anything but the weight blob.  SALR_COOPERATIVE=1 asks for a cooperative launch
  // instead, which guarantees co-residency outright.
  cudaLaunchAttribute attr[1];
  const char* coop = getenv("SALR_COOPERATIVE");
  if (coop && coop[0] == '1') {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SALR_TRY(cudaLaunchKernelEx(&cfg, salr_stream_kernel<BNT, kStreamDecoders>, p, tx, ta,
                              tb));
  return SALR_OK;
}

// Output tiles of 128 x 128 beyond 2^27 would let the layer kernel's work units (up to 8
// parts per tile) overflow its 32-bit counts; such an output (M x N) is far beyond any
// GPU's memory anyway.
bool too_many_tiles(int64_t N, int64_t M) { return (N / 128) * ((M + 127) / 128) > (1ll << 27); }

int check_linear_args(const void* X, int64_t M, salr_handle h, const void* A, const void* B,
                      int64_t R, const void* Y) {
  if (!valid_handle(h)) return SALR_ERR_INVALID;
  if (!X || !Y || M < 1) return SALR_ERR_INVALID;
  if (R < 0) return SALR_ERR_INVALID;
  if (R > 0 && (!A || !B)) return SALR_ERR_INVALID;
  if (R % 8 != 0 || R > 128) return SALR_ERR_UNSUPPORTED;
  if (M > (1ll << 24)) return SALR_ERR_UNSUPPORTED;
  if (too_many_tiles(h->N, M)) return SALR_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(Y) || (R > 0 && (!aligned16(A) || !aligned16(B))))
    return SALR_ERR_UNSUPPORTED;
  return SALR_OK;
}

}  // namespace

int noalloc_reset(int dev);  // defined with salr_linear_noalloc below

namespace {

constexpr char kImageMagic[8] = {'S', 'A', 'L', 'R', 'B', 'L', 'K', '1'};
// Version 2: block values in quarter / 4-column group / row / column order (version 1 held
// them row-major and is refused).
constexpr uint32_t kImageVersion = 2;
constexpr int64_t kImageHeader = 64;

struct ImageHeader {
  char magic[8];
  uint32_t version;
  uint32_t header_bytes;
  int64_t N, K, keep, nnz;
  float sparsity;
  uint32_t zero;
  int64_t blob_bytes;
};
static_assert(sizeof(ImageHeader) == kImageHeader, "image header is 64 bytes");

int64_t image_offsets_bytes(int64_t nblocks) { return ((nblocks + 1) * 4 + 15) / 16 * 16; }

int64_t keep_for(int64_t K, float sparsity) {
  return K - static_cast<int64_t>(std::floor(static_cast<double>(sparsity) * K));
}

// the shape rules salr_encode applies, shared by salr_load
int check_shape(int64_t N, int64_t K) {
  if (N < 128 || K < 64 || N % 128 || K % 64 || K > 64 * kPreMaxKBlocks) return SALR_ERR_UNSUPPORTED;
  if (N > (1ll << 22)) return SALR_ERR_UNSUPPORTED;
  return SALR_OK;
}

void publish(salr_weight_s* h, salr_handle* out) {
  h->magic = kMagic;
  {
    std::lock_guard<std::mutex> g(g_mu);
    live().insert(h);
  }
  *out = h;
}

}  // namespace

extern "C" {

const char* salr_status_string(int status) {
  switch (status) {
    case SALR_OK: return "SALR_OK";
    case SALR_ERR_INVALID: return "SALR_ERR_INVALID";
    case SALR_ERR_UNSUPPORTED: return "SALR_ERR_UNSUPPORTED";
    case SALR_ERR_CUDA: return "SALR_ERR_CUDA";
    case SALR_ERR_OOM: return "SALR_ERR_OOM";
    case SALR_ERR_TIMEOUT: return "SALR_ERR_TIMEOUT";
    default: return "SALR_ERR_UNKNOWN";
  }
}

int salr_encode(const void* W, int64_t N, int64_t K, float sparsity, void* stream,
                salr_handle* out) {
  if (!W || !out) return SALR_ERR_INVALID;
  if (!(sparsity >= 0.0f && sparsity < 1.0f)) return SALR_ERR_INVALID;
  const int shape = check_shape(N, K);
  if (shape != SALR_OK) return shape;
  if (!aligned16(W)) return SALR_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t keep = keep_for(K, sparsity);
  const int64_t nwords = K / 64;
  const int64_t nblocks = (N / 128) * nwords;

  // The blob is written straight into the handle: its capacity is the largest size the
  // kept count allows (each block pads its values by at most 14 bytes), so the encoder
  // needs no size round trip to the host before writing it.
  const int64_t capacity = (kBitmapBytes + 16) * nblocks + 2 * N * keep;
  if (capacity / 16 >= (1ll << 32)) return SALR_ERR_UNSUPPORTED;  // offsets are uint32 x 16 B

  salr_weight_s* h = new (std::nothrow) salr_weight_s();
  if (!h) return SALR_ERR_OOM;
  std::memset(h, 0, sizeof(*h));
  cudaGetDevice(&h->device);
  h->N = N;
  h->K = K;
  h->keep = keep;
  h->sparsity = sparsity;
  h->nblocks = nblocks;

  // scratch: the row-major bitmap, block sizes, and [kept entries, largest block]
  uint8_t* scratch = nullptr;
  const size_t bits_bytes = round256(N * nwords * sizeof(uint64_t));
  const size_t size_bytes = round256(nblocks * sizeof(uint32_t));
  auto fail = [&](int code) {
    if (scratch) cudaFreeAsync(scratch, st);
    cudaStreamSynchronize(st);
    release(h);
    return code;
  };
  cudaError_t e;
  if ((e = alloc_handle_memory(h, capacity, st)) != cudaSuccess ||
      (e = dev_alloc_async(reinterpret_cast<void**>(&scratch), bits_bytes + size_bytes + 256,
                           st)) != cudaSuccess)
    return fail(cuda_status(e));
  uint64_t* bits = reinterpret_cast<uint64_t*>(scratch);
  uint32_t* size16 = reinterpret_cast<uint32_t*>(scratch + bits_bytes);
  unsigned long long* nnz_d = reinterpret_cast<unsigned long long*>(scratch + bits_bytes + size_bytes);
  if ((e = cudaMemsetAsync(h->status, 0, sizeof(int), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(nnz_d, 0, 2 * sizeof(unsigned long long), st)) != cudaSuccess)
    return fail(cuda_status(e));

  const int mask_smem = static_cast<int>(K * sizeof(uint16_t));
  if (mask_smem > 48 * 1024) {
    static std::atomic<bool> attr_set[64];  // zero-initialised: false
    if (h->device < 0 || h->device >= 64) return fail(SALR_ERR_UNSUPPORTED);
    if (!attr_set[h->device]) {
      if ((e = cudaFuncSetAttribute(encode_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    mask_smem)) != cudaSuccess)
        return fail(cuda_status(e));
      attr_set[h->device] = true;
    }
  }
  encode_mask_kernel<<<static_cast<unsigned>(N), kEncThreads, mask_smem, st>>>(
      static_cast<const uint16_t*>(W), static_cast<int>(K), static_cast<int>(keep), bits,
      h->status);
  encode_count_kernel<<<static_cast<unsigned>((nblocks + 7) / 8), 256, 0, st>>>(
      bits, static_cast<int>(nwords), static_cast<int>(nblocks), size16, nnz_d,
      reinterpret_cast<unsigned int*>(nnz_d + 1));
  const unsigned long long cap16 = static_cast<unsigned long long>(capacity / 16);
  encode_scan_kernel<<<1, 1024, 0, st>>>(size16, static_cast<int>(nblocks), cap16, h->offsets,
                                         h->status);
  encode_scatter_kernel<<<static_cast<unsigned>(nblocks), kBlockRows, 0, st>>>(
      static_cast<const uint16_t*>(W), static_cast<int>(K), bits, h->offsets, cap16, h->blob,
      h->status);
  if ((e = cudaGetLastError()) != cudaSuccess) return fail(cuda_status(e));

  uint32_t total16 = 0;
  int status = 0;
  unsigned long long nnz[2] = {0, 0};
  if ((e = cudaMemcpyAsync(&total16, h->offsets + nblocks, sizeof(uint32_t),
                           cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(&status, h->status, sizeof(int), cudaMemcpyDeviceToHost, st)) !=
          cudaSuccess ||
      (e = cudaMemcpyAsync(nnz, nnz_d, 2 * sizeof(unsigned long long), cudaMemcpyDeviceToHost,
                           st)) != cudaSuccess ||
      (e = cudaFreeAsync(scratch, st)) != cudaSuccess)
    return fail(cuda_status(e));
  scratch = nullptr;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return fail(cuda_status(e));
  if (status & DEV_ERR_NAN) return fail(SALR_ERR_INVALID);
  if (status & DEV_ERR_RANGE) return fail(SALR_ERR_UNSUPPORTED);

  h->nnz = static_cast<int64_t>(nnz[0]);
  h->max16 = static_cast<uint32_t>(nnz[1]);
  h->blob_bytes = static_cast<int64_t>(total16) * 16;
  publish(h, out);
  return SALR_OK;
}

int salr_decode(salr_handle h, void* W_out, void* stream) {
  if (!valid_handle(h) || !W_out) return SALR_ERR_INVALID;
  if (!aligned16(W_out)) return SALR_ERR_UNSUPPORTED;
  SALR_TRY(launch_expand(h, static_cast<uint16_t*>(W_out), static_cast<cudaStream_t>(stream)));
  return SALR_OK;
}

int salr_linear_plan(int64_t N, int64_t K, int64_t M, int64_t R, int32_t sms, salr_plan* out) {
  if (!out || M < 1 || R < 0 || sms < 0) return SALR_ERR_INVALID;
  const int shape = check_shape(N, K);
  if (shape != SALR_OK) return shape;
  if (R % 8 != 0 || R > 128 || M > (1ll << 24) || too_many_tiles(N, M)) return SALR_ERR_UNSUPPORTED;
  if (sms == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return SALR_ERR_CUDA;
    }
    sms = n;
  }
  const LinearPlan p = plan_linear(N, K, M, R, sms);
  out->path = p.path;
  out->kernels = p.kernels;
  out->token_tile = p.bnt;
  out->tile_rows = p.path == 0 ? 128 : p.rows;
  out->grid = p.grid;
  out->units = p.units;
  out->tiles = p.tiles;
  out->whole_tiles = p.path == 0 ? 0 : p.splits == 1 ? p.tiles : p.full;
  out->splits = p.path == 0 ? 1 : p.splits;
  out->split_sum_bytes = p.sum_bytes;
  out->dense_scratch_bytes = p.dense_bytes;
  out->group_rows = p.group_rows;
  return SALR_OK;
}

int salr_linear(const void* X, int64_t M, salr_handle h, const void* A_cat, const void* B_cat,
                int64_t R, void* Y, void* stream) {
  int rc = check_linear_args(X, M, h, A_cat, B_cat, R, Y);
  if (rc != SALR_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M <= 64) {
    rc = ensure_stream_scratch(h, st);
    if (rc != SALR_OK) return rc;
    const int bnt = M <= 16 ? 16 : M <= 32 ? 32 : 64;
    StreamParams sp{};
    sp.blob = h->blob;
    sp.offsets = h->offsets;
    sp.Y = static_cast<uint16_t*>(Y);
    bind_call(sp, h->sscr.acc, h->sscr.counters, h->sscr.tacc, h->sscr.tflags);
    sp.status = h->status;
    sp.N = static_cast<int>(h->N);
    sp.K = static_cast<int>(h->K);
    sp.M = static_cast<int>(M);
    sp.R = static_cast<int>(R);
    sp.R16 = static_cast<int>((R + 15) / 16 * 16);
    sp.kblocks = static_cast<int>(h->K / 64);
    sp.RT = static_cast<int>(h->N / 128);
    sp.units = sp.RT * sp.kblocks;
    sp.bpc = stream_blocks_per_copy(h->max16);
    sp.cbuf = static_cast<int>((sp.bpc * h->max16 * 16 + 32 + 1023) / 1024 * 1024);
    sp.X = static_cast<const uint16_t*>(X);
    CUtensorMap tx, ta, tb;
    std::memset(&ta, 0, sizeof(ta));
    std::memset(&tb, 0, sizeof(tb));
    if (!make_map(&tx, X, h->K, M, 64, bnt)) return SALR_ERR_CUDA;
    if (R > 0) {
      if (!make_map(&ta, A_cat, R, h->K, 64, 64)) return SALR_ERR_CUDA;
      if (!make_map(&tb, B_cat, h->N, R, 64, sp.R16)) return SALR_ERR_CUDA;
    }
    const int sms = device_sms(h->device);
    switch (bnt) {
      case 16: rc = launch_stream<16>(sp, tx, ta, tb, sms, st); break;
      case 32: rc = launch_stream<32>(sp, tx, ta, tb, sms, st); break;
      default: rc = launch_stream<64>(sp, tx, ta, tb, sms, st);
    }
    return rc;
  }
  // prefill shapes: t = X A_cat once (own kernel), then the fused decode + GEMM
  const int sms = device_sms(h->device);
  if (h->K / 64 > kPreMaxKBlocks) return SALR_ERR_UNSUPPORTED;
  const LinearPlan pl = plan_linear(h->N, h->K, M, R, sms);
  const int bnt = pl.bnt, TT = pl.TT, KB = pl.KB;
  const int R16 = static_cast<int>((R + 15) / 16 * 16);
  CUtensorMap tx, ta, tb, tt;
  std::memset(&ta, 0, sizeof(ta));
  std::memset(&tb, 0, sizeof(tb));
  std::memset(&tt, 0, sizeof(tt));
  if (!make_map(&tx, X, h->K, M, 64, bnt)) return SALR_ERR_CUDA;
  // the layer kernel's parameters and scratch first: nothing may be queued between the
  // t kernel and the layer kernel, which may start while t is still running
  PrefillParams pp{};
  pp.blob = h->blob;
  pp.offsets = h->offsets;
  pp.Y = static_cast<uint16_t*>(Y);
  pp.status = h->status;
  pp.N = static_cast<int>(h->N);
  pp.K = static_cast<int>(h->K);
  pp.M = static_cast<int>(M);
  pp.R16 = R > 0 ? R16 : 0;
  pp.kblocks = KB;
  pp.TT = TT;
  pp.cbuf = static_cast<int>((h->max16 * 16 + 32 + 1023) / 1024 * 1024);
  pp.full = pl.full;
  pp.splits = pl.splits;
  if (pp.splits > 1) {
    const size_t ntail = static_cast<size_t>(pl.tiles - pl.full);
    rc = ensure_workspace(h, ntail * pl.rows * bnt, ntail * 4, st);
    if (rc != SALR_OK) return rc;
    pp.acc = h->work.ws;
    pp.counters = h->work.counters;
  }
  // persistent: at most one CTA per SM, each taking units cta, cta + grid, ...
  pp.units = pl.units;
  const int grid = pl.grid;
  // With several token tiles, every weight block would be expanded once per token tile.
  // Then the weight is expanded once into a dense scratch from the library pool (freed
  // in stream order after the call), and the layer kernel takes its weight tiles from
  // there by TMA.
  CUtensorMap tw;
  std::memset(&tw, 0, sizeof(tw));
  uint8_t* wdense = nullptr;
  pp.dense = pl.path == 2 ? 1 : 0;
  pp.wide = pl.rows == 256 ? 1 : 0;
  pp.rtiles = static_cast<int>(h->N / pl.rows);
  pp.group_rows = pl.group_rows;
  if (pp.dense) {
    const cudaError_t e =
        dev_alloc_async(reinterpret_cast<void**>(&wdense), static_cast<size_t>(h->N) * h->K * 2, st);
    if (e != cudaSuccess) return cuda_status(e);
    const cudaError_t le = launch_expand(h, reinterpret_cast<uint16_t*>(wdense), st);
    if (le != cudaSuccess || !make_map(&tw, wdense, h->K, h->N, 64, 128)) {
      cudaFreeAsync(wdense, st);
      return le != cudaSuccess ? cuda_status(le) : SALR_ERR_CUDA;
    }
  }
  auto release_dense = [&](int code) {
    if (wdense) cudaFreeAsync(wdense, st);
    return code;
  };
  if (R > 0) {
    rc = ensure_tscratch(h, M, st);
    if (rc != SALR_OK) return release_dense(rc);
    if (!make_map(&ta, A_cat, R, h->K, 64, 64)) return release_dense(SALR_ERR_CUDA);
    // B_cat^T in chunks of 64 ranks (ranks past R read as zero)
    if (!make_map(&tb, B_cat, h->N, R, 64, 64)) return release_dense(SALR_ERR_CUDA);
    if (!make_map(&tt, h->tscr.T, 128, M, 64, bnt)) return release_dense(SALR_ERR_CUDA);
    TParams tp{};
    tp.T = h->tscr.T;
    tp.T32 = h->tscr.T32;
    tp.counters = h->tscr.counters;
    tp.status = h->status;
    tp.M = static_cast<int>(M);
    tp.R16 = R16;
    tp.kblocks = KB;
    tp.TT = TT;
    // At least four K blocks per CTA: the split sums meet in L2, and a few blocks per CTA
    // keep that reduction narrow.  The layer kernel launches as soon as the t kernel has
    // started and needs t only for its adapter iterations, at the end of each unit; when
    // the layer kernel leaves SMs free, the t kernel keeps to those, so that both run at
    // once and no layer CTA waits for an SM.
    const int free_sms = grid < sms ? sms - grid : sms;
    tp.splits = std::max(1, std::min(KB / 4, free_sms / TT));
    rc = bnt == 128 ? launch_t<128>(tp, tx, ta, TT * tp.splits, st)
                    : launch_t<256>(tp, tx, ta, TT * tp.splits, st);
    if (rc != SALR_OK) return release_dense(rc);
  }
  rc = bnt == 128  ? launch_prefill<128, false>(pp, tx, tb, tt, tw, grid, R > 0, st)
       : pp.wide    ? launch_prefill<256, true>(pp, tx, tb, tt, tw, grid, R > 0, st)
                    : launch_prefill<256, false>(pp, tx, tb, tt, tw, grid, R > 0, st);
  return release_dense(rc);
}

int salr_linear_host(const void* X_host, int64_t M, salr_handle h, const void* A_cat,
                     const void* B_cat, int64_t R, void* Y_host, void* stream) {
  if (!valid_handle(h) || !X_host || !Y_host || M < 1) return SALR_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(M) * h->K * 2, yb = static_cast<size_t>(M) * h->N * 2;
  if (xb > h->x_cap) {
    SALR_TRY(cudaStreamSynchronize(st));
    cudaFree(h->x_stage);
    h->x_stage = nullptr;
    h->x_cap = 0;
    SALR_TRY(dev_alloc(reinterpret_cast<void**>(&h->x_stage), xb));
    h->x_cap = xb;
  }
  if (yb > h->y_cap) {
    SALR_TRY(cudaStreamSynchronize(st));
    cudaFree(h->y_stage);
    h->y_stage = nullptr;
    h->y_cap = 0;
    SALR_TRY(dev_alloc(reinterpret_cast<void**>(&h->y_stage), yb));
    h->y_cap = yb;
  }
  SALR_TRY(cudaMemcpyAsync(h->x_stage, X_host, xb, cudaMemcpyHostToDevice, st));
  const int rc = salr_linear(h->x_stage, M, h, A_cat, B_cat, R, h->y_stage, stream);
  if (rc != SALR_OK) return rc;
  SALR_TRY(cudaMemcpyAsync(Y_host, h->y_stage, yb, cudaMemcpyDeviceToHost, st));
  return SALR_OK;
}

int salr_free(salr_handle h) {
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!h || !live().count(h) || h->magic != kMagic) return SALR_ERR_INVALID;
    live().erase(h);
  }
  cudaDeviceSynchronize();
  release(h);
  return SALR_OK;
}

int salr_info(salr_handle h, int64_t* N, int64_t* K, int64_t* nnz, int64_t* bytes) {
  if (!valid_handle(h)) return SALR_ERR_INVALID;
  if (N) *N = h->N;
  if (K) *K = h->K;
  if (nnz) *nnz = h->nnz;
  if (bytes) *bytes = h->blob_bytes + (h->nblocks + 1) * static_cast<int64_t>(sizeof(uint32_t));
  return SALR_OK;
}

int salr_format_view(salr_handle h, const void** blob, int64_t* blob_bytes, const void** offsets,
                     int64_t* n_offsets) {
  if (!valid_handle(h)) return SALR_ERR_INVALID;
  if (blob) *blob = h->blob;
  if (blob_bytes) *blob_bytes = h->blob_bytes;
  if (offsets) *offsets = h->offsets;
  if (n_offsets) *n_offsets = h->nblocks + 1;
  return SALR_OK;
}

// ------------------------------------------------------------------------------------
// Serialised image of a handle: the byte form of the compressed weight.  Layout (all
// little-endian; include/salr.h documents it for readers of the files):
//   [0,64)   header: "SALRBLK1", u32 version 2, u32 header bytes 64, i64 N, i64 K,
//            i64 keep, i64 nnz, f32 sparsity, u32 0, i64 blob bytes
//   [64,..)  offset table, (nblocks + 1) x u32, zero padded to a multiple of 16 bytes
//   then     the blob (bitmaps, kept values, zero padding), exactly as on the device
// ------------------------------------------------------------------------------------
int salr_save_size(salr_handle h, int64_t* bytes) {
  if (!valid_handle(h) || !bytes) return SALR_ERR_INVALID;
  *bytes = kImageHeader + image_offsets_bytes(h->nblocks) + h->blob_bytes;
  return SALR_OK;
}

int salr_save(salr_handle h, void* buf, int64_t buf_bytes, void* stream) {
  int64_t need = 0;
  if (salr_save_size(h, &need) != SALR_OK || !buf) return SALR_ERR_INVALID;
  if (buf_bytes < need) return SALR_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* out = static_cast<uint8_t*>(buf);
  ImageHeader hd;
  std::memset(&hd, 0, sizeof(hd));
  std::memcpy(hd.magic, kImageMagic, sizeof(hd.magic));
  hd.version = kImageVersion;
  hd.header_bytes = static_cast<uint32_t>(kImageHeader);
  hd.N = h->N;
  hd.K = h->K;
  hd.keep = h->keep;
  hd.nnz = h->nnz;
  hd.sparsity = h->sparsity;
  hd.blob_bytes = h->blob_bytes;
  std::memcpy(out, &hd, sizeof(hd));
  const int64_t ob = image_offsets_bytes(h->nblocks);
  const int64_t used = (h->nblocks + 1) * 4;
  std::memset(out + kImageHeader + used, 0, ob - used);
  SALR_TRY(cudaMemcpyAsync(out + kImageHeader, h->offsets, used, cudaMemcpyDeviceToHost, st));
  SALR_TRY(cudaMemcpyAsync(out + kImageHeader + ob, h->blob, h->blob_bytes,
                           cudaMemcpyDeviceToHost, st));
  SALR_TRY(cudaStreamSynchronize(st));
  return SALR_OK;
}

int salr_load(const void* buf, int64_t buf_bytes, void* stream, salr_handle* out) {
  if (!buf || !out || buf_bytes < kImageHeader) return SALR_ERR_INVALID;
  const uint8_t* in = static_cast<const uint8_t*>(buf);
  ImageHeader hd;
  std::memcpy(&hd, in, sizeof(hd));
  if (std::memcmp(hd.magic, kImageMagic, sizeof(hd.magic)) != 0 || hd.version != kImageVersion ||
      hd.header_bytes != kImageHeader || hd.zero != 0)
    return SALR_ERR_INVALID;
  if (!(hd.sparsity >= 0.0f && hd.sparsity < 1.0f)) return SALR_ERR_INVALID;
  const int shape = check_shape(hd.N, hd.K);
  if (shape != SALR_OK) return shape;
  if (hd.keep != keep_for(hd.K, hd.sparsity) || hd.nnz != hd.N * hd.keep) return SALR_ERR_INVALID;
  const int64_t nwords = hd.K / 64;
  const int64_t nblocks = (hd.N / 128) * nwords;
  const int64_t ob = image_offsets_bytes(nblocks);
  if (hd.blob_bytes < 0 || hd.blob_bytes % 16 ||
      hd.blob_bytes > (buf_bytes - kImageHeader - ob))
    return SALR_ERR_INVALID;
  // offsets: from 0, each block at least its bitmap and at most a dense block, ending at
  // the blob's end.  These bounds keep every device read of the checks below in range.
  const uint8_t* offs_in = in + kImageHeader;
  constexpr uint32_t kMin16 = kBitmapBytes / 16;
  constexpr uint32_t kMax16 = (kBitmapBytes + 2 * kBlockRows * kBlockCols) / 16;
  uint32_t prev = 0, max16 = 0;
  std::memcpy(&prev, offs_in, 4);
  if (prev != 0) return SALR_ERR_INVALID;
  for (int64_t b = 1; b <= nblocks; ++b) {
    uint32_t cur;
    std::memcpy(&cur, offs_in + 4 * b, 4);
    if (cur < prev || cur - prev < kMin16 || cur - prev > kMax16) return SALR_ERR_INVALID;
    max16 = std::max(max16, cur - prev);
    prev = cur;
  }
  if (static_cast<int64_t>(prev) * 16 != hd.blob_bytes) return SALR_ERR_INVALID;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  salr_weight_s* h = new (std::nothrow) salr_weight_s();
  if (!h) return SALR_ERR_OOM;
  std::memset(h, 0, sizeof(*h));
  cudaGetDevice(&h->device);
  h->N = hd.N;
  h->K = hd.K;
  h->keep = hd.keep;
  h->sparsity = hd.sparsity;
  h->nblocks = nblocks;
  h->max16 = max16;
  h->blob_bytes = hd.blob_bytes;
  uint32_t* row_keep = nullptr;
  unsigned long long* nnz_d = nullptr;
  auto fail = [&](int code) {
    cudaStreamSynchronize(st);
    cudaFree(row_keep);
    cudaFree(nnz_d);
    release(h);
    return code;
  };
  cudaError_t e;
  if ((e = alloc_handle_memory(h, h->blob_bytes, st)) != cudaSuccess ||
      (e = dev_alloc(reinterpret_cast<void**>(&row_keep), hd.N * sizeof(uint32_t))) !=
          cudaSuccess ||
      (e = dev_alloc(reinterpret_cast<void**>(&nnz_d), sizeof(unsigned long long))) !=
          cudaSuccess)
    return fail(cuda_status(e));
  if ((e = cudaMemsetAsync(h->status, 0, sizeof(int), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(row_keep, 0, hd.N * sizeof(uint32_t), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(nnz_d, 0, sizeof(unsigned long long), st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->offsets, offs_in, (nblocks + 1) * sizeof(uint32_t),
                           cudaMemcpyHostToDevice, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->blob, in + kImageHeader + ob, h->blob_bytes,
                           cudaMemcpyHostToDevice, st)) != cudaSuccess)
    return fail(cuda_status(e));
  load_check_blocks_kernel<<<static_cast<unsigned>((nblocks + 7) / 8), 256, 0, st>>>(
      h->blob, h->offsets, static_cast<int>(nwords), static_cast<int>(nblocks), row_keep, nnz_d,
      h->status);
  load_check_rows_kernel<<<static_cast<unsigned>((hd.N + 255) / 256), 256, 0, st>>>(
      row_keep, static_cast<int>(hd.N), static_cast<uint32_t>(hd.keep), h->status);
  if ((e = cudaGetLastError()) != cudaSuccess) return fail(cuda_status(e));
  int status = 0;
  unsigned long long nnz = 0;
  if ((e = cudaMemcpyAsync(&status, h->status, sizeof(int), cudaMemcpyDeviceToHost, st)) !=
          cudaSuccess ||
      (e = cudaMemcpyAsync(&nnz, nnz_d, sizeof(nnz), cudaMemcpyDeviceToHost, st)) !=
          cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess)
    return fail(cuda_status(e));
  if (status != 0 || static_cast<int64_t>(nnz) != hd.nnz) return fail(SALR_ERR_INVALID);
  h->nnz = hd.nnz;
  cudaFree(row_keep);
  cudaFree(nnz_d);
  publish(h, out);
  return SALR_OK;
}

// ------------------------------------------------------------------------------------
// salr_residual_adapter: the rank-r adapter of the pruning residual (salr_svd.cuh).
// ------------------------------------------------------------------------------------
}  // extern "C"

namespace {

template <typename TA, bool TR, int MODE>
cudaError_t launch_skinny(const TA* A, int lda, int rows, int red, const float* Bm, int ldb,
                          int ncols, float* outf, uint16_t* outb, int ldo, int sms,
                          cudaStream_t st) {
  const int tiles = rows / 64;
  int splits = 1;
  if (MODE == 0) splits = std::max(1, std::min(red / 32, (2 * sms + tiles - 1) / tiles));
  const int chunk = (red / 32 + splits - 1) / splits * 32;
  splits = (red + chunk - 1) / chunk;
  skinny_gemm_kernel<TA, TR, MODE><<<dim3(tiles, splits), 256, 0, st>>>(
      A, lda, rows, red, chunk, Bm, ldb, ncols, outf, outb, ldo);
  return cudaGetLastError();
}

struct SvdScratch {
  uint16_t* E;
  float *Y, *Z, *S, *Om, *Rinv, *MA, *MB, *sig;
  double* G;
  int* status;
};

// Y (rows x lp, l live columns) <- a basis of its columns by CholeskyQR: Y R^-1 with
// R^T R = Y^T Y.  One pass leaves the basis orthonormal up to about eps cond(Y)^2, which
// is all the subspace iteration needs between products; the basis the projection uses
// takes a second pass, which restores orthogonality to rounding level.  Each pass
// writes the spare buffer and swaps it with Y (all three tall buffers have one size).
cudaError_t orthonormalise(float*& Y, int rows, int l, int lp, int passes, SvdScratch& s,
                           int sms, cudaStream_t st) {
  const int grid = std::max(1, std::min(sms, (rows + 31) / 32));
  const int rpc = ((rows + grid - 1) / grid + 31) / 32 * 32;
  const int gsmem = l * l * static_cast<int>(sizeof(double));
  const int csmem = l * (l + 1) * static_cast<int>(sizeof(double));
  for (int pass = 0; pass < passes; ++pass) {
    cudaError_t e = cudaMemsetAsync(s.G, 0, static_cast<size_t>(l) * l * sizeof(double), st);
    if (e != cudaSuccess) return e;
    gram_kernel<<<(rows + rpc - 1) / rpc, 1024, gsmem, st>>>(Y, lp, rows, l, rpc, s.G);
    chol_inv_kernel<<<1, 1024, csmem, st>>>(s.G, l, s.Rinv, lp);
    e = launch_skinny<float, false, 1>(Y, lp, rows, lp, s.Rinv, lp, lp, s.S, nullptr, lp, sms, st);
    if (e != cudaSuccess) return e;
    std::swap(Y, s.S);
  }
  return cudaSuccess;
}

int svd_kernel_attributes(int dev) {
  static std::atomic<bool> set[64];  // zero-initialised: false
  if (dev < 0 || dev >= 64) return SALR_ERR_UNSUPPORTED;
  if (set[dev]) return SALR_OK;
  const int big = kSvdMaxL * (kSvdMaxL + 1) * static_cast<int>(sizeof(double));
  SALR_TRY(cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSvdMaxL * kSvdMaxL * static_cast<int>(sizeof(double))));
  SALR_TRY(cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
  SALR_TRY(cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
  set[dev] = true;
  return SALR_OK;
}

}  // namespace

extern "C" {

int salr_residual_adapter(const void* W, salr_handle h, int64_t r, const void* omega, int64_t l,
                          int q, void* A_out, void* B_out, void* sigma_out, void* stream) {
  if (!valid_handle(h) || !W || !omega || !A_out || !B_out) return SALR_ERR_INVALID;
  if (r < 1 || l < r || l > kSvdMaxL || l > h->N || l > h->K || q < 0 || q > 16)
    return SALR_ERR_INVALID;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(omega) & 3u) ||
      (reinterpret_cast<uintptr_t>(A_out) & 1u) || (reinterpret_cast<uintptr_t>(B_out) & 1u) ||
      (reinterpret_cast<uintptr_t>(sigma_out) & 3u))
    return SALR_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = static_cast<int>(h->N), K = static_cast<int>(h->K);
  const int L = static_cast<int>(l), R = static_cast<int>(r);
  const int LP = (L + 31) / 32 * 32;
  const int sms = device_sms(h->device);
  const int attr = svd_kernel_attributes(h->device);
  if (attr != SALR_OK) return attr;

  // scratch, one stream-ordered allocation
  const size_t e_bytes = round256(static_cast<size_t>(N) * K * sizeof(uint16_t));
  const size_t y_bytes = round256(static_cast<size_t>(N) * LP * sizeof(float));
  const size_t z_bytes = round256(static_cast<size_t>(K) * LP * sizeof(float));
  const size_t s_bytes = std::max(y_bytes, z_bytes);
  const size_t m_bytes = round256(static_cast<size_t>(LP) * LP * sizeof(float));
  const size_t d_bytes = round256(static_cast<size_t>(L) * L * sizeof(double));
  const size_t sig_bytes = round256(static_cast<size_t>(LP) * sizeof(float));
  const size_t f32_bytes = 3 * s_bytes + z_bytes + 3 * m_bytes + sig_bytes;
  const size_t total = e_bytes + f32_bytes + d_bytes + 256;
  uint8_t* mem = nullptr;
  cudaError_t e = dev_alloc_async(reinterpret_cast<void**>(&mem), total, st);
  if (e != cudaSuccess) return cuda_status(e);
  SvdScratch sc;
  uint8_t* p = mem;
  sc.E = reinterpret_cast<uint16_t*>(p);
  p += e_bytes;
  uint8_t* f32 = p;
  sc.Y = reinterpret_cast<float*>(p);
  p += s_bytes;
  sc.Z = reinterpret_cast<float*>(p);
  p += s_bytes;
  sc.Om = reinterpret_cast<float*>(p);
  p += z_bytes;
  sc.S = reinterpret_cast<float*>(p);
  p += s_bytes;
  sc.Rinv = reinterpret_cast<float*>(p);
  p += m_bytes;
  sc.MA = reinterpret_cast<float*>(p);
  p += m_bytes;
  sc.MB = reinterpret_cast<float*>(p);
  p += m_bytes;
  sc.sig = reinterpret_cast<float*>(p);
  p += sig_bytes;
  sc.G = reinterpret_cast<double*>(p);
  p += d_bytes;
  sc.status = reinterpret_cast<int*>(p);

  auto run = [&]() -> cudaError_t {
    cudaError_t err;
    // every fp32 buffer starts at zero: padding columns stay zero throughout
    if ((err = cudaMemsetAsync(f32, 0, f32_bytes, st)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(sc.status, 0, sizeof(int), st)) != cudaSuccess) return err;
    if ((err = cudaMemcpy2DAsync(sc.Om, LP * sizeof(float), omega, L * sizeof(float),
                                 L * sizeof(float), K, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
      return err;
    residual_kernel<<<static_cast<unsigned>(h->nblocks), kBlockRows, 0, st>>>(
        static_cast<const uint16_t*>(W), h->blob, h->offsets, K, sc.E);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // Y = E Omega, Q = orth(Y)
    if ((err = launch_skinny<uint16_t, false, 0>(sc.E, K, N, K, sc.Om, LP, L, sc.Y, nullptr, LP,
                                                 sms, st)) != cudaSuccess)
      return err;
    if ((err = orthonormalise(sc.Y, N, L, LP, q > 0 ? 1 : 2, sc, sms, st)) != cudaSuccess)
      return err;
    for (int it = 0; it < q; ++it) {
      if ((err = cudaMemsetAsync(sc.Z, 0, s_bytes, st)) != cudaSuccess) return err;
      if ((err = launch_skinny<uint16_t, true, 0>(sc.E, K, K, N, sc.Y, LP, L, sc.Z, nullptr, LP,
                                                  sms, st)) != cudaSuccess)
        return err;
      if ((err = orthonormalise(sc.Z, K, L, LP, 1, sc, sms, st)) != cudaSuccess) return err;
      if ((err = cudaMemsetAsync(sc.Y, 0, s_bytes, st)) != cudaSuccess) return err;
      if ((err = launch_skinny<uint16_t, false, 0>(sc.E, K, N, K, sc.Z, LP, L, sc.Y, nullptr, LP,
                                                   sms, st)) != cudaSuccess)
        return err;
      if ((err = orthonormalise(sc.Y, N, L, LP, it + 1 == q ? 2 : 1, sc, sms, st)) !=
          cudaSuccess)
        return err;
    }
    // Z = E^T Q = B^T; Z^T Z = B B^T, diagonalised on one CTA
    if ((err = cudaMemsetAsync(sc.Z, 0, s_bytes, st)) != cudaSuccess) return err;
    if ((err = launch_skinny<uint16_t, true, 0>(sc.E, K, K, N, sc.Y, LP, L, sc.Z, nullptr, LP,
                                                sms, st)) != cudaSuccess)
      return err;
    if ((err = cudaMemsetAsync(sc.G, 0, static_cast<size_t>(L) * L * sizeof(double), st)) !=
        cudaSuccess)
      return err;
    {
      const int grid = std::max(1, std::min(sms, (K + 31) / 32));
      const int rpc = ((K + grid - 1) / grid + 31) / 32 * 32;
      gram_kernel<<<(K + rpc - 1) / rpc, 1024, L * L * static_cast<int>(sizeof(double)), st>>>(
          sc.Z, LP, K, L, rpc, sc.G);
    }
    jacobi_eig_kernel<<<1, 1024, 2 * L * (L | 1) * static_cast<int>(sizeof(float)), st>>>(
        sc.G, L, R, sc.MA, sc.MB, LP, sc.sig, sc.status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // A' = Z U_r S_r^(-1/2) (K x r), B' = (Q U_r S_r^(1/2))^T (r x N)
    if ((err = launch_skinny<float, false, 2>(sc.Z, LP, K, LP, sc.MA, LP, R, nullptr,
                                              static_cast<uint16_t*>(A_out), R, sms, st)) !=
        cudaSuccess)
      return err;
    if ((err = launch_skinny<float, false, 3>(sc.Y, LP, N, LP, sc.MB, LP, R, nullptr,
                                              static_cast<uint16_t*>(B_out), N, sms, st)) !=
        cudaSuccess)
      return err;
    if (sigma_out &&
        (err = cudaMemcpyAsync(sigma_out, sc.sig, R * sizeof(float), cudaMemcpyDeviceToDevice,
                               st)) != cudaSuccess)
      return err;
    return cudaSuccess;
  };
  e = run();
  int status = 0;
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(&status, sc.status, sizeof(int), cudaMemcpyDeviceToHost, st);
  cudaFreeAsync(mem, st);
  const cudaError_t es = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e);
  if (es != cudaSuccess) return cuda_status(es);
  if (status & DEV_ERR_TIMEOUT) return SALR_ERR_TIMEOUT;
  return SALR_OK;
}

int salr_sync_status(salr_handle h, void* stream) {
  if (!valid_handle(h)) return SALR_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int status = 0;
  SALR_TRY(cudaStreamSynchronize(st));
  SALR_TRY(cudaMemcpy(&status, h->status, sizeof(int), cudaMemcpyDeviceToHost));
  SALR_TRY(cudaMemset(h->status, 0, sizeof(int)));
  if (status == 0) return SALR_OK;
  // a kernel that gave up may have left partial sums behind: start the next call clean
  if (h->work.ws) SALR_TRY(cudaMemset(h->work.ws, 0, h->work.ws_elems * sizeof(float)));
  if (h->work.counters)
    SALR_TRY(cudaMemset(h->work.counters, 0, h->work.n_counters * sizeof(uint32_t)));
  if (h->tscr.T32) {
    SALR_TRY(cudaMemset(h->tscr.T32, 0, static_cast<size_t>(h->tscr.rows) * 128 * sizeof(float)));
    SALR_TRY(cudaMemset(h->tscr.counters, 0, static_cast<size_t>(h->tscr.rows / 128) * 4 * sizeof(uint32_t)));
  }
  if (h->sscr.acc) {
    SALR_TRY(cudaMemset(h->sscr.acc, 0, static_cast<size_t>(h->N) * 64 * sizeof(float)));
    SALR_TRY(cudaMemset(h->sscr.counters, 0, static_cast<size_t>(h->N / 128) * 4 * sizeof(uint32_t)));
    SALR_TRY(cudaMemset(h->sscr.tacc, 0, kTBuf * sizeof(float)));
    SALR_TRY(cudaMemset(h->sscr.tflags, 0, 2 * sizeof(uint32_t)));
  }
  const int nrc = noalloc_reset(h->device);
  if (nrc != SALR_OK) return nrc;
  if (status & DEV_ERR_TIMEOUT) return SALR_ERR_TIMEOUT;
  // a NaN, or (in the bounds-checked build) an offset or size out of range
  if (status & (DEV_ERR_NAN | DEV_ERR_RANGE | DEV_ERR_FORMAT)) return SALR_ERR_INVALID;
  return SALR_ERR_UNSUPPORTED;
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// salr_linear_noalloc: the small-M layer with its scratch in a fixed device array.
//
// Some callers cannot let a library allocate device memory on their behalf: serving
// loops that pre-plan every byte of device memory and forbid allocations once running
// (an allocation can fail under memory pressure or stall the device while it is made),
// and embedders whose own allocator owns the GPU.  For them the scratch the small-M
// kernel needs lives in one file-scope array, allocated when the library's device code
// is loaded and held by every GPU that loads it until the process exits.
// ------------------------------------------------------------------------------------
namespace {

constexpr int64_t kNoAllocMaxM = 16;     // tokens per call
constexpr int64_t kNoAllocMaxN = 32768;  // output features
// layout: [t counts: 2 u32][t accumulator: 16 x 128 f32]
//         [split-tile arrival counts: N/128 x 4 u32][split-tile sums: N x 16 f32]
// Nothing in it scales with the SM count: the kernel keeps every per-CTA quantity in
// shared memory.
constexpr int kNaTBuf = 16 * 128;
constexpr size_t kNaFlags = 0;
constexpr size_t kNaTacc = 256;
constexpr size_t kNaCounters = kNaTacc + kNaTBuf * sizeof(float);
constexpr size_t kNaAcc = kNaCounters + (kNoAllocMaxN / 128) * 4 * sizeof(uint32_t);
constexpr size_t kNaBytes = kNaAcc + static_cast<size_t>(kNoAllocMaxN) * 16 * sizeof(float);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

std::mutex g_na_mu;
unsigned char* g_na_ptr[64] = {nullptr};

// Device address of the scratch array for the current device (looked up, and cleared on
// the caller's stream, once per device).  Every call leaves the array zero again on the
// device, so nothing about a call is kept on the host.
int noalloc_scratch(int dev, cudaStream_t st, unsigned char** out) {
  if (dev < 0 || dev >= 64) return SALR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_na_mu);
  if (!g_na_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return SALR_ERR_CUDA;
    SALR_TRY(cudaMemsetAsync(p, 0, kNaBytes, st));
    g_na_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_na_ptr[dev];
  return SALR_OK;
}

}  // namespace

// After a call that gave up, clear the shared array of the device (if it is in use) so
// that the next call starts clean.
int noalloc_reset(int dev) {
  if (dev < 0 || dev >= 64) return SALR_OK;
  std::lock_guard<std::mutex> g(g_na_mu);
  if (!g_na_ptr[dev]) return SALR_OK;
  int cur = 0;
  SALR_TRY(cudaGetDevice(&cur));
  if (cur != dev) SALR_TRY(cudaSetDevice(dev));
  const cudaError_t e = cudaMemset(g_na_ptr[dev], 0, kNaBytes);
  if (cur != dev) cudaSetDevice(cur);
  return cuda_status(e);
}

extern "C" int salr_linear_noalloc(const void* X, int64_t M, salr_handle h, const void* A_cat,
                                   const void* B_cat, int64_t R, void* Y, void* stream) {
  int rc = check_linear_args(X, M, h, A_cat, B_cat, R, Y);
  if (rc != SALR_OK) return rc;
  if (M > kNoAllocMaxM || h->N > kNoAllocMaxN) return SALR_ERR_UNSUPPORTED;
  int dev = 0;
  SALR_TRY(cudaGetDevice(&dev));
  if (dev != h->device) return SALR_ERR_INVALID;
  unsigned char* scr = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = noalloc_scratch(dev, st, &scr);
  if (rc != SALR_OK) return rc;
  StreamParams sp{};
  sp.blob = h->blob;
  sp.offsets = h->offsets;
  sp.Y = static_cast<uint16_t*>(Y);
  bind_call(sp, reinterpret_cast<float*>(scr + kNaAcc),
            reinterpret_cast<uint32_t*>(scr + kNaCounters), reinterpret_cast<float*>(scr + kNaTacc),
            reinterpret_cast<uint32_t*>(scr + kNaFlags));
  sp.status = h->status;
  sp.N = static_cast<int>(h->N);
  sp.K = static_cast<int>(h->K);
  sp.M = static_cast<int>(M);
  sp.R = static_cast<int>(R);
  sp.R16 = static_cast<int>((R + 15) / 16 * 16);
  sp.kblocks = static_cast<int>(h->K / 64);
  sp.RT = static_cast<int>(h->N / 128);
  sp.units = sp.RT * sp.kblocks;
  sp.bpc = stream_blocks_per_copy(h->max16);
  sp.cbuf = static_cast<int>((sp.bpc * h->max16 * 16 + 32 + 1023) / 1024 * 1024);
  sp.X = static_cast<const uint16_t*>(X);
  CUtensorMap tx, ta, tb;
  std::memset(&ta, 0, sizeof(ta));
  std::memset(&tb, 0, sizeof(tb));
  if (!make_map(&tx, X, h->K, M, 64, 16)) return SALR_ERR_CUDA;
  if (R > 0) {
    if (!make_map(&ta, A_cat, R, h->K, 64, 64)) return SALR_ERR_CUDA;
    if (!make_map(&tb, B_cat, h->N, R, 64, sp.R16)) return SALR_ERR_CUDA;
  }
  return launch_stream<16>(sp, tx, ta, tb, device_sms(h->device), st);
}
