/*
 * salr.h - C ABI of the SALR sparse + low-rank inference linear layer for NVIDIA B200.
 *
 * The layer (SALR, "Sparsity-Aware Low-Rank Representation for Efficient Fine-Tuning of
 * Large Language Models"; the authors' abstract and the gist.science technical summary):
 *
 *     Y = X (M (.) W)^T + X A_cat B_cat
 *
 * W (N x K, out x in) is the frozen base weight, statically magnitude-pruned per row
 * (technical summary, Methodology 1) and stored as a bitmap plus a compact array of the
 * kept values with a per-block offset table (Methodology 4, "Bitmap Encoding" and the
 * lookup table read by "Stage 1").  A_cat (K x R) and B_cat (R x N) are the low-rank
 * adapters (task LoRAs and the truncated-SVD residual adapter) stacked along rank into
 * one GEMM on the shared input (Methodology 3).  salr_linear runs the two-stage
 * pipeline of Methodology 4: bitmap blocks are expanded on CUDA cores while tensor cores
 * consume the previously expanded blocks.
 *
 * Conventions for every entry point
 *   - Matrices are row-major; bf16 is passed as its 16-bit pattern (uint16).
 *   - "device" pointers are CUDA device memory of the device current at the call;
 *     "host" pointers are page-locked host memory (cudaHostAlloc / cudaHostRegister).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  All
 *     calls are stream-ordered unless stated otherwise.
 *   - Every call returns a salr_status.  Argument errors are detected on the host before
 *     any work is queued; nothing is written in that case.
 *   - Handles and the scratch of salr_encode, salr_load and salr_residual_adapter take
 *     device memory from a stream-ordered pool the library owns on each device; memory
 *     given back to it stays reserved for reuse, up to 1 GiB per device.
 *   - The library never traps or spins without a bound on the GPU.  Errors found on the
 *     device (a NaN in W, a pipeline wait that ran out of time) are recorded in the
 *     handle's status word; salr_encode reports them itself, salr_sync_status reads them.
 *   - Bounds-checked build: compiled with -DSALR_CHECKS (python -m
 *     sparse_rank_linear_b200.build --checks gives libsalr_checks.so, which the Python
 *     binding loads when SALR_LIBRARY names it), every shared- or global-memory offset
 *     the kernels derive from the data (block offsets and sizes, value positions, tile
 *     rows, ring indices) is checked before use; a failed check skips the access and
 *     sets a range bit that salr_sync_status reports as SALR_ERR_INVALID.
 *   - Environment, read at each call: SALR_WAIT_LIMIT_CYCLES=n bounds every device wait
 *     at n SM cycles (default 2e9, about one second; failure tests lower it);
 *     SALR_FAIL_T_WAIT=1 makes the small-M kernel's readers of t wait for one part more
 *     than is ever added (failure tests only: the call then reports SALR_ERR_TIMEOUT);
 *     SALR_WIDE_MIN_ROUNDS=n sets how many full rounds of 256-row tiles the dense-scratch
 *     path needs before it uses them (default 8; tests set 0 to reach them on small
 *     shapes); SALR_TILE_GROUP_ROWS=n sets the prefill kernel's tile group (tests);
 *     SALR_STREAM_SKEW=S (0 .. 192, default 0) makes the small-M kernel's CTA ranges
 *     shrink with the CTA index; SALR_COOPERATIVE=1 launches the small-M kernel
 *     cooperatively instead of with programmatic stream serialization; SALR_FAKE_OOM=1
 *     makes allocations fail.
 *
 * Shape rules (v1): N % 128 == 0, 128 <= N <= 2^22, K % 64 == 0, 64 <= K <= 32768,
 * R % 8 == 0, R <= 128, 1 <= M <= 2^24, at most 2^27 output tiles of 128 x 128
 * ((N / 128) * ceil(M / 128)), all pointers 16-byte aligned.
 */
#ifndef SALR_H_
#define SALR_H_

#include <stdint.h>

#if defined(__GNUC__)
#define SALR_API __attribute__((visibility("default")))
#else
#define SALR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct salr_weight_s* salr_handle; /* opaque; owns its device buffers */

typedef enum {
  SALR_OK = 0,
  SALR_ERR_INVALID = 1,     /* bad argument, bad handle, NaN in W, bad sparsity      */
  SALR_ERR_UNSUPPORTED = 2, /* shape or alignment outside the v1 rules above         */
  SALR_ERR_CUDA = 3,        /* a CUDA runtime/driver call or a launch failed         */
  SALR_ERR_OOM = 4,         /* a device or host allocation failed                    */
  SALR_ERR_TIMEOUT = 5      /* a bounded wait inside a kernel gave up                */
} salr_status;

/*
 * salr_encode - prune W by magnitude and store it in the bitmap block format.
 *
 * Defined by: technical summary, Methodology 1 (static magnitude mask on the frozen base,
 * adapters stay dense) and Methodology 4 (bitmap + compact values + lookup table).
 *
 * W        device, N x K bf16, read only; may be freed once the call returns.
 * sparsity fraction pruned per row, 0 <= sparsity < 1.  Each row keeps
 *          keep = K - floor(sparsity * K) entries: those of largest |w|, and among equal
 *          |w| those of lowest column index.  |+0| = |-0|; +-Inf rank highest; a NaN
 *          makes the call fail with SALR_ERR_INVALID.
 * out      receives a new handle on SALR_OK (unchanged otherwise).
 *
 * Synchronises `stream` once (to size the value array and to read the NaN check).
 *
 * Encoded format (also readable through salr_format_view): W is cut into blocks of
 * 128 rows x 64 columns; block b = i * (K/64) + j covers rows 128i..128i+127 and
 * columns 64j..64j+63 and starts at byte 16 * offsets[b] of the blob.  A block holds
 * 128 little-endian uint64 words (word r: bit c set when W[128i+r, 64j+c] is kept),
 * then the kept values as bf16 (a kept -0 stays -0), then zero bytes up to a multiple
 * of 16.  Within a block the values are ordered by row quarter (block rows 32q..32q+31),
 * then by 4-column group (block columns 4n..4n+3), then by row, then by column: a warp
 * rebuilding one quarter, one row per thread, then finds each group's values of its 32
 * rows side by side.  offsets has nblocks + 1 uint32 entries; the last is the blob size
 * in 16-byte units.
 */
SALR_API int salr_encode(const void* W, int64_t N, int64_t K, float sparsity, void* stream,
                salr_handle* out);

/*
 * salr_decode - expand an encoded weight back to dense M (.) W, for checking.
 *
 * W_out device, N x K bf16, caller-allocated, fully overwritten; pruned entries are
 *       +0.0 (0x0000), kept entries bit-identical to W.
 */
SALR_API int salr_decode(salr_handle h, void* W_out, void* stream);

/*
 * salr_linear - Y = X (M (.) W)^T + (X A_cat) B_cat.
 *
 * Defined by: technical summary, Methodology 3 (one concatenated adapter GEMM on the
 * shared input) and Methodology 4 (two-stage pipelined bitmap decoding + tensor-core
 * GEMM).
 *
 * X     device, M x K bf16.
 * M     number of tokens, >= 1.
 * A_cat device, K x R bf16; B_cat device, R x N bf16.  R == 0 means no adapter; the
 *       pointers are then ignored and may be NULL.
 * Y     device, M x N bf16, overwritten (no accumulation into Y).
 *
 * Arithmetic: products of bf16 inputs accumulate in fp32 on the tensor cores.  The
 * adapter's inner product t = X A_cat is accumulated in fp32 and rounded once to bf16
 * before it multiplies B_cat.  The order of the fp32 sums is not fixed (split K, and
 * for M <= 64 partial sums of a row tile are added in L2 in arrival order), so results
 * are not bitwise reproducible from call to call, but always satisfy ||Y - Y*||_F <= 4e-3 ||Y*||_F and |Y - Y*| <= 1e-2 * sum|products| against the
 * exact result Y*.
 *
 * The handle holds the split-K workspace used by this call; it is grown on demand
 * (a cudaMalloc) and is not safe to share between calls running concurrently on
 * different streams.  For M > 64 it holds one fp32 sum of 128 rows x 128 or 256 tokens
 * per output tile that the layer kernel splits along K.  Those are the tiles of its
 * last, partial round over the SMs, or every tile when there are fewer tiles than SMs.
 *
 * Kernels: for M <= 64 one persistent kernel.  For larger M, a t = X A_cat kernel (when
 * R > 0) and a persistent layer kernel that may start while t still runs.  From M > 256
 * on, the weight is first expanded once to a dense bf16 scratch of N x K x 2 bytes, taken
 * from the library's pool on `stream` and given back to it in stream order at the end
 * of the call; the layer kernel then reads dense weight tiles instead of decoding them
 * once per 256 tokens.
 *
 * For M <= 64 the call may start while the previous kernel on `stream` is still
 * running (programmatic dependent launch): before that kernel has completed it reads
 * only the handle's encoded weight; X, A_cat, B_cat, the scratch and Y are touched
 * afterwards.  Whatever writes the encoded weight (salr_encode) must therefore have
 * completed, or be ordered on the stream before the previous kernel.
 */
SALR_API int salr_linear(const void* X, int64_t M, salr_handle h, const void* A_cat,
                const void* B_cat, int64_t R, void* Y, void* stream);

/*
 * salr_linear_host - salr_linear with the activations in host memory.
 *
 * X_host (M x K bf16) and Y_host (M x N bf16) are page-locked host buffers; A_cat and
 * B_cat are device buffers as for salr_linear (adapters are weights and stay resident).
 * Queues the host-to-device copy of X, the layer and the device-to-host copy of Y on
 * `stream` through staging buffers owned by the handle; Y_host is valid once the
 * stream has been synchronised.
 */
SALR_API int salr_linear_host(const void* X_host, int64_t M, salr_handle h, const void* A_cat,
                     const void* B_cat, int64_t R, void* Y_host, void* stream);

/*
 * salr_linear_noalloc - salr_linear for callers that cannot have the library allocate.
 *
 * No counterpart in the SALR paper: this is an interface variant of this library, not
 * part of the method.  It computes the same layer as salr_linear (same arguments, same
 * arithmetic and tolerance) for M <= 16 and N <= 32768, and never allocates device
 * memory: the scratch it needs (fp32 partial sums and their arrival counts, the fp32
 * t = X A_cat accumulator and its counts, about 2 MiB) is one fixed array in the
 * library's device code, present on every GPU that loads the library until the process
 * exits.  Meant for
 * callers whose device memory is planned up front and who may not allocate during
 * inference (a failing or stalling cudaMalloc is not acceptable there).  The handle and
 * all inputs and outputs are still the caller's.
 *
 * Returns SALR_ERR_UNSUPPORTED for M > 16 or N > 32768.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) and clears the array on
 * `stream`.  Each call then leaves the array ready for the next one; after a call that
 * gave up (salr_sync_status reports it) the array is cleared again.  All calls
 * on one device share the one array, so calls whose executions overlap on the GPU
 * (different streams, or different threads) race and give wrong results: order them on
 * one stream.
 */
SALR_API int salr_linear_noalloc(const void* X, int64_t M, salr_handle h, const void* A_cat,
                                 const void* B_cat, int64_t R, void* Y, void* stream);

/*
 * salr_linear_plan - how salr_linear runs a call, without running it.
 *
 * No counterpart in the SALR paper: a planning query of this library.  It reports the
 * kernels, tiles and work split salr_linear chooses for M tokens and R adapter ranks on
 * an N x K weight.  It also reports the device memory that call needs beyond its
 * arguments: the transient dense weight scratch and the fp32 split sums held in the
 * handle's workspace.
 *
 * N, K   the weight's shape, with the rules of salr_encode.
 * M, R   as for salr_linear.
 * sms    the device's SM count (> 0).  With 0, the current CUDA device's count is used.
 * out    filled on success.
 *
 * Host logic only: nothing is allocated or launched, so with sms > 0 it needs no GPU.
 * Returns SALR_ERR_INVALID for a NULL `out`, M < 1, R < 0 or sms < 0.  Returns
 * SALR_ERR_UNSUPPORTED for shapes, M or R that salr_linear rejects, and SALR_ERR_CUDA
 * when sms == 0 and there is no device.
 */
typedef struct {
  int32_t path;        /* 0: one persistent kernel (M <= 64); 1: t kernel + fused decode and
                          GEMM; 2: weight expansion + t kernel + GEMM on dense weight tiles */
  int32_t kernels;     /* kernel launches per call */
  int32_t token_tile;  /* tokens per MMA tile: 16, 32, 64, 128 or 256 */
  int32_t tile_rows;   /* weight rows per output tile: 128, or 256 on path 2 when
                          N % 256 == 0 (two MMAs share each X tile) */
  int32_t grid;        /* CTAs of the layer kernel, at most one per SM */
  int32_t units;       /* work units of the layer kernel: 128 x 64 weight blocks (path 0),
                          else whole tiles plus the K parts of split tiles */
  int32_t tiles;       /* output tiles of tile_rows weight rows x token_tile (paths 1, 2) */
  int32_t whole_tiles; /* tiles computed whole (paths 1, 2) */
  int32_t splits;      /* K parts of each remaining tile (paths 1, 2; 1 = none) */
  int64_t split_sum_bytes;     /* fp32 sums of the split tiles in the handle's workspace */
  int64_t dense_scratch_bytes; /* transient dense bf16 weight (path 2), else 0 */
  int32_t group_rows;  /* paths 1, 2: 0 when the output tiles go token tile first; else
                          they go in groups of this many row tiles, token tile by token
                          tile (when X outgrows about half the L2) */
} salr_plan;
SALR_API int salr_linear_plan(int64_t N, int64_t K, int64_t M, int64_t R, int32_t sms,
                              salr_plan* out);

/* salr_free - release a handle and every device buffer it owns.  Freeing an unknown or
 * already freed handle returns SALR_ERR_INVALID and touches nothing. */
SALR_API int salr_free(salr_handle h);

/* salr_info - shape and size of an encoded weight.  Any output pointer may be NULL.
 * nnz = number of kept entries; bytes = blob bytes + offset-table bytes. */
SALR_API int salr_info(salr_handle h, int64_t* N, int64_t* K, int64_t* nnz, int64_t* bytes);

/* salr_format_view - read-only device pointers to the encoded format described under
 * salr_encode (blob and offset table), owned by the handle. */
SALR_API int salr_format_view(salr_handle h, const void** blob, int64_t* blob_bytes,
                     const void** offsets, int64_t* n_offsets);

/*
 * Serialised image: the byte form of an encoded weight, for storing the compressed model
 * (technical summary, Methodology 4: bitmap encoding is what makes the size reduction
 * real, and Experimental Results: model size halved).  The image is the encoded format
 * above behind a fixed header; all fields little-endian:
 *
 *   bytes [0, 64)   header
 *                     0  char[8] "SALRBLK1"       32  int64 keep (entries kept per row)
 *                     8  uint32 version = 2       40  int64 nnz = N * keep
 *                    12  uint32 header size = 64  48  float32 sparsity
 *                    16  int64 N                  52  uint32 0
 *                    24  int64 K                  56  int64 blob bytes (multiple of 16)
 *   then            offset table, (N/128)(K/64) + 1 uint32, zero bytes up to a multiple
 *                   of 16
 *   then            the blob, byte for byte
 *
 * The image holds no device addresses and no state of earlier calls: any GPU can load
 * it.  It carries no checksum; salr_load checks its structure instead (below).
 */

/* salr_save_size - size in bytes of the image salr_save writes for `h`. */
SALR_API int salr_save_size(salr_handle h, int64_t* bytes);

/*
 * salr_save - write the image of `h` to host memory.
 *
 * buf       host memory (page-locked or pageable), at least salr_save_size bytes; only
 *           the first salr_save_size bytes are written.
 * stream    the copies of the offset table and the blob are queued on it after work
 *           already queued there (so after the salr_encode that made `h`), and the call
 *           returns once they are complete.
 * Returns SALR_ERR_INVALID for an unknown handle, a NULL buf or buf_bytes too small
 * (nothing is written then).
 */
SALR_API int salr_save(salr_handle h, void* buf, int64_t buf_bytes, void* stream);

/*
 * salr_load - make a new handle on the current device from an image in host memory.
 *
 * buf       host memory holding an image; bytes past the image's end are ignored.
 * out       receives the new handle on SALR_OK (unchanged otherwise).  The handle is the
 *           one salr_encode gave for the same weight: salr_decode, salr_linear and the
 *           rest behave the same way on it.
 *
 * Checks before anything is used: the header (magic, version, N and K under the shape
 * rules, keep = K - floor(sparsity * K), nnz = N * keep), the offset table on the host
 * (starts at 0, each block at least its 1 KB bitmap and at most a dense block, ends at
 * the blob size), then on the device every block (its bitmap's population matches its
 * size, no kept value is NaN, padding is zero) and every row (exactly `keep` bits set).
 * A failed check returns SALR_ERR_INVALID (SALR_ERR_UNSUPPORTED for a shape outside the
 * rules) and frees everything the call allocated.  Synchronises `stream`.
 */
SALR_API int salr_load(const void* buf, int64_t buf_bytes, void* stream, salr_handle* out);

/*
 * salr_residual_adapter - the rank-r adapter of what pruning removed from W0.
 *
 * Defined by: technical summary, Methodology 2 ("Residual Decomposition": E = W - W_hat,
 * its rank-r truncated SVD E_r kept as a low-rank adapter; "Theoretical Guarantee": the
 * per-entry error then shrinks by 1 - r/min(d, k)).  Computed by a randomized range
 * finder with subspace iteration and a direct SVD of the projected matrix (Halko,
 * Martinsson and Tropp, SIAM Review 2011): the pages fix the result, not the route.
 *
 * W       device, N x K bf16: the dense frozen base that `h` was encoded from.  E is W
 *         where the handle's mask drops an entry and 0 where it keeps one (exact).
 * r       adapter rank, 1 <= r <= l.
 * omega   device, K x l fp32 row-major: the random test matrix (drawn by the caller,
 *         e.g. standard normal; only the space its columns span matters).  Read only.
 * l       columns of omega, r <= l <= min(160, N, K); l - r is the oversampling.
 * q       subspace iterations, 0 <= q <= 16 (each multiplies by E^T and E once more).
 * A_out   device, K x r bf16 (row-major), B_out device, r x N bf16 (row-major): the
 *         adapter in the X A B orientation, A' = V_r S_r^(1/2) and B' = S_r^(1/2) U_r^T,
 *         so that A' B' approximates E_r^T and X A' B' approximates X E_r^T.  Directions
 *         whose singular value is at or below 1e-6 of the largest get zero columns/rows.
 * sigma_out  device, r fp32, or NULL: the estimated singular values, descending.
 *
 * Arithmetic: E times the tall bases in fp32 on CUDA cores; Gram matrices in fp64;
 * orthonormal bases by CholeskyQR twice; the small symmetric eigenproblem by cyclic
 * Jacobi in fp64.  Scratch (about 2 N K + 4 (N + 3 K) l' bytes, l' = l rounded up to 32)
 * comes from the stream-ordered allocator and is released before the call returns.
 * Synchronises `stream`.  SALR_ERR_TIMEOUT if the Jacobi iteration hit its sweep bound.
 */
SALR_API int salr_residual_adapter(const void* W, salr_handle h, int64_t r, const void* omega,
                                   int64_t l, int q, void* A_out, void* B_out, void* sigma_out,
                                   void* stream);

/* salr_sync_status - synchronise `stream`, return the first device-side error recorded
 * for this handle since the last call (SALR_OK if none) and clear it. */
SALR_API int salr_sync_status(salr_handle h, void* stream);

/* salr_status_string - static, human-readable name of a status code. */
SALR_API const char* salr_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SALR_H_ */
