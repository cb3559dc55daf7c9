// salr_svd.cuh - GPU builder of the residual adapter: the rank-r truncated SVD of the
// part of W0 that pruning removed.
//
// The method (SALR technical summary, Methodology 2, "Residual Decomposition" and
// "Theoretical Guarantee"): E = W0 - W_hat, E_r its rank-r truncated SVD, added back as
// a low-rank adapter; the per-entry error then shrinks by (1 - r/min(d, k)).  The pages
// fix the result only.  It is reached here by a randomized range finder with subspace
// (power) iteration and a direct SVD of the small projected matrix (Halko, Martinsson
// and Tropp, "Finding structure with randomness", SIAM Review 2011):
//
//   Y = E Omega, Q = orth(Y); q times: Q = orth(E orth(E^T Q)); Z = E^T Q (= B^T);
//   Z^T Z = U_b L U_b^T (so B = U_b S V^T with S = L^(1/2), V = Z U_b S^-1);
//   A' = V_r S_r^(1/2) = Z U_b,r S_r^(-1/2) (K x r),  B'^T = Q U_b,r S_r^(1/2) (N x r).
//
// Kernels: the residual E (bf16, exact), skinny products of E or E^T with a tall fp32
// matrix (CUDA-core fp32 FMA, split over the long dimension), fp64 Gram matrices,
// CholeskyQR (twice per orthonormalisation, columns that turn out dependent set to
// zero), and one-CTA cyclic Jacobi on the small Gram matrix.  All loops are bounded;
// no kernel waits on another.
#pragma once
#include <cstdint>
#include "salr_codec.cuh"

namespace salr {

constexpr int kSvdMaxL = 160;  // columns of the random test matrix (r + oversampling)
constexpr int kSvdMaxSweeps = 40;

// E[n, k] = W[n, k] where the mask drops it, +0 where it keeps it.  One CTA of 128
// threads per 128 x 64 block; thread r handles row r of the block.
__global__ void __launch_bounds__(kBlockRows) residual_kernel(const uint16_t* __restrict__ W,
                                                              const uint8_t* __restrict__ blob,
                                                              const uint32_t* __restrict__ offsets,
                                                              int K, uint16_t* __restrict__ E) {
  const int b = blockIdx.x, nwords = K / 64;
  const int i = b / nwords, j = b % nwords, r = threadIdx.x;
  const uint64_t word =
      reinterpret_cast<const uint64_t*>(blob + static_cast<size_t>(offsets[b]) * 16)[r];
  const size_t base = static_cast<size_t>(i * kBlockRows + r) * K + j * kBlockCols;
  const uint4* src = reinterpret_cast<const uint4*>(W + base);
  uint4* dst = reinterpret_cast<uint4*>(E + base);
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    uint4 v = src[c8];
    uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t m = static_cast<uint32_t>(word >> (8 * c8 + 2 * e)) & 3u;
      if (m & 1u) h[e] &= 0xFFFF0000u;
      if (m & 2u) h[e] &= 0x0000FFFFu;
    }
    dst[c8] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// Out (rows x ncols) = A (rows x red) * Bm (red x ncols), fp32 FMA.
//   A is bf16 or fp32; TRANS_A: element (m, k) is A[k * lda + m], else A[m * lda + k].
//   Bm is fp32 with leading dimension ldb; its columns past ncols are never read.
// CTA tile: 64 output rows x up to 160 columns, the reduction in chunks of 32 over
// [blockIdx.y * red_chunk, ...).  256 threads as 16 x 16: rows 4 ty .. 4 ty + 3,
// columns tx + 16 j.
//   MODE 0: atomicAdd into outf[m * ldo + c] (split reduction, outf zeroed first)
//   MODE 1: outf[m * ldo + c] = v
//   MODE 2: outb[m * ldo + c] = bf16(v)              (row-major bf16)
//   MODE 3: outb[c * ldo + m] = bf16(v)              (transposed bf16)
// Shapes: rows % 64 == 0, red % 32 == 0, red_chunk % 32 == 0, ncols <= 160; A rows
// 16-byte aligned (lda a multiple of 8 elements for bf16, 4 for fp32).
template <typename TA, bool TRANS_A, int MODE>
__global__ void __launch_bounds__(256) skinny_gemm_kernel(const TA* __restrict__ A, int lda,
                                                          int rows, int red, int red_chunk,
                                                          const float* __restrict__ Bm, int ldb,
                                                          int ncols, float* __restrict__ outf,
                                                          uint16_t* __restrict__ outb, int ldo) {
  __shared__ float As[32][65];         // [reduction][row]
  __shared__ float Bs[32][kSvdMaxL];   // [reduction][column]
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const int m0 = blockIdx.x * 64;
  const int k_begin = blockIdx.y * red_chunk;
  const int k_end = min(red, k_begin + red_chunk);
  const int nj = (ncols + 15) / 16;
  float acc[4][10];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 10; ++j) acc[i][j] = 0.f;

  for (int k0 = k_begin; k0 < k_end; k0 += 32) {
    // ---- A tile: 64 rows x 32 reduction entries
    if constexpr (sizeof(TA) == 2) {
      if (!TRANS_A) {
        const int row = t >> 2, cc = (t & 3) * 8;
        const uint4 v = *reinterpret_cast<const uint4*>(A + static_cast<size_t>(m0 + row) * lda + k0 + cc);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          As[cc + 2 * e][row] = bf16_to_f32(h[e] & 0xFFFFu);
          As[cc + 2 * e + 1][row] = bf16_to_f32(h[e] >> 16);
        }
      } else {
        const int kr = t >> 3, cc = (t & 7) * 8;
        const uint4 v = *reinterpret_cast<const uint4*>(A + static_cast<size_t>(k0 + kr) * lda + m0 + cc);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          As[kr][cc + 2 * e] = bf16_to_f32(h[e] & 0xFFFFu);
          As[kr][cc + 2 * e + 1] = bf16_to_f32(h[e] >> 16);
        }
      }
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int idx = t + 256 * half;
        if (!TRANS_A) {
          const int row = idx >> 3, cc = (idx & 7) * 4;
          const float4 v = *reinterpret_cast<const float4*>(A + static_cast<size_t>(m0 + row) * lda + k0 + cc);
          As[cc][row] = v.x;
          As[cc + 1][row] = v.y;
          As[cc + 2][row] = v.z;
          As[cc + 3][row] = v.w;
        } else {
          const int kr = idx >> 4, cc = (idx & 15) * 4;
          const float4 v = *reinterpret_cast<const float4*>(A + static_cast<size_t>(k0 + kr) * lda + m0 + cc);
          As[kr][cc] = v.x;
          As[kr][cc + 1] = v.y;
          As[kr][cc + 2] = v.z;
          As[kr][cc + 3] = v.w;
        }
      }
    }
    // ---- B tile: 32 reduction entries x ncols (columns past ncols read as zero)
    for (int idx = t; idx < 32 * 16 * nj; idx += 256) {
      const int kr = idx / (16 * nj), c = idx % (16 * nj);
      Bs[kr][c] = c < ncols ? Bm[static_cast<size_t>(k0 + kr) * ldb + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kr = 0; kr < 32; ++kr) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kr][4 * ty + i];
#pragma unroll
      for (int j = 0; j < 10; ++j) {
        if (j < nj) {
          const float bv = Bs[kr][tx + 16 * j];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(a[i], bv, acc[i][j]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + 4 * ty + i;
#pragma unroll
    for (int j = 0; j < 10; ++j) {
      const int c = tx + 16 * j;
      if (j >= nj || c >= ncols) continue;
      const float v = acc[i][j];
      if constexpr (MODE == 0) atomicAdd(outf + static_cast<size_t>(m) * ldo + c, v);
      if constexpr (MODE == 1) outf[static_cast<size_t>(m) * ldo + c] = v;
      if constexpr (MODE == 2)
        outb[static_cast<size_t>(m) * ldo + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      if constexpr (MODE == 3)
        outb[static_cast<size_t>(c) * ldo + m] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
}

// G (l x l, fp64, zeroed first) += Y^T Y over this CTA's rows of Y (rows x ldy fp32).
// 1024 threads as 32 x 32, thread (tx, ty) owning G[5 ty + a][5 tx + b]: products of a
// 32-row chunk are summed in fp32 registers, each chunk's sums added into this CTA's
// fp64 partial G in shared memory, and the partial G added into G at the end.
__global__ void __launch_bounds__(1024) gram_kernel(const float* __restrict__ Y, int ldy, int rows,
                                                    int l, int rows_per_cta,
                                                    double* __restrict__ G) {
  extern __shared__ double Gs[];  // l x l
  __shared__ float Ys[32][kSvdMaxL + 1];
  const int t = threadIdx.x, tx = t & 31, ty = t >> 5;
  const int r_begin = blockIdx.x * rows_per_cta;
  const int r_end = min(rows, r_begin + rows_per_cta);
  for (int idx = t; idx < l * l; idx += 1024) Gs[idx] = 0.0;
  for (int r0 = r_begin; r0 < r_end; r0 += 32) {
    __syncthreads();
    for (int idx = t; idx < 32 * kSvdMaxL; idx += 1024) {
      const int rr = idx / kSvdMaxL, c = idx % kSvdMaxL;
      Ys[rr][c] = (r0 + rr < r_end && c < l) ? Y[static_cast<size_t>(r0 + rr) * ldy + c] : 0.f;
    }
    __syncthreads();
    float acc[5][5];
#pragma unroll
    for (int a = 0; a < 5; ++a)
#pragma unroll
      for (int b = 0; b < 5; ++b) acc[a][b] = 0.f;
#pragma unroll 4
    for (int rr = 0; rr < 32; ++rr) {
      float ya[5], yb[5];
#pragma unroll
      for (int a = 0; a < 5; ++a) ya[a] = Ys[rr][5 * ty + a];
#pragma unroll
      for (int b = 0; b < 5; ++b) yb[b] = Ys[rr][5 * tx + b];
#pragma unroll
      for (int a = 0; a < 5; ++a)
#pragma unroll
        for (int b = 0; b < 5; ++b) acc[a][b] = fmaf(ya[a], yb[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 5; ++a)
#pragma unroll
      for (int b = 0; b < 5; ++b) {
        const int i = 5 * ty + a, j = 5 * tx + b;
        if (i < l && j < l) Gs[i * l + j] += static_cast<double>(acc[a][b]);
      }
  }
  __syncthreads();
  for (int idx = t; idx < l * l; idx += 1024) atomicAdd(G + idx, Gs[idx]);
}

// One CTA: Cholesky G = R^T R (R upper, G l x l fp64) and R^-1 written to Rinv (ldr x ldr
// fp32, zero outside l x l).  A pivot at or below 1e-12 of the largest diagonal entry
// marks its column as dependent: its row of R is dropped and its column of R^-1 is
// zero, so Y R^-1 has an exact zero column there and orthonormal columns elsewhere.
__global__ void __launch_bounds__(1024) chol_inv_kernel(const double* __restrict__ G, int l,
                                                        float* __restrict__ Rinv, int ldr) {
  extern __shared__ double Rs[];  // l x (l + 1): the odd stride spreads column walks over the banks
  __shared__ double tmp[kSvdMaxL];
  __shared__ unsigned char dead[kSvdMaxL];
  __shared__ double s_d;  // the current pivot's square root
  const int t = threadIdx.x, nt = blockDim.x, tx = t & 31, ty = t >> 5;
  const int ld = l + 1;
  for (int idx = t; idx < l * l; idx += nt) Rs[(idx / l) * ld + idx % l] = G[idx];
  __syncthreads();
  double dmax = 0.0;
  for (int j = 0; j < l; ++j) dmax = fmax(dmax, Rs[j * ld + j]);
  const double tol = 1e-12 * dmax;
  if (t == 0) {
    dead[0] = !(Rs[0] > tol);
    s_d = dead[0] ? 1.0 : sqrt(Rs[0]);
  }
  __syncthreads();
  // right-looking Cholesky on the upper triangle; the pivot of column j + 1 is taken
  // by thread 0, which also owns the update of that diagonal entry
  for (int j = 0; j < l; ++j) {
    const double d = s_d;
    const bool is_dead = dead[j];
    for (int k = j + t; k < l; k += nt)
      Rs[j * ld + k] = is_dead ? (k == j ? 1.0 : 0.0) : (k == j ? d : Rs[j * ld + k] / d);
    __syncthreads();
    if (!is_dead) {
      for (int a = j + 1 + ty; a < l; a += 32) {
        const double ra = Rs[j * ld + a];
        for (int b = j + 1 + tx; b < l; b += 32)
          if (b >= a) Rs[a * ld + b] -= ra * Rs[j * ld + b];
      }
    }
    if (t == 0 && j + 1 < l) {
      const double piv = Rs[(j + 1) * ld + j + 1];
      dead[j + 1] = !(piv > tol);
      s_d = dead[j + 1] ? 1.0 : sqrt(piv);
    }
    __syncthreads();
  }
  // clear the lower triangle, then invert the upper triangle in place, column by column
  for (int idx = t; idx < l * l; idx += nt)
    if (idx / l > idx % l) Rs[(idx / l) * ld + idx % l] = 0.0;
  __syncthreads();
  const int warp = t >> 5, lane = t & 31, nwarp = nt >> 5;
  for (int j = 0; j < l; ++j) {
    const double djj = 1.0 / Rs[j * ld + j];
    for (int i = warp; i < j; i += nwarp) {  // one warp per entry, lanes split the sum
      double s = 0.0;
      for (int k = i + lane; k < j; k += 32) s += Rs[i * ld + k] * Rs[k * ld + j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) tmp[i] = s;
    }
    __syncthreads();
    for (int i = t; i < j; i += nt) Rs[i * ld + j] = -tmp[i] * djj;
    if (t == 0) Rs[j * ld + j] = djj;
    __syncthreads();
  }
  for (int idx = t; idx < ldr * ldr; idx += nt) {
    const int i = idx / ldr, j = idx % ldr;
    float v = 0.f;
    if (i < l && j < l && !dead[j]) v = static_cast<float>(Rs[i * ld + j]);
    Rinv[idx] = v;
  }
}

__device__ __forceinline__ float block_sum_f32(float v, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < nw; ++w) s += sh[w];
  __syncthreads();
  return s;
}

// One CTA: cyclic Jacobi on the symmetric H (l x l, fp64 from gram_kernel, iterated in
// fp32: H itself carries the fp32 rounding of its inputs), pairs in round-robin order
// so that each round's rotations touch disjoint rows and columns.  H and the
// accumulated rotations U stay in shared memory.  A pair is rotated only when its
// off-diagonal entry is not negligible against its diagonal (1e-7 relative); the
// iteration stops when the off-diagonal mass is below 1e-12 of the total or a whole
// sweep rotated nothing, after at most kSvdMaxSweeps sweeps (status bit DEV_ERR_TIMEOUT
// if that bound is hit).  Then, with the eigenvalues sorted descending (lambda = s^2):
//   sigma[i] = s_i (i < r), MA[:, i] = U[:, pi(i)] s_i^(-1/2), MB[:, i] = U[:, pi(i)] s_i^(1/2)
// (MA, MB ldm x ldm fp32, zero outside l x r; a direction with s_i at or below 1e-6 of
// s_1 gets zero columns).
__global__ void __launch_bounds__(1024) jacobi_eig_kernel(const double* __restrict__ Hin, int l,
                                                          int r, float* __restrict__ MA,
                                                          float* __restrict__ MB, int ldm,
                                                          float* __restrict__ sigma,
                                                          int* status) {
  extern __shared__ float jsm[];  // H, then U, each l rows of odd stride ld
  const int ld = l | 1;            // an odd stride spreads column walks over the banks
  float* H = jsm;
  float* U = jsm + l * ld;
  __shared__ float red_sh[32];
  __shared__ float cs_c[kSvdMaxL / 2 + 1], cs_s[kSvdMaxL / 2 + 1];
  __shared__ int pr_p[kSvdMaxL / 2 + 1], pr_q[kSvdMaxL / 2 + 1];
  __shared__ int perm[kSvdMaxL];
  __shared__ float lam[kSvdMaxL];
  __shared__ int rotated;
  const int t = threadIdx.x, nt = blockDim.x;
  for (int idx = t; idx < l * l; idx += nt) {
    const int i = idx / l, j = idx % l;
    H[i * ld + j] = static_cast<float>(Hin[idx]);
    U[i * ld + j] = (i == j) ? 1.f : 0.f;
  }
  __syncthreads();
  const int lp = l + (l & 1);  // even count; index l (if l is odd) is a dummy
  const int npair = lp / 2, m = lp - 1;
  const int tpp = nt / npair;  // threads per pair (at least 12 for l <= 160)
  const int my_pair = t / tpp, my_sub = t % tpp;
  bool converged = false;
  for (int sweep = 0; sweep < kSvdMaxSweeps && !converged; ++sweep) {
    float off = 0.f, all = 0.f;
    for (int i = t >> 5; i < l; i += 32)
      for (int j = t & 31; j < l; j += 32) {
        const float v = H[i * ld + j] * H[i * ld + j];
        all += v;
        if (i != j) off += v;
      }
    off = block_sum_f32(off, red_sh);
    all = block_sum_f32(all, red_sh);
    if (!(off > 1e-12f * all)) {
      converged = true;
      break;
    }
    if (t == 0) rotated = 0;
    __syncthreads();
    for (int round = 0; round < m; ++round) {
      if (t < npair) {
        int p, q;
        if (t == 0) {
          p = round % m;
          q = m;
        } else {
          p = (round + t) % m;
          q = (round - t + m) % m;
        }
        if (p > q) {
          const int x = p;
          p = q;
          q = x;
        }
        float c = 1.f, sn = 0.f;
        bool rot = false;
        if (q < l) {
          const float a = H[p * ld + p], d = H[q * ld + q], b = H[p * ld + q];
          if (fabsf(b) > 1e-7f * sqrtf(fabsf(a * d)) && b != 0.f) {
            const float tau = (d - a) / (2.f * b);
            const float tt = (tau >= 0.f ? 1.f : -1.f) / (fabsf(tau) + sqrtf(1.f + tau * tau));
            c = rsqrtf(1.f + tt * tt);
            sn = tt * c;
            rot = true;
          }
        }
        if (rot) rotated = 1;
        cs_c[t] = c;
        cs_s[t] = sn;
        pr_p[t] = p;
        pr_q[t] = rot ? q : p;  // an empty or dummy pair rotates nothing
      }
      __syncthreads();
      // H <- H J and U <- U J: columns p, q of every row; thread t serves pair
      // t / tpp, rows t % tpp, t % tpp + tpp, ...
      if (my_pair < npair && pr_p[my_pair] != pr_q[my_pair]) {
        const int p = pr_p[my_pair], q = pr_q[my_pair];
        const float c = cs_c[my_pair], sn = cs_s[my_pair];
        for (int x = my_sub; x < l; x += tpp) {
          const float hp = H[x * ld + p], hq = H[x * ld + q];
          H[x * ld + p] = c * hp - sn * hq;
          H[x * ld + q] = sn * hp + c * hq;
          const float up = U[x * ld + p], uq = U[x * ld + q];
          U[x * ld + p] = c * up - sn * uq;
          U[x * ld + q] = sn * up + c * uq;
        }
      }
      __syncthreads();
      // H <- J^T H: rows p, q of every column
      if (my_pair < npair && pr_p[my_pair] != pr_q[my_pair]) {
        const int p = pr_p[my_pair], q = pr_q[my_pair];
        const float c = cs_c[my_pair], sn = cs_s[my_pair];
        for (int x = my_sub; x < l; x += tpp) {
          const float hp = H[p * ld + x], hq = H[q * ld + x];
          H[p * ld + x] = c * hp - sn * hq;
          H[q * ld + x] = sn * hp + c * hq;
        }
      }
      __syncthreads();
    }
    if (!rotated) converged = true;
    __syncthreads();
  }
  if (!converged && t == 0) atomicOr(status, DEV_ERR_TIMEOUT);
  // eigenvalues, sorted descending (ties by index)
  for (int i = t; i < l; i += nt) lam[i] = H[i * ld + i];
  __syncthreads();
  for (int i = t; i < l; i += nt) {
    int rank = 0;
    for (int j = 0; j < l; ++j) rank += (lam[j] > lam[i]) || (lam[j] == lam[i] && j < i);
    perm[rank] = i;
  }
  __syncthreads();
  const float s1 = sqrtf(fmaxf(lam[perm[0]], 0.f));
  for (int idx = t; idx < ldm * ldm; idx += nt) {
    const int row = idx / ldm, col = idx % ldm;
    float va = 0.f, vb = 0.f;
    if (row < l && col < r) {
      const float sv = sqrtf(fmaxf(lam[perm[col]], 0.f));
      if (sv > 1e-6f * s1 && sv > 0.f) {
        const float u = U[row * ld + perm[col]];
        va = u * rsqrtf(sv);
        vb = u * sqrtf(sv);
      }
    }
    MA[idx] = va;
    MB[idx] = vb;
  }
  for (int i = t; i < r; i += nt) sigma[i] = sqrtf(fmaxf(lam[perm[i]], 0.f));
}

}  // namespace salr
