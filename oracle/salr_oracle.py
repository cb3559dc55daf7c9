"""fp64 CPU oracle for the SALR inference linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library; the only shared module
is ``salr_synth`` (seeded inputs, no method arithmetic).

What it computes, and where the SALR pages define it ("Sparsity-Aware Low-Rank
Representation for Efficient Fine-Tuning of Large Language Models", gist.science
technical summary, and the authors' abstract on the scholarfeed author page):

* ``magnitude_mask`` / ``prune``: static magnitude pruning of the frozen base weight
  W0 to a given sparsity, A and B left dense (Technical Summary, Methodology 1; the
  abstract's sparsity of one half).  Granularity per output row, ties to the lower column index.
* ``encode_format`` / ``decode_format``: the bitmap-plus-compact-values storage with a
  per-block offset table (Methodology 4, "Bitmap Encoding", and its first pipeline stage,
  which reads the bitmaps through lookup tables).  The on-device block layout is this library's own definition and is
  written out in ``include/salr.h``; the oracle follows that definition literally.
* ``linear``: Y = X (M (.) W)^T + sum_i (X A_i) B_i, the layer a SALR model runs at
  inference (Methodology 3, "Adapter Concatenation", with the pruned base of
  Methodology 1).  Exact fp64 on exactly widened bf16 inputs; nothing is rounded.
* ``concat_adapters``: stacking adapters along rank (Methodology 3).
* ``residual`` / ``truncated_svd_adapter``: E = W0 - W_hat and its rank-r truncated SVD
  (Methodology 2, "Residual Decomposition" and "Theoretical Guarantee").
* ``randomized_svd_adapter``: the same adapter computed the way the GPU builder does,
  by a randomized range finder with subspace (power) iteration and a dense SVD of the
  small projected matrix (Halko, Martinsson and Tropp, "Finding structure with
  randomness", SIAM Review 2011: the randomized subspace iteration, then the direct
  SVD of the projected matrix).  The pages fix only the result, a rank-r truncated SVD;
  the randomized route is this library's reading of how to reach it at scale.  The
  random test matrix is an input, so both sides use the same draws.
* ``abs_bound`` / ``check_tolerance``: the per-element and Frobenius acceptance test.

Every function here is pinned by ``tests/test_oracle.py`` against brute force, closed
forms, hand-worked fixtures and invariants (none of which re-types the function).
"""
from __future__ import annotations

import math

import numpy as np

from salr_synth import bf16_bits_to_f64

ROWS_PER_BLOCK = 128
COLS_PER_BLOCK = 64
BITMAP_BYTES = ROWS_PER_BLOCK * COLS_PER_BLOCK // 8


class OracleError(ValueError):
    pass


def keep_count(K: int, sparsity: float) -> int:
    """Entries kept per row: K - floor(sparsity * K).

    The pages fix only "50% sparsity" (abstract); for a fraction s*K that is not an
    integer this library reads the pruned count as floor(s*K).
    """
    if not (0.0 <= sparsity < 1.0) or math.isnan(sparsity):
        raise OracleError("sparsity must lie in [0, 1)")
    return K - int(math.floor(sparsity * K))


def magnitude_mask(w_bits: np.ndarray, sparsity: float) -> np.ndarray:
    """Boolean keep-mask of a bf16 weight (N x K bit patterns), per row.

    Methodology 1: prune W0 by magnitude.  Each row keeps its ``keep_count`` entries
    of largest |w|; among equal |w| the lower column index is kept first.  |+0| = |-0|;
    +-Inf rank above every finite value; a NaN anywhere is an error.
    """
    w = bf16_bits_to_f64(np.asarray(w_bits, dtype=np.uint16))
    if np.isnan(w).any():
        raise OracleError("NaN in W")
    n, k = w.shape
    keep = keep_count(k, sparsity)
    # A stable sort of -|w| lists each row by decreasing magnitude and, within a run
    # of equal magnitudes, by increasing column index.
    order = np.argsort(-np.abs(w), axis=1, kind="stable")
    mask = np.zeros((n, k), dtype=bool)
    np.put_along_axis(mask, order[:, :keep], True, axis=1)
    return mask


def prune(w_bits: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """M (.) W as bf16 bits: kept entries unchanged (sign of a kept zero included),
    pruned entries +0.0 (bit pattern 0x0000)."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    return np.where(mask, w_bits, np.uint16(0)).astype(np.uint16)


def _quarter_group_order(a: np.ndarray) -> np.ndarray:
    """A 128 x 64 block viewed as [quarter][4-column group][row in quarter][column in
    group] (4 x 16 x 32 x 4), the order of the format's value array."""
    return a.reshape(4, ROWS_PER_BLOCK // 4, COLS_PER_BLOCK // 4, 4).transpose(0, 2, 1, 3)


def encode_format(wp_bits: np.ndarray, mask: np.ndarray):
    """Byte image of the encoded weight, following the block layout of ``salr.h``.

    Returns ``(offsets, blob)``: ``offsets`` (uint32, one per block plus a final
    total) in 16-byte units, ``blob`` (uint8).  Block b = i * (K/64) + j covers rows
    128 i .. 128 i + 127 and columns 64 j .. 64 j + 63.  A block is: 128 little-endian
    uint64 bitmap words (word r, bit c set when W[128 i + r, 64 j + c] is kept), then
    the kept values as little-endian bf16, then zero bytes up to a multiple of 16.  The
    values are ordered by row quarter (block rows 32q .. 32q + 31), then by 4-column
    group (block columns 4n .. 4n + 3), then by row, then by column: the pages fix only
    "a bitmap plus a compact array of the kept values"; this order is the library's.
    """
    n, k = wp_bits.shape
    if n % ROWS_PER_BLOCK or k % COLS_PER_BLOCK:
        raise OracleError("N must be a multiple of 128 and K of 64")
    nbi, nbj = n // ROWS_PER_BLOCK, k // COLS_PER_BLOCK
    pieces = []
    offsets = np.zeros(nbi * nbj + 1, dtype=np.uint64)
    pos = 0
    weights = (np.uint64(1) << np.arange(64, dtype=np.uint64))
    for i in range(nbi):
        for j in range(nbj):
            rs = slice(i * ROWS_PER_BLOCK, (i + 1) * ROWS_PER_BLOCK)
            cs = slice(j * COLS_PER_BLOCK, (j + 1) * COLS_PER_BLOCK)
            m = mask[rs, cs]
            words = (m.astype(np.uint64) * weights[None, :]).sum(axis=1, dtype=np.uint64)
            # (row, col) -> (quarter, group, row in quarter, col in group): boolean
            # indexing then walks the values in the format's order
            mq = _quarter_group_order(m)
            vals = _quarter_group_order(wp_bits[rs, cs])[mq]
            body = words.astype("<u8").tobytes() + vals.astype("<u2").tobytes()
            pad = (-len(body)) % 16
            body += b"\x00" * pad
            offsets[i * nbj + j] = pos // 16
            pieces.append(body)
            pos += len(body)
    offsets[-1] = pos // 16
    if pos // 16 >= 1 << 32:
        raise OracleError("blob too large for 32-bit offsets")
    return offsets.astype(np.uint32), np.frombuffer(b"".join(pieces), dtype=np.uint8)


def decode_format(offsets: np.ndarray, blob: np.ndarray, n: int, k: int) -> np.ndarray:
    """Inverse of ``encode_format``: dense bf16 bits with pruned entries +0.0."""
    nbi, nbj = n // ROWS_PER_BLOCK, k // COLS_PER_BLOCK
    out = np.zeros((n, k), dtype=np.uint16)
    raw = np.asarray(blob, dtype=np.uint8).tobytes()
    for i in range(nbi):
        for j in range(nbj):
            b = i * nbj + j
            start = int(offsets[b]) * 16
            words = np.frombuffer(raw, dtype="<u8", count=ROWS_PER_BLOCK, offset=start)
            bits = ((words[:, None] >> np.arange(64, dtype=np.uint64)[None, :])
                    & np.uint64(1)).astype(bool)
            nnz = int(bits.sum())
            vals = np.frombuffer(raw, dtype="<u2", count=nnz, offset=start + BITMAP_BYTES)
            blk_q = np.zeros((4, COLS_PER_BLOCK // 4, ROWS_PER_BLOCK // 4, 4), dtype=np.uint16)
            blk_q[_quarter_group_order(bits)] = vals
            blk = blk_q.transpose(0, 2, 1, 3).reshape(ROWS_PER_BLOCK, COLS_PER_BLOCK)
            out[i * ROWS_PER_BLOCK:(i + 1) * ROWS_PER_BLOCK,
                j * COLS_PER_BLOCK:(j + 1) * COLS_PER_BLOCK] = blk
    return out


def _f64(a):
    a = np.asarray(a)
    return bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def concat_adapters(pairs):
    """A_cat = [A_1 | A_2 | ...] (K x sum r_i), B_cat = [B_1; B_2; ...] (sum r_i x N):
    the adapters stacked along their rank dimension (Methodology 3)."""
    if not pairs:
        return None, None
    return (np.concatenate([np.asarray(a) for a, _ in pairs], axis=1),
            np.concatenate([np.asarray(b) for _, b in pairs], axis=0))


def linear(x, wp, adapters=()):
    """Y* = X Wp^T + sum_i (X A_i) B_i in fp64 (no rounding of the adapter product).

    ``x`` is M x K, ``wp`` is N x K (the pruned weight), each adapter a pair (A_i K x r_i,
    B_i r_i x N); bf16 inputs are given as uint16 bit patterns and widened exactly.
    ``adapters`` may also hold a single concatenated pair (A_cat, B_cat).
    """
    X = _f64(x)
    Y = X @ _f64(wp).T
    for a, b in adapters:
        if a is None or np.asarray(a).size == 0:
            continue
        Y = Y + (X @ _f64(a)) @ _f64(b)
    return Y


def abs_bound(x, wp, adapters=()):
    """S[m,n] = sum_k |X[m,k] Wp[n,k]| + sum_j (sum_k |X[m,k] A[k,j]|) |B[j,n]|: the sum of
    the magnitudes of every product that feeds Y[m,n], adapter chain included."""
    X = np.abs(_f64(x))
    S = X @ np.abs(_f64(wp)).T
    for a, b in adapters:
        if a is None or np.asarray(a).size == 0:
            continue
        S = S + (X @ np.abs(_f64(a))) @ np.abs(_f64(b))
    return S


REL_FRO_TOL = 4e-3
ELEM_TOL = 1e-2


def check_tolerance(y, y_star, s):
    """Acceptance test of a computed Y against the oracle.

    Returns ``(ok, rel_fro, worst)``: ``rel_fro`` = ||Y - Y*||_F / ||Y*||_F (must be
    <= 4e-3) and ``worst`` = max |Y - Y*| / S over all elements (must be <= 1e-2).
    """
    y = _f64(y)
    err = y - y_star
    denom = np.linalg.norm(y_star)
    rel = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(s > 0, np.abs(err) / np.where(s > 0, s, 1.0),
                         np.where(err == 0, 0.0, np.inf))
    worst = float(ratio.max()) if ratio.size else 0.0
    ok = bool(np.isfinite(y).all() and rel <= REL_FRO_TOL and worst <= ELEM_TOL)
    return ok, rel, worst


def residual(w_bits, wp_bits):
    """E = W0 - W_hat, the part of the frozen base removed by pruning (Methodology 2).
    The pages write W - W_hat; W here is the frozen base W0, the only matrix pruned."""
    return _f64(w_bits) - _f64(wp_bits)


def truncated_svd_adapter(E, r: int):
    """Rank-r truncated SVD of the residual as an adapter pair in the X A B orientation.

    With E = U S V^T (E is N x K, out x in), X E^T = X V S U^T, so the adapter is
    A' = V_r S_r^(1/2) (K x r) and B' = S_r^(1/2) U_r^T (r x N); A' B' = E_r^T.  How S is
    split between the factors is not stated on the pages; the product does not depend
    on it.  Returns (A', B', singular values of E).
    """
    E = np.asarray(E, dtype=np.float64)
    U, sv, Vt = np.linalg.svd(E, full_matrices=False)
    r = int(min(r, len(sv)))
    root = np.sqrt(sv[:r])
    A = Vt[:r].T * root[None, :]
    B = root[:, None] * U[:, :r].T
    return A, B, sv


def randomized_svd_adapter(E, r: int, omega, q: int):
    """Rank-r adapter of E (N x K) from a randomized range finder, in fp64.

    Steps, in the order of the published algorithm (randomized subspace iteration, then
    the direct SVD): Q spans E Omega (Omega the K x l test matrix, given); q times, Q is
    replaced by an orthonormal basis of E (orthonormal basis of E^T Q); then
    B = Q^T E (l x K) is decomposed exactly, B = U_b S V^T, and U = Q U_b.  The adapter
    pair is the rank-r part in the X A B orientation: A' = V_r S_r^(1/2) (K x r) and
    B' = S_r^(1/2) U_r^T (r x N), so A' B' approximates E_r^T.  Orthonormal bases are
    taken by Householder QR (a library step); the subspace, not the basis, is what the
    result depends on.  Returns (A', B', singular values of B, descending).
    """
    E = np.asarray(E, dtype=np.float64)
    omega = np.asarray(omega, dtype=np.float64)
    n, k = E.shape
    l = omega.shape[1]
    if omega.shape[0] != k or not (1 <= r <= l <= min(n, k)) or q < 0:
        raise OracleError("need omega K x l with 1 <= r <= l <= min(N, K) and q >= 0")
    Q = np.linalg.qr(E @ omega)[0]
    for _ in range(q):
        Z = np.linalg.qr(E.T @ Q)[0]
        Q = np.linalg.qr(E @ Z)[0]
    B = Q.T @ E
    Ub, sv, Vt = np.linalg.svd(B, full_matrices=False)
    root = np.sqrt(sv[:r])
    A = Vt[:r].T * root[None, :]
    Bp = root[:, None] * (Q @ Ub[:, :r]).T
    return A, Bp, sv


def mse_factor(r: int, d: int, k: int) -> float:
    """The stated per-entry MSE reduction factor of a rank-r residual adapter,
    (1 - r / min(d, k)) (abstract; Methodology 2, "Theoretical Guarantee")."""
    return 1.0 - r / min(d, k)
