"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against brute force, a closed form, a hand-worked fixture
or an invariant, chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, a wrong tie rule) fails at least one of them.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import salr_synth as synth
from salr_synth import bf16_bits_to_f64

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def to_bits(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def read_matrix_blocks(path):
    out, meta = {}, {}
    lines = [l.split("#")[0].strip() for l in open(path)]
    lines = [l for l in lines if l]
    i = 0
    while i < len(lines):
        head = lines[i].split()
        if head[0] == "sparsity":
            meta["sparsity"] = float(head[1])
            i += 1
            continue
        name, r, c = head[0], int(head[1]), int(head[2])
        rows = [[float(v) for v in lines[i + 1 + k].split()] for k in range(r)]
        out[name] = np.array(rows, dtype=np.float64).reshape(r, c)
        i += 1 + r
    return out, meta


# ---------------------------------------------------------------- mask

def rank_counting_mask(vals, keep):
    """Independent formulation: entry i is kept iff fewer than `keep` entries beat it,
    where j beats i when |w_j| > |w_i|, or |w_j| == |w_i| and j < i."""
    a = [abs(float(v)) for v in vals]
    kept = []
    for i in range(len(a)):
        beaters = sum(1 for j in range(len(a)) if a[j] > a[i] or (a[j] == a[i] and j < i))
        kept.append(beaters < keep)
    return np.array(kept)


def test_mask_handworked_rows(golden_dir):
    for line in open(os.path.join(golden_dir, "mask_rows.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        vals_s, s_s, kept_s = [p.strip() for p in line.split("|")]
        vals = [float(v) for v in vals_s.split()]
        s = float(s_s)
        expect = sorted(int(v) for v in kept_s.split())
        m = oracle.magnitude_mask(to_bits([vals]), s)
        assert sorted(np.nonzero(m[0])[0].tolist()) == expect, line


def test_mask_bruteforce_many_ties():
    rng = np.random.default_rng(1)
    palette = np.array([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0, np.inf, -np.inf])
    for K in (4, 7, 8, 13, 16):
        for s in (0.0, 0.25, 0.5, 0.75):
            rows = palette[rng.integers(0, len(palette), size=(12, K))]
            m = oracle.magnitude_mask(to_bits(rows), s)
            keep = oracle.keep_count(K, s)
            for r in range(rows.shape[0]):
                assert (m[r] == rank_counting_mask(rows[r], keep)).all()


def test_mask_exhaustive_small_rows():
    # every row of length 6 over a small alphabet with many equal magnitudes
    K, keep = 6, 3
    for combo in itertools.product([0.0, 1.0, -1.0, 2.0], repeat=K):
        m = oracle.magnitude_mask(to_bits([combo]), 0.5)[0]
        assert m.sum() == keep
        assert (m == rank_counting_mask(combo, keep)).all()


def test_mask_invariants_on_workload_rows():
    wl = synth.WORKLOADS["q_proj"]
    rows = np.array([0, 1, 17, 2048, 4095])
    w = synth.weight(wl, rows=rows)
    m = oracle.magnitude_mask(w, 0.5)
    a = np.abs(bf16_bits_to_f64(w))
    keep = wl.K // 2
    assert (m.sum(axis=1) == keep).all()
    for r in range(len(rows)):
        kept, pruned = a[r][m[r]], a[r][~m[r]]
        assert kept.min() >= pruned.max()
        thr = kept.min()
        tie_kept = np.nonzero(m[r] & (a[r] == thr))[0]
        tie_pruned = np.nonzero(~m[r] & (a[r] == thr))[0]
        if len(tie_pruned):
            assert tie_kept.max() < tie_pruned.min()


def test_mask_heavy_tail_rows_have_ties():
    # bf16 rows of 8192 heavy-tailed values tie at the threshold; the rule decides
    wl = synth.WORKLOADS["large"]
    w = synth.weight(wl, rows=[3])
    a = np.abs(bf16_bits_to_f64(w[0]))
    m = oracle.magnitude_mask(w, 0.5)[0]
    thr = a[m].min()
    assert (a == thr).sum() > 1
    assert m.sum() == wl.K // 2


def test_mask_rejects_nan_and_bad_sparsity():
    w = to_bits([[1.0, float("nan"), 2.0, 3.0]])
    with pytest.raises(oracle.OracleError):
        oracle.magnitude_mask(w, 0.5)
    for s in (-0.1, 1.0, 1.5, float("nan")):
        with pytest.raises(oracle.OracleError):
            oracle.keep_count(8, s)


def test_keep_count_closed_form():
    assert oracle.keep_count(4096, 0.5) == 2048
    assert oracle.keep_count(11008, 0.5) == 5504
    assert oracle.keep_count(7, 0.5) == 4
    assert oracle.keep_count(10, 0.3) == 7
    assert oracle.keep_count(64, 0.0) == 64


def test_prune_keeps_sign_of_kept_zero_and_zeroes_pruned():
    w = to_bits([[-0.0, 1.0, -2.0, 0.0]])
    m = np.array([[True, False, True, False]])
    p = oracle.prune(w, m)
    assert p.tolist() == [[0x8000, 0x0000, int(to_bits([-2.0])[0]), 0x0000]]


# ---------------------------------------------------------------- format

def test_format_handworked_block(golden_dir):
    wbits = np.zeros((128, 64), dtype=np.uint16)
    mask = np.zeros((128, 64), dtype=bool)
    checks, offs = [], None
    for line in open(os.path.join(golden_dir, "format_block.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        p = line.split()
        if p[0] == "kept":
            r, c, v = int(p[1]), int(p[2]), int(p[3], 16)
            wbits[r, c] = v
            mask[r, c] = True
        elif p[0] == "bytes":
            checks.append((int(p[1]), bytes(int(x, 16) for x in p[2:])))
        elif p[0] == "offsets":
            offs = [int(x) for x in p[1:]]
    o, blob = oracle.encode_format(wbits, mask)
    assert o.tolist() == offs
    raw = blob.tobytes()
    covered = set()
    for at, expect in checks:
        assert raw[at:at + len(expect)] == expect, at
        covered |= set(range(at, at + len(expect)))
    # every other bitmap byte is zero
    assert all(raw[i] == 0 for i in range(1024) if i not in covered)
    assert len(raw) == offs[-1] * 16
    assert (oracle.decode_format(o, blob, 128, 64) == wbits).all()


def test_format_roundtrip_and_block_sizes():
    wl = synth.Workload("t", 256, 192, (8,), (4,))
    w = synth.weight(wl)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    offs, blob = oracle.encode_format(wp, m)
    assert (oracle.decode_format(offs, blob, 256, 192) == wp).all()
    nb = np.diff(offs.astype(np.int64))
    for b in range(len(nb)):
        i, j = divmod(b, 3)
        nnz = int(m[128 * i:128 * (i + 1), 64 * j:64 * (j + 1)].sum())
        assert nb[b] == (1024 + 2 * nnz + 15) // 16
    assert m.sum() == 256 * 96  # exactly 50% of every row


# ---------------------------------------------------------------- linear

def test_linear_handworked(golden_dir):
    mats, meta = read_matrix_blocks(os.path.join(golden_dir, "linear_handworked.txt"))
    wb = to_bits(mats["W"])
    m = oracle.magnitude_mask(wb, meta["sparsity"])
    wp = oracle.prune(wb, m)
    assert (bf16_bits_to_f64(wp) == mats["Wp"]).all()
    ad = [(to_bits(mats["A1"]), to_bits(mats["B1"])), (to_bits(mats["A2"]), to_bits(mats["B2"]))]
    y = oracle.linear(to_bits(mats["X"]), wp, ad)
    assert (y == mats["Y"]).all()
    s = oracle.abs_bound(to_bits(mats["X"]), wp, ad)
    assert (s == mats["S"]).all()
    acat, bcat = oracle.concat_adapters(ad)
    assert (oracle.linear(to_bits(mats["X"]), wp, [(acat, bcat)]) == mats["Y"]).all()


def exact_linear(X, W, A, B):
    """Brute force in exact rational arithmetic (Python Fractions)."""
    M, K = len(X), len(X[0])
    N = len(W)
    R = len(A[0]) if A else 0
    F = [[Fraction(v) for v in row] for row in X]
    Wf = [[Fraction(v) for v in row] for row in W]
    Af = [[Fraction(v) for v in row] for row in A]
    Bf = [[Fraction(v) for v in row] for row in B]
    Y = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        t = [sum(F[m][k] * Af[k][j] for k in range(K)) for j in range(R)]
        for n in range(N):
            acc = sum(F[m][k] * Wf[n][k] for k in range(K))
            acc += sum(t[j] * Bf[j][n] for j in range(R))
            Y[m][n] = acc
    return Y


def test_linear_exact_bruteforce_small_integers():
    rng = np.random.default_rng(7)
    for (M, N, K, R) in [(1, 3, 5, 1), (4, 6, 8, 3), (3, 2, 9, 4)]:
        X = rng.integers(-8, 9, size=(M, K)).astype(np.float64)
        W = rng.integers(-8, 9, size=(N, K)).astype(np.float64) / 4
        A = rng.integers(-4, 5, size=(K, R)).astype(np.float64)
        B = rng.integers(-4, 5, size=(R, N)).astype(np.float64) / 2
        wb = to_bits(W)
        m = oracle.magnitude_mask(wb, 0.5)
        wp = oracle.prune(wb, m)
        Wpf = bf16_bits_to_f64(wp)
        y = oracle.linear(to_bits(X), wp, [(to_bits(A), to_bits(B))])
        ex = exact_linear(X.tolist(), Wpf.tolist(), A.tolist(), B.tolist())
        assert y.tolist() == [[float(v) for v in row] for row in ex]


def test_linear_identity_rows_reproduce_wp_columns():
    # X = rows of the identity and no adapter: Y[k, n] = Wp[n, k] exactly (N != K
    # so a transposed operand cannot pass)
    wl = synth.Workload("t", 48, 32, (4,), (1,))
    w = synth.weight(wl)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    eye = to_bits(np.eye(32))
    y = oracle.linear(eye, wp, [])
    assert (y == bf16_bits_to_f64(wp).T).all()
    # adapter alone (W = 0): Y[k] = A[k] B
    a = synth.draw("normal", 0, 10, (32, 4), 0.5)
    b = synth.draw("normal", 0, 20, (4, 48), 0.5)
    y2 = oracle.linear(eye, np.zeros((48, 32), np.uint16), [(a, b)])
    assert np.allclose(y2, bf16_bits_to_f64(a) @ bf16_bits_to_f64(b), rtol=0, atol=1e-15)


def test_sparsity_zero_is_dense_layer():
    wl = synth.Workload("t", 16, 24, (2,), (3,))
    w = synth.weight(wl)
    m = oracle.magnitude_mask(w, 0.0)
    assert m.all()
    assert (oracle.prune(w, m) == w).all()


def test_concat_identity_three_adapters():
    wl = synth.WORKLOADS["up_proj"]
    K, N = 256, 192
    X = synth.draw("normal", 0, 2, (5, K), 1.0)
    ad = [(synth.draw("normal", 0, 10 + i, (K, r), 0.01),
           synth.draw("normal", 0, 20 + i, (r, N), 0.01)) for i, r in enumerate(wl.ranks)]
    zero = np.zeros((N, K), np.uint16)
    separate = sum(oracle.linear(X, zero, [p]) for p in ad)
    acat, bcat = oracle.concat_adapters(ad)
    assert acat.shape == (K, 96) and bcat.shape == (96, N)
    joint = oracle.linear(X, zero, [(acat, bcat)])
    assert np.linalg.norm(joint - separate) <= 1e-12 * np.linalg.norm(separate)
    # order of the stack is irrelevant
    acat2, bcat2 = oracle.concat_adapters(ad[::-1])
    assert np.allclose(oracle.linear(X, zero, [(acat2, bcat2)]), joint, rtol=1e-13, atol=0)


# ---------------------------------------------------------------- tolerance

def test_tolerance_catches_planted_mistakes():
    wl = synth.WORKLOADS["tiny"]
    w = synth.weight(wl)
    x = synth.activations(wl, 16)
    ad = synth.adapters(wl)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    ystar = oracle.linear(x, wp, ad)
    s = oracle.abs_bound(x, wp, ad)
    # the correct result rounded to bf16 passes
    ok, rel, worst = oracle.check_tolerance(to_bits(ystar), ystar, s)
    assert ok and rel < 3e-3 and worst < 4e-3
    # dropped adapter term
    assert not oracle.check_tolerance(to_bits(oracle.linear(x, wp, [])), ystar, s)[0]
    # unpruned weight
    assert not oracle.check_tolerance(to_bits(oracle.linear(x, w, ad)), ystar, s)[0]
    # pruning the lower-magnitude half instead
    wrong = oracle.prune(w, ~m)
    assert not oracle.check_tolerance(to_bits(oracle.linear(x, wrong, ad)), ystar, s)[0]
    # sign of the adapter flipped
    flip = [(a, b ^ np.uint16(0x8000)) for a, b in ad]
    assert not oracle.check_tolerance(to_bits(oracle.linear(x, wp, flip)), ystar, s)[0]
    # one wrong element
    bad = ystar.copy()
    bad[3, 7] += 0.05 * s[3, 7]
    assert not oracle.check_tolerance(bad, ystar, s)[0]


# ---------------------------------------------------------------- residual SVD

def test_svd_adapter_closed_form_known_spectrum():
    rng = np.random.default_rng(3)
    N, K, r = 40, 24, 5
    q1, _ = np.linalg.qr(rng.standard_normal((N, N)))
    q2, _ = np.linalg.qr(rng.standard_normal((K, K)))
    sv = np.sort(rng.uniform(0.1, 3.0, size=K))[::-1]
    E = q1[:, :K] @ np.diag(sv) @ q2.T
    A, B, got = oracle.truncated_svd_adapter(E, r)
    assert np.allclose(got, sv, rtol=1e-12)
    Er_t = A @ B  # = E_r^T
    expect = q1[:, :r] @ np.diag(sv[:r]) @ q2[:, :r].T
    assert np.allclose(Er_t.T, expect, atol=1e-11)
    tail = np.linalg.norm(E - Er_t.T) ** 2
    assert abs(tail - (sv[r:] ** 2).sum()) <= 1e-10 * (sv ** 2).sum()


def test_svd_residual_eckart_young_bound_on_pruned_weight():
    wl = synth.WORKLOADS["tiny"]
    w = synth.weight(wl)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    E = oracle.residual(w, wp)
    # the residual is exactly the pruned-away half
    assert (E[m] == 0).all() and (E[~m] == bf16_bits_to_f64(w)[~m]).all()
    total = np.linalg.norm(E) ** 2
    for r in (1, 8, 32, 128):
        A, B, sv = oracle.truncated_svd_adapter(E, r)
        tail = np.linalg.norm(E - (A @ B).T) ** 2
        assert abs(tail - (total - (sv[:r] ** 2).sum())) <= 1e-10 * total
        assert tail <= oracle.mse_factor(r, wl.N, wl.K) * total * (1 + 1e-12)


def test_svd_truncation_is_optimal_against_random_rank_r():
    rng = np.random.default_rng(5)
    E = rng.standard_normal((30, 20))
    r = 4
    A, B, _ = oracle.truncated_svd_adapter(E, r)
    best = np.linalg.norm(E - (A @ B).T)
    for _ in range(200):
        P = rng.standard_normal((30, r))
        Q, _ = np.linalg.qr(P)
        cand = Q @ (Q.T @ E)  # best approximation within a random rank-r column space
        assert np.linalg.norm(E - cand) >= best - 1e-12


def _known_spectrum(rng, N, K, sv):
    q1, _ = np.linalg.qr(rng.standard_normal((N, N)))
    q2, _ = np.linalg.qr(rng.standard_normal((K, K)))
    k = len(sv)
    return q1[:, :k] @ np.diag(sv) @ q2[:, :k].T, q1, q2


def test_randomized_adapter_exact_when_rank_fits_the_sample():
    # rank(E) <= l: the range finder captures range(E) exactly, so the result is the
    # exact truncated SVD (closed form from the construction)
    rng = np.random.default_rng(11)
    sv = np.array([5.0, 3.0, 2.0, 1.5, 0.7, 0.2])
    E, q1, q2 = _known_spectrum(rng, 40, 24, sv)
    r, l = 4, 8
    A, B, got = oracle.randomized_svd_adapter(E, r, rng.standard_normal((24, l)), 0)
    assert np.allclose(got[:6], sv, rtol=1e-10) and np.all(np.abs(got[6:]) < 1e-10)
    expect = q1[:, :r] @ np.diag(sv[:r]) @ q2[:, :r].T  # E_r
    assert A.shape == (24, r) and B.shape == (r, 40)
    assert np.allclose((A @ B).T, expect, atol=1e-10)


def test_randomized_adapter_ritz_values_and_eckart_young_floor():
    # singular values of Q^T E never exceed those of E (interlacing), and no rank-r
    # product beats the truncated SVD's error
    rng = np.random.default_rng(12)
    E = rng.standard_normal((50, 36))
    sv = np.linalg.svd(E, compute_uv=False)
    total = (sv ** 2).sum()
    for q in (0, 1, 3):
        for r, l in ((3, 5), (8, 12)):
            A, B, got = oracle.randomized_svd_adapter(E, r, rng.standard_normal((36, l)), q)
            assert np.all(got <= sv[:l] * (1 + 1e-12))
            err = np.linalg.norm(E - (A @ B).T) ** 2
            assert err >= (total - (sv[:r] ** 2).sum()) * (1 - 1e-12)
            # the adapter is the rank-r truncation of the projection Q Q^T E, so its
            # error is the projection's error plus the dropped Ritz values
            assert abs(err - (total - (got[:r] ** 2).sum())) <= 1e-9 * total


def test_randomized_adapter_converges_on_a_decaying_spectrum():
    # square, non-symmetric E with geometric singular values: subspace iteration on
    # E and E^T reaches the truncated SVD; a wrong operand (E for E^T) would not
    rng = np.random.default_rng(13)
    sv = 0.7 ** np.arange(50)
    E, _, _ = _known_spectrum(rng, 50, 50, sv)
    r, l = 5, 10
    opt = (sv[r:] ** 2).sum()
    A, B, got = oracle.randomized_svd_adapter(E, r, rng.standard_normal((50, l)), 6)
    err = np.linalg.norm(E - (A @ B).T) ** 2
    assert err <= opt * (1 + 1e-8)
    assert np.allclose(got[:r], sv[:r], rtol=1e-8)


def test_randomized_adapter_depends_only_on_the_sampled_subspace():
    rng = np.random.default_rng(14)
    E = rng.standard_normal((30, 26))
    om = rng.standard_normal((26, 9))
    G = rng.standard_normal((9, 9)) + 3 * np.eye(9)
    for q in (0, 2):
        A1, B1, s1 = oracle.randomized_svd_adapter(E, 4, om, q)
        A2, B2, s2 = oracle.randomized_svd_adapter(E, 4, om @ G, q)
        assert np.allclose(s1, s2, rtol=1e-9)
        assert np.allclose(A1 @ B1, A2 @ B2, atol=1e-9)


def test_randomized_adapter_meets_the_stated_mse_factor_on_a_pruned_weight():
    # the pages' guarantee, (1 - r/min(d, k)) of the residual energy left, holds for the
    # randomized adapter of a pruned synthetic weight too (its top singular values are
    # above the mean, so even a partial capture clears the bound)
    wl = synth.WORKLOADS["tiny"]
    w = synth.weight(wl)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    E = oracle.residual(w, wp)
    total = np.linalg.norm(E) ** 2
    rng = np.random.default_rng(15)
    for r in (8, 32):
        A, B, _ = oracle.randomized_svd_adapter(E, r, rng.standard_normal((wl.K, r + 8)), 2)
        err = np.linalg.norm(E - (A @ B).T) ** 2
        assert err <= oracle.mse_factor(r, wl.N, wl.K) * total


def test_mse_factor_values():
    assert oracle.mse_factor(64, 4096, 4096) == 1 - 64 / 4096
    assert oracle.mse_factor(8, 256, 128) == 1 - 8 / 128


# ---------------------------------------------------------------- inputs

def test_synth_reproducible_and_row_addressable():
    wl = synth.WORKLOADS["tiny"]
    w1, w2 = synth.weight(wl), synth.weight(wl)
    assert (w1 == w2).all()
    assert (synth.weight(wl, rows=[5, 200]) == w1[[5, 200]]).all()
    f = bf16_bits_to_f64(synth.weight(synth.WORKLOADS["q_proj"], rows=np.arange(64)))
    assert abs(f.mean()) < 1e-3 and abs(f.std() - 0.02) < 5e-4
    x = bf16_bits_to_f64(synth.activations(synth.WORKLOADS["q_proj"], 16))
    assert abs(x.std() - 1.0) < 0.02
    assert (synth.activations(synth.WORKLOADS["q_proj"], 1) ==
            synth.activations(synth.WORKLOADS["q_proj"], 16)[:1]).all()
