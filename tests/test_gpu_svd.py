"""GPU parity of the residual-adapter builder (salr_residual_adapter) against the oracle.

The builder is a randomized range finder with subspace iteration, so two references
apply: the oracle's fp64 run of the same algorithm on the same random test matrix (the
products A' B' must agree to bf16 output precision), and the exact truncated SVD
(Eckart-Young: no rank-r product beats it; on a spectrum that decays the builder must
reach it).
"""
import numpy as np
import pytest

import oracle
import salr_synth as synth
from gpu_util import to_bits, to_dev
from salr_synth import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
salr = pytest.importorskip("sparse_rank_linear_b200")

PROD_TOL = 5e-3  # bf16 A' and B' (2^-9 relative each) against the fp64 product


@pytest.fixture(scope="module", autouse=True)
def lib():
    from sparse_rank_linear_b200.build import build
    build()
    assert torch.cuda.is_available()
    return salr.load_library()


def f64(bits):
    return bf16_bits_to_f64(bits)


def run(w_bits, s, r, l, q, seed=1):
    """GPU adapter of W's residual at sparsity s with a numpy-drawn test matrix; returns
    (A', B', sigma) as fp64 arrays, the residual E and the test matrix."""
    rng = np.random.default_rng(seed)
    N, K = w_bits.shape
    omega = rng.standard_normal((K, l)).astype(np.float32)
    W = to_dev(w_bits)
    h = salr.encode(W, s)
    A, B, sig = salr.residual_adapter(W, h, r, q=q, omega=torch.from_numpy(omega).cuda())
    h.free()
    wp = oracle.prune(w_bits, oracle.magnitude_mask(w_bits, float(np.float32(s))))
    E = oracle.residual(w_bits, wp)
    return f64(to_bits(A)), f64(to_bits(B)), sig.cpu().numpy().astype(np.float64), E, omega


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("shape,r,l,q", [((256, 256), 8, 16, 2), ((512, 1024), 32, 48, 2),
                                         ((384, 640), 20, 31, 0), ((256, 192), 40, 72, 3)])
def test_matches_the_oracle_run_of_the_same_algorithm(shape, r, l, q):
    wl = synth.Workload("t", shape[0], shape[1], (8,), (1,))
    w = synth.weight(wl)
    A, B, sig, E, omega = run(w, 0.5, r, l, q)
    Ao, Bo, svo = oracle.randomized_svd_adapter(E, r, omega.astype(np.float64), q)
    assert A.shape == (shape[1], r) and B.shape == (r, shape[0])
    assert rel(A @ B, Ao @ Bo) <= PROD_TOL
    assert np.allclose(sig, svo[:r], rtol=1e-4)


def decaying_residual_weight(N, K, sv, seed=3):
    """W whose first K/2 columns are large (|w| >= 1: all kept at 50%) and whose last K/2
    hold a matrix of singular values ``sv`` (all |w| < 1: all pruned), so E is known."""
    rng = np.random.default_rng(seed)
    half = K // 2
    u, _ = np.linalg.qr(rng.standard_normal((N, len(sv))))
    v, _ = np.linalg.qr(rng.standard_normal((half, len(sv))))
    F = (u * sv) @ v.T
    assert np.abs(F).max() < 1.0
    big = rng.uniform(1.0, 2.0, (N, half)) * rng.choice([-1.0, 1.0], (N, half))
    full = np.concatenate([big, F], axis=1).astype(np.float32)
    bits = full.view(np.uint32)
    return ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)  # RNE to bf16


def test_reaches_the_truncated_svd_on_a_decaying_spectrum():
    N, K, r = 512, 768, 12
    w = decaying_residual_weight(N, K, 4.0 * 0.8 ** np.arange(200))
    A, B, sig, E, _ = run(w, 0.5, r, r + 16, 3)
    Ae, Be, sv = oracle.truncated_svd_adapter(E, r)
    assert rel(A @ B, Ae @ Be) <= PROD_TOL
    assert np.allclose(sig, sv[:r], rtol=1e-3)
    total = (sv ** 2).sum()
    err = np.linalg.norm(E - (A @ B).T) ** 2
    opt = total - (sv[:r] ** 2).sum()
    assert opt * (1 - 1e-3) <= err <= opt * (1 + 1e-2)


def test_eckart_young_and_the_stated_mse_factor_on_a_pruned_weight():
    wl = synth.Workload("t", 1024, 1024, (8,), (1,))
    w = synth.weight(wl)
    r = 64
    A, B, sig, E, _ = run(w, 0.5, r, 80, 2)
    sv = np.linalg.svd(E, compute_uv=False)
    total = (sv ** 2).sum()
    err = np.linalg.norm(E - (A @ B).T) ** 2
    # no rank-r product beats the truncated SVD (bf16 factors may land a hair below)
    assert err >= (total - (sv[:r] ** 2).sum()) * (1 - 1e-4)
    # the pages' guarantee for the residual adapter
    assert err <= oracle.mse_factor(r, wl.N, wl.K) * total
    # Ritz values never exceed the singular values they estimate
    assert np.all(sig <= sv[:r] * (1 + 1e-4))


def exact_rank3_residual_weight(N, K, seed=4):
    """Large kept half as above; the pruned half is sum_i 2^-(i+2) s_i t_i^T with sign
    vectors s_i, t_i, so every entry is one of +-1/4 +-1/8 +-1/16 (exact in bf16) and E
    has rank exactly 3."""
    rng = np.random.default_rng(seed)
    half = K // 2
    F = sum(2.0 ** -(i + 2) * np.outer(rng.choice([-1.0, 1.0], N), rng.choice([-1.0, 1.0], half))
            for i in range(3))
    big = rng.uniform(1.0, 2.0, (N, half)) * rng.choice([-1.0, 1.0], (N, half))
    full = np.concatenate([big, F], axis=1).astype(np.float32)
    bits = full.view(np.uint32)
    out = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    assert (f64(out)[:, half:] == F).all()
    return out


def test_rank_deficient_residual_is_reproduced():
    # E of rank 3 with l = 24: the dependent directions are dropped, no NaN appears,
    # and with r >= 3 the adapter reproduces E itself
    N, K = 256, 384
    w = exact_rank3_residual_weight(N, K)
    A, B, sig, E, _ = run(w, 0.5, 6, 24, 1)
    assert np.linalg.matrix_rank(E) == 3
    assert np.isfinite(A).all() and np.isfinite(B).all()
    assert rel(A @ B, E.T) <= PROD_TOL
    sv = np.linalg.svd(E, compute_uv=False)
    assert np.allclose(sig[:3], sv[:3], rtol=1e-4)
    assert np.all(sig[3:] <= 1e-5 * sig[0])


def test_nothing_pruned_gives_a_zero_adapter():
    wl = synth.Workload("t", 256, 256, (8,), (1,))
    A, B, sig, E, _ = run(synth.weight(wl), 0.0, 8, 16, 2)
    assert (E == 0).all()
    assert (A == 0).all() and (B == 0).all() and (sig == 0).all()


def test_default_test_matrix_and_odd_sizes():
    # the binding draws omega itself; odd l exercises the dummy index of the Jacobi
    # ordering; the adapter still meets the stated factor
    wl = synth.Workload("t", 384, 512, (8,), (1,))
    w = synth.weight(wl)
    W = to_dev(w)
    h = salr.encode(W, 0.5)
    A, B, sig = salr.residual_adapter(W, h, 7, q=2, oversample=6)  # l = 13
    h.free()
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    E = oracle.residual(w, wp)
    Ab, Bb = f64(to_bits(A)), f64(to_bits(B))
    err = np.linalg.norm(E - (Ab @ Bb).T) ** 2
    assert err <= oracle.mse_factor(7, wl.N, wl.K) * np.linalg.norm(E) ** 2
    assert np.all(np.diff(sig.cpu().numpy()) <= 0)
