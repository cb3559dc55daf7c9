"""The allocation-free entry point, through the C ABI, against the fp64 oracle.

salr_linear_noalloc serves callers that may not let a library allocate device memory
while they run (memory planned ahead of time, no allocation allowed during inference);
its scratch is a fixed array in the library's device code.  It must give the layer the
oracle defines, within the tolerance every salr_linear test uses, call after call, and
must not allocate.  This file is named to be collected last so that a run stopping at
the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest

import oracle
import salr_synth as synth
from gpu_util import to_bits, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
salr = pytest.importorskip("sparse_rank_linear_b200")


@pytest.fixture(scope="module")
def lib():
    from sparse_rank_linear_b200.build import build
    build()
    assert torch.cuda.is_available()
    return salr.load_library()


def call_noalloc(lib, X, h, A, B, Y):
    P = ctypes.c_void_p
    return lib.salr_linear_noalloc(P(X.data_ptr()), X.shape[0], h.handle,
                                   P(A.data_ptr() if A is not None else 0),
                                   P(B.data_ptr() if B is not None else 0),
                                   0 if A is None else A.shape[1], P(Y.data_ptr()),
                                   P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M", [16, 5])
def test_noalloc_matches_oracle_twice(lib, M):
    wl = synth.WORKLOADS["q_proj"]
    w = synth.weight(wl)
    x = synth.activations(wl, M)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(np.concatenate([a for a, _ in ad], axis=1))
    B = to_dev(np.concatenate([b for _, b in ad], axis=0))
    X = to_dev(x)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ref = oracle.linear(x, wp, ad)
    s = oracle.abs_bound(x, wp, ad)
    # the regular entry point on the same inputs meets the same bound
    assert oracle.check_tolerance(to_bits(salr.linear(X, h, A, B)), ref, s)[0]
    assert h.sync_status() == 0
    free_before = None
    for call in range(2):
        if call == 1:
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
        Y = torch.full((M, wl.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(lib, X, h, A, B, Y) == 0
        assert h.sync_status() == 0
        ok, rel, worst = oracle.check_tolerance(to_bits(Y), ref, s)
        assert ok, f"call {call}: rel_fro={rel:.2e} worst={worst:.2e} against the oracle"
    torch.cuda.synchronize()
    # the second call allocated nothing on the device
    assert torch.cuda.mem_get_info()[0] == free_before
    h.free()


def test_noalloc_without_adapter_and_limits(lib):
    wl = synth.Workload("t", 384, 320, (), (3,))
    w, x = synth.weight(wl), synth.activations(wl, 3)
    h = salr.encode(to_dev(w), 0.5)
    X = to_dev(x)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ref = oracle.linear(x, wp)
    for _ in range(2):
        Y = torch.empty(3, 384, dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(lib, X, h, None, None, Y) == 0
        assert h.sync_status() == 0
        assert oracle.check_tolerance(to_bits(Y), ref, oracle.abs_bound(x, wp))[0]
    # more tokens than the fixed scratch holds: a clear refusal, nothing launched
    X17 = to_dev(synth.activations(wl, 17))
    Y17 = torch.empty(17, 384, dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(lib, X17, h, None, None, Y17) == 2
    h.free()


def test_noalloc_recovers_after_a_wait_runs_out(lib, monkeypatch):
    # the readers of t wait for one part more than is ever added, under a short bound:
    # the call gives up and reports SALR_ERR_TIMEOUT; salr_sync_status clears the fixed
    # array, and the next calls match the oracle again
    wl = synth.WORKLOADS["q_proj"]
    w, x, ad = synth.weight(wl), synth.activations(wl, 16), synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(np.concatenate([a for a, _ in ad], axis=1))
    B = to_dev(np.concatenate([b for _, b in ad], axis=0))
    X = to_dev(x)
    Y = torch.empty(16, wl.N, dtype=torch.bfloat16, device="cuda")
    monkeypatch.setenv("SALR_WAIT_LIMIT_CYCLES", "400000")
    monkeypatch.setenv("SALR_FAIL_T_WAIT", "1")
    assert call_noalloc(lib, X, h, A, B, Y) == 0
    assert h.sync_status() == 5  # SALR_ERR_TIMEOUT
    monkeypatch.delenv("SALR_FAIL_T_WAIT")
    monkeypatch.delenv("SALR_WAIT_LIMIT_CYCLES")
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ref, s = oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad)
    for call in range(2):
        Y = torch.full((16, wl.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(lib, X, h, A, B, Y) == 0
        assert h.sync_status() == 0
        ok, rel, worst = oracle.check_tolerance(to_bits(Y), ref, s)
        assert ok, f"call {call} after the timeout: rel_fro={rel:.2e} worst={worst:.2e}"
    h.free()
