"""Failure handling on the GPU, without faulting it.

* A bounded device wait that runs out: the readers of t = X A_cat are made to wait for
  one part more than is ever added (SALR_FAIL_T_WAIT) with a short wait bound
  (SALR_WAIT_LIMIT_CYCLES).  The kernel must give up, report SALR_ERR_TIMEOUT through
  salr_sync_status, and the next ordinary call on the same handle must be correct.
* The bounds-checked debug build (compiled with SALR_CHECKS): every data-derived offset
  is tested and a failure is recorded instead of performed.  Small shapes of every
  kernel must run clean (status 0) and match the oracle.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
import salr_synth as synth
from gpu_util import assert_close, to_bits, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
salr = pytest.importorskip("sparse_rank_linear_b200")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SALR_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def lib():
    from sparse_rank_linear_b200.build import build
    build()
    assert torch.cuda.is_available()
    return salr.load_library()


def test_t_wait_runs_out_then_next_call_is_correct(monkeypatch):
    wl = synth.WORKLOADS["q_proj"]
    w, x, ad = synth.weight(wl), synth.activations(wl, 16), synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(np.concatenate([a for a, _ in ad], axis=1))
    B = to_dev(np.concatenate([b for _, b in ad], axis=0))
    X = to_dev(x)
    monkeypatch.setenv("SALR_WAIT_LIMIT_CYCLES", "400000")  # ~0.2 ms per wait
    monkeypatch.setenv("SALR_FAIL_T_WAIT", "1")
    salr.linear(X, h, A, B)
    assert h.sync_status() == SALR_ERR_TIMEOUT
    monkeypatch.delenv("SALR_FAIL_T_WAIT")
    monkeypatch.delenv("SALR_WAIT_LIMIT_CYCLES")  # back to the default bound (~1 s)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ystar, s = oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad)
    for call in range(2):
        Y = salr.linear(X, h, A, B)
        assert h.sync_status() == 0
        assert_close(to_bits(Y), ystar, s, f"after the timeout, call {call}")
    h.free()


CHECKED_RUN = r"""
import sys
sys.path.insert(0, {root!r})
sys.path.insert(0, {tests!r})
import numpy as np, torch
import oracle, salr_synth as synth
import sparse_rank_linear_b200 as salr
from gpu_util import to_bits, to_dev
cases = [("tiny", 256, 256, (8,), 16), ("q", 1024, 1024, (64, 16), 16), ("q1", 1024, 1024, (8,), 1),
         ("mid", 768, 1088, (72,), 300), ("dense", 1280, 512, (16,), 600), ("nor", 384, 320, (), 40)]
for name, N, K, ranks, M in cases:
    wl = synth.Workload(name, N, K, ranks, (M,))
    w, x, ad = synth.weight(wl), synth.activations(wl, M), synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    d = to_bits(h.decode())
    st = h.sync_status()
    assert st == 0 and (d == wp).all(), (name, "decode", st, int((d != wp).sum()))
    A = to_dev(np.concatenate([a for a, _ in ad], axis=1)) if ad else None
    B = to_dev(np.concatenate([b for _, b in ad], axis=0)) if ad else None
    Y = salr.linear(to_dev(x), h, A, B)
    st = h.sync_status()
    assert st == 0, (name, "linear", st)
    ok, rel, worst = oracle.check_tolerance(to_bits(Y), oracle.linear(x, wp, ad),
                                            oracle.abs_bound(x, wp, ad))
    assert ok, (name, rel, worst)
    h.free()
print("checked build clean")
"""


def test_checked_build_runs_small_shapes_clean():
    from sparse_rank_linear_b200.build import build
    path = build(checks=True)
    env = dict(os.environ, SALR_LIBRARY=path)
    code = CHECKED_RUN.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-3000:]
    assert "checked build clean" in out.stdout
