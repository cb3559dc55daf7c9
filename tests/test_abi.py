"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
entry point include/salr.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

from sparse_rank_linear_b200 import binding
from sparse_rank_linear_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "salr.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SALR_API\s+[\w\s\*]+?\b(salr_\w+)\s*\(", text)))


def test_header_declares_the_three_calls_and_helpers():
    names = declared_functions()
    for must in ("salr_encode", "salr_decode", "salr_linear", "salr_free"):
        assert must in names
    assert set(names) == set(binding.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (salr_\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing but the C ABI is exported
    assert exported == set(declared_functions())


def test_status_strings(lib):
    assert binding.status_string(0) == "SALR_OK"
    assert binding.status_string(1) == "SALR_ERR_INVALID"
    assert binding.status_string(5) == "SALR_ERR_TIMEOUT"
    assert binding.status_string(99) == "SALR_ERR_UNKNOWN"


def test_bad_arguments_rejected_on_host(lib):
    P = ctypes.c_void_p
    h = P()
    fake = P(0x10000)  # never dereferenced: every call below fails its checks first
    # encode: null W, null out, bad sparsity, bad shapes, misaligned W
    assert lib.salr_encode(P(0), 128, 64, 0.5, P(0), ctypes.byref(h)) == 1
    assert lib.salr_encode(fake, 128, 64, 0.5, P(0), None) == 1
    for s in (-0.1, 1.0, float("nan")):
        assert lib.salr_encode(fake, 128, 64, s, P(0), ctypes.byref(h)) == 1
    assert lib.salr_encode(fake, 100, 64, 0.5, P(0), ctypes.byref(h)) == 2
    assert lib.salr_encode(fake, 128, 96, 0.5, P(0), ctypes.byref(h)) == 2
    assert lib.salr_encode(fake, 128, 64 * 513, 0.5, P(0), ctypes.byref(h)) == 2
    assert lib.salr_encode(P(0x10002), 128, 64, 0.5, P(0), ctypes.byref(h)) == 2
    assert h.value is None
    # unknown handles are rejected without being dereferenced
    for bad in (P(0), fake):
        assert lib.salr_free(bad) == 1
        assert lib.salr_decode(bad, fake, P(0)) == 1
        assert lib.salr_linear(fake, 1, bad, P(0), P(0), 0, fake, P(0)) == 1
        assert lib.salr_linear_host(fake, 1, bad, P(0), P(0), 0, fake, P(0)) == 1
        assert lib.salr_info(bad, None, None, None, None) == 1
        assert lib.salr_format_view(bad, None, None, None, None) == 1
        assert lib.salr_sync_status(bad, P(0)) == 1
        n = ctypes.c_int64()
        assert lib.salr_save_size(bad, ctypes.byref(n)) == 1
        assert lib.salr_save(bad, fake, 1 << 20, P(0)) == 1
        assert lib.salr_residual_adapter(fake, bad, 8, fake, 16, 2, fake, fake, None, P(0)) == 1


def test_fake_oom_reported(lib):
    # the allocation-failure path, forced on the host: no GPU work is queued
    code = ("import ctypes; from sparse_rank_linear_b200 import binding as b; "
            "l=b.load_library(); h=ctypes.c_void_p(); "
            "print(l.salr_encode(ctypes.c_void_p(0x10000), 128, 64, 0.5, ctypes.c_void_p(0), "
            "ctypes.byref(h)))")
    env = dict(os.environ, SALR_FAKE_OOM="1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=ROOT, timeout=120)
    assert out.stdout.strip() == "4", out.stderr


def test_missing_library_fails_loudly(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(RuntimeError, match="not built"):
            binding.load_library(str(tmp_path / "absent.so"))
    finally:
        binding._lib = saved


def test_load_rejects_bad_images_on_host(lib):
    # every image below fails a check made on the host before any CUDA call
    import image_util as iu
    import salr_synth as synth
    P = ctypes.c_void_p
    w = synth.weight(synth.WORKLOADS["tiny"])
    good = iu.image(w, 0.5)
    f, offs, blob = iu.split(good)
    n, k, keep, nnz, s = f[3], f[4], f[5], f[6], f[7]

    def load(img):
        h = P()
        buf = ctypes.create_string_buffer(img, len(img))
        rc = lib.salr_load(ctypes.cast(buf, P), len(img), P(0), ctypes.byref(h))
        assert h.value is None
        return rc

    def pk(**kw):
        a = dict(n=n, k=k, keep=keep, nnz=nnz, sparsity=s, offs=offs, blob=blob)
        a.update(kw)
        return iu.pack(**a)

    o = offs.astype(np.int64)
    bad = {
        "short": good[:63],
        "magic": pk(magic=b"SALRBLK2"),
        "version": pk(version=2),
        "header size": pk(header_bytes=72),
        "reserved word": pk(zero=1),
        "keep": pk(keep=keep + 1, nnz=n * (keep + 1)),
        "nnz": pk(nnz=nnz - 1),
        "sparsity nan": pk(sparsity=float("nan")),
        "sparsity one": pk(sparsity=1.0),
        "first offset": pk(offs=np.concatenate([[1], o[1:]])),
        "block under a bitmap": pk(offs=np.concatenate([[0, 63], o[2:]])),
        "block over a dense block": pk(offs=np.concatenate([[0], o[1:] + 1025])),
        "offsets fall": pk(offs=np.concatenate([[0, o[2], o[1]], o[3:]])),
        "end short of the blob": pk(blob=np.concatenate([blob, np.zeros(16, np.uint8)])),
        "truncated": good[:-1],
    }
    for name, img in bad.items():
        assert load(img) == 1, name
    # the blob size field must be a multiple of 16 and fit the buffer
    odd = bytearray(good)
    odd[56:64] = (len(blob) + 8).to_bytes(8, "little")
    assert load(bytes(odd)) == 1
    # shapes outside the rules are unsupported, as for salr_encode
    assert load(pk(n=100)) == 2
    assert load(pk(k=96)) == 2
