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
        "version": pk(version=1),  # row-major value order, refused
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


# ---------------------------------------------------------------- launch plan (host logic)
def _plan(N, K, M, R=0, sms=148):
    return binding.plan(N, K, M, R, sms)


def test_linear_plan_of_the_workloads(lib):
    # hand-derived: tiles = N/128 x ceil(M / token tile); with at least as many tiles as
    # SMs the full rounds stay whole and the rem left over are split in s parts, s
    # minimising ceil(rem s / 148) / s
    q16 = _plan(4096, 4096, 16, 80)
    assert (q16["path"], q16["kernels"], q16["token_tile"], q16["units"], q16["grid"]) == \
        (0, 1, 16, 32 * 64, 148)
    assert _plan(256, 256, 16, 8)["grid"] == 8  # tiny: 2 x 4 blocks
    d128 = _plan(4096, 11008, 128, 128)  # 32 tiles < 148 SMs: each split in 148 // 32 = 4
    assert (d128["path"], d128["kernels"], d128["tiles"], d128["whole_tiles"], d128["splits"],
            d128["units"], d128["grid"]) == (1, 2, 32, 0, 4, 128, 128)
    assert d128["split_sum_bytes"] == 32 * 128 * 128 * 4
    assert d128["dense_scratch_bytes"] == 0
    # dense path.  256-row tiles only from 8 full rounds of them (up_proj and down_proj
    # have fewer: 344 and 256 tiles of 256 rows on 148 SMs), so 128-row tiles here
    up = _plan(11008, 4096, 2048, 96)  # 688 tiles = 4 x 148 + 96; 96 x 3 = 288 -> 2 rounds of 1/3
    assert (up["path"], up["kernels"], up["token_tile"], up["tile_rows"], up["tiles"],
            up["whole_tiles"], up["splits"], up["units"]) == (2, 3, 256, 128, 688, 592, 3, 880)
    assert up["split_sum_bytes"] == 96 * 128 * 256 * 4
    assert up["dense_scratch_bytes"] == 11008 * 4096 * 2
    # X of 16 MB stays in L2: token tile first
    assert up["group_rows"] == 0
    dn = _plan(4096, 11008, 4096, 128)  # 512 = 3 x 148 + 68; 68 x 2 = 136 -> 1 round of 1/2
    assert (dn["tile_rows"], dn["tiles"], dn["whole_tiles"], dn["splits"], dn["units"]) == \
        (128, 512, 444, 2, 580)
    # X of 90 MB: groups of round(sqrt(148 x 5.6 MB / 2.8 MB)) = 17 row tiles
    assert dn["group_rows"] == 17
    # 24 full rounds of 256-row tiles, and the busiest CTA gets no more 128-row block steps
    # (2 x (24 x 128 + 32)) than with 128-row tiles (48 x 128 + 2 x 32)
    lg = _plan(28672, 8192, 8192, 96)  # 3584 = 24 x 148 + 32; 32 x 4 = 128 -> 1 round of 1/4
    assert (lg["tile_rows"], lg["tiles"], lg["whole_tiles"], lg["splits"]) == (256, 3584, 3552, 4)
    # X of 134 MB, 256-row tiles as large as its token tiles: groups of round(sqrt(148)) = 12
    assert lg["group_rows"] == 12
    # 256-row tiles would leave up_proj M = 512 at 86 tiles on 148 SMs: 128-row tiles
    u512 = _plan(11008, 4096, 512)
    assert (u512["tile_rows"], u512["tiles"], u512["whole_tiles"], u512["splits"]) == (128, 172, 148, 6)
    # N not a multiple of 256, and the fused path, keep 128-row tiles
    assert _plan(384, 256, 600)["tile_rows"] == 128
    assert _plan(28672, 8192, 128, 96)["tile_rows"] == 128
    l128 = _plan(28672, 8192, 128, 96)  # 224 = 148 + 76; 76 x 7 = 532 -> 4 rounds of 1/7
    assert (l128["path"], l128["whole_tiles"], l128["splits"], l128["units"]) == (1, 148, 7, 680)
    u256 = _plan(11008, 4096, 256, 96)  # 86 tiles, 148 // 86 = 1: nothing split
    assert (u256["tiles"], u256["whole_tiles"], u256["splits"], u256["grid"]) == (86, 86, 1, 86)
    assert u256["split_sum_bytes"] == 0
    # no adapter: no t kernel
    assert _plan(11008, 4096, 2048, 0)["kernels"] == 2
    assert _plan(4096, 11008, 128, 0)["kernels"] == 1
    # whole rounds only: nothing split
    full = _plan(128 * 148, 4096, 256)
    assert (full["tiles"], full["whole_tiles"], full["splits"]) == (148, 148, 1)


def _makespan(p, KB):
    """Largest number of K blocks one CTA of the persistent layer kernel multiplies, with
    CTA c taking units c, c + grid, ... and the split units first."""
    s, tiles, whole = p["splits"], p["tiles"], p["whole_tiles"]
    nsu = (tiles - whole) * s if s > 1 else 0
    load = [0] * p["grid"]
    for u in range(p["units"]):
        if u < nsu:
            i = u % s
            blocks = (i + 1) * KB // s - i * KB // s
        else:
            blocks = KB
        load[u % p["grid"]] += blocks
    return max(load)


@pytest.mark.parametrize("sms", [148, 132, 64])
def test_linear_plan_split_never_lengthens_a_cta(lib, sms):
    rng = np.random.default_rng(7)
    for _ in range(150):
        RT = int(rng.integers(1, 400))
        KB = int(rng.integers(1, 200))
        M = int(rng.integers(65, 20000))
        p = _plan(128 * RT, 64 * KB, M, 0, sms)
        tiles = p["tiles"]
        assert p["tile_rows"] in (128, 256)
        if p["tile_rows"] == 256:
            assert p["path"] == 2 and p["token_tile"] == 256 and RT % 2 == 0
        assert tiles == 128 * RT // p["tile_rows"] * -(-M // p["token_tile"])
        s = p["splits"]
        assert p["units"] == p["whole_tiles"] + (tiles - p["whole_tiles"]) * s
        assert p["grid"] == min(p["units"], sms)
        if s > 1:
            if tiles >= sms:
                # only the last, partial round is split, into at most 8 parts of >= 4 blocks
                assert p["whole_tiles"] == tiles // sms * sms < tiles
                assert s <= 8 and KB // s >= 4
            else:
                assert p["whole_tiles"] == 0 and s == min(KB, sms // tiles)
        else:
            assert p["whole_tiles"] == tiles
        # against taking every tile whole: never longer, and shorter when s > 1
        whole = {"splits": 1, "tiles": tiles, "whole_tiles": tiles, "units": tiles,
                 "grid": min(tiles, sms)}
        assert _makespan(p, KB) <= _makespan(whole, KB)
        # a CTA takes tiles // sms whole tiles and at most ceil(rem s / sms) parts of at
        # most ceil(KB / s) blocks
        if s > 1 and tiles >= sms:
            rem = tiles - p["whole_tiles"]
            assert _makespan(p, KB) <= tiles // sms * KB + -(-rem * s // sms) * -(-KB // s)
        if s > 1:
            assert _makespan(p, KB) < _makespan(whole, KB)


def test_linear_plan_rejects_bad_arguments(lib):
    out = binding.SalrPlan()
    f = lib.salr_linear_plan
    assert f(4096, 4096, 0, 0, 148, ctypes.byref(out)) == 1      # M < 1
    assert f(4096, 4096, 16, -8, 148, ctypes.byref(out)) == 1    # R < 0
    assert f(4096, 4096, 16, 0, -1, ctypes.byref(out)) == 1      # sms < 0
    assert f(4096, 4096, 16, 0, 148, None) == 1                  # no output
    assert f(4096, 4096, 16, 12, 148, ctypes.byref(out)) == 2    # R % 8
    assert f(4096, 4096, 16, 136, 148, ctypes.byref(out)) == 2   # R > 128
    assert f(4000, 4096, 16, 0, 148, ctypes.byref(out)) == 2     # N % 128
    assert f(4096, 4000, 16, 0, 148, ctypes.byref(out)) == 2     # K % 64
    assert f(4096, 64 * 513, 512, 0, 148, ctypes.byref(out)) == 2  # K past the layer kernels
    assert f(4096, 4096, (1 << 24) + 1, 0, 148, ctypes.byref(out)) == 2
    # an output of more than 2^27 tiles of 128 x 128 (work-unit counts stay 32-bit)
    assert f(1 << 22, 64, 1 << 24, 0, 148, ctypes.byref(out)) == 2
    assert f(1 << 16, 64, 1 << 24, 0, 148, ctypes.byref(out)) == 0


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "salr.h"

int main(void) {
  salr_plan p;
  int rc = salr_linear_plan(11008, 4096, 2048, 96, 148, &p);
  if (rc != SALR_OK) { printf("plan %d\n", rc); return 1; }
  printf("%d %d %d %d %d %d %d %lld\n", p.path, p.kernels, p.tile_rows, p.tiles, p.whole_tiles,
         p.splits, p.units, (long long)p.dense_scratch_bytes);
  if (strcmp(salr_status_string(SALR_ERR_UNSUPPORTED), "SALR_ERR_UNSUPPORTED") != 0) return 2;
  if (salr_free(NULL) != SALR_ERR_INVALID) return 3;
  return 0;
}
"""


def test_header_is_plain_c_and_links_from_a_c_program(lib, tmp_path):
    # the boundary is a C ABI: the header compiles as C99 and a C program links the
    # library and calls the host-only entry points (no GPU needed)
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), LIB, f"-Wl,-rpath,{os.path.dirname(LIB)}"],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.split() == ["2", "3", "128", "688", "592", "3", "880", str(11008 * 4096 * 2)]
