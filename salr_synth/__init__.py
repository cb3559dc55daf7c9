"""Seeded synthetic inputs for the SALR linear layer (weights, activations, adapters).

This module is the one piece shared by the fp64 oracle and the CUDA path's tests and
benchmark.  It draws random numbers and rounds them to bf16; it holds none of the
method's arithmetic (no pruning, encoding or contraction).

Generator definition (counter-based, so any element can be drawn on its own):

* ``mix64`` is the SplitMix64 output function (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): ``z ^= z>>30; z *= 0xbf58476d1ce4e5b9;
  z ^= z>>27; z *= 0x94d049bb133111eb; z ^= z>>31`` on 64-bit words.
* A tensor's stream key is ``mix64(seed * 0x9E3779B97F4A7C15 + tensor_id)``.
* Draw ``j`` of element ``i`` (flat row-major index) is ``mix64(key + (D*i + j + 1) *
  0x9E3779B97F4A7C15)`` with ``D`` draws per element.  A draw becomes a uniform from
  its top 53 bits: ``u = ((d >> 11) + 0.5) / 2**53`` in (0, 1).
* Normal: Box-Muller, ``z = sqrt(-2 ln u1) * cos(2 pi u2)`` in fp64.
* Student-t with nu = 4: ``z / sqrt(v / 4)`` where ``v = -2 ln(u3 u4)`` is a chi-square
  variable with 4 degrees of freedom.
* The fp64 sample times the scale is rounded to fp32 (round to nearest even) and then
  to bf16 (round to nearest even); tensors are returned as uint16 bf16 bit patterns.

Tensor ids: W = 1, X = 2, adapter i: A = 10 + i, B = 20 + i.  The workloads are the
LLM projection shapes the SALR pages evaluate on (Llama-family q/up/down projections),
with the value distributions stated per workload below.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 20

TID_W = 1
TID_X = 2


def tid_a(i: int) -> int:
    return 10 + i


def tid_b(i: int) -> int:
    return 20 + i


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.array([np.uint64(seed) * GOLDEN + np.uint64(tensor_id)], dtype=np.uint64)
    return mix64(base)[0]


def _uniforms(key: np.uint64, idx: np.ndarray, draws: int, j: int) -> np.ndarray:
    ctr = idx * np.uint64(draws) + np.uint64(j + 1)
    d = mix64(key + ctr * GOLDEN)
    return ((d >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the bit patterns."""
    b = x32.astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _draw_chunk(kind: str, key: np.uint64, scale: float, lo: int, hi: int) -> np.ndarray:
    idx = np.arange(lo, hi, dtype=np.uint64)
    if kind == "normal":
        u1 = _uniforms(key, idx, 2, 0)
        u2 = _uniforms(key, idx, 2, 1)
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    elif kind == "student_t4":
        u1 = _uniforms(key, idx, 4, 0)
        u2 = _uniforms(key, idx, 4, 1)
        u3 = _uniforms(key, idx, 4, 2)
        u4 = _uniforms(key, idx, 4, 3)
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        v = -2.0 * np.log(u3 * u4)
        z = z / np.sqrt(v / 4.0)
    else:
        raise ValueError(kind)
    return f32_to_bf16_bits((z * scale).astype(np.float32))


def draw(kind: str, seed: int, tensor_id: int, shape, scale: float,
         rows: np.ndarray | None = None) -> np.ndarray:
    """bf16 bits of a seeded tensor of ``shape`` (2-D, row-major).

    ``rows`` selects a subset of rows (drawn by their own counters), so a sampled
    check never needs the whole tensor.
    """
    nrows, ncols = int(shape[0]), int(shape[1])
    key = stream_key(seed, tensor_id)
    with np.errstate(over="ignore"):
        if rows is not None:
            rows = np.asarray(rows, dtype=np.int64)
            out = np.empty((len(rows), ncols), dtype=np.uint16)
            for j, r in enumerate(rows):
                out[j] = _draw_chunk(kind, key, scale, int(r) * ncols, int(r + 1) * ncols)
            return out
        total = nrows * ncols
        out = np.empty(total, dtype=np.uint16)
        spans = [(lo, min(lo + _CHUNK, total)) for lo in range(0, total, _CHUNK)]

        def work(span):
            lo, hi = span
            out[lo:hi] = _draw_chunk(kind, key, scale, lo, hi)

        if len(spans) > 2:
            with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
                list(ex.map(work, spans))
        else:
            for s in spans:
                work(s)
    return out.reshape(nrows, ncols)


@dataclass(frozen=True)
class Workload:
    """One evaluated layer shape: W is N x K (out x in), adapters of the listed ranks."""
    name: str
    N: int
    K: int
    ranks: tuple
    Ms: tuple
    w_kind: str = "normal"
    w_scale: float = 0.02
    ab_scale: float = 0.01
    sparsity: float = 0.5
    seed: int = 0

    @property
    def R(self) -> int:
        return int(sum(self.ranks))


WORKLOADS = {
    "tiny": Workload("tiny", 256, 256, (8,), (16,)),
    "q_proj": Workload("q_proj", 4096, 4096, (64, 16), (1, 16)),
    "up_proj": Workload("up_proj", 11008, 4096, (64, 16, 16), (2048,)),
    "down_proj": Workload("down_proj", 4096, 11008, (128,), (1, 128, 4096)),
    "large": Workload("large", 28672, 8192, (64, 32), (16, 8192), w_kind="student_t4"),
}


def weight(wl: Workload, rows=None) -> np.ndarray:
    return draw(wl.w_kind, wl.seed, TID_W, (wl.N, wl.K), wl.w_scale, rows)


def activations(wl: Workload, M: int, rows=None) -> np.ndarray:
    return draw("normal", wl.seed, TID_X, (M, wl.K), 1.0, rows)


def adapters(wl: Workload):
    """List of (A_i, B_i) bf16 bit arrays: A_i is K x r_i, B_i is r_i x N."""
    out = []
    for i, r in enumerate(wl.ranks):
        a = draw("normal", wl.seed, tid_a(i), (wl.K, r), wl.ab_scale)
        b = draw("normal", wl.seed, tid_b(i), (r, wl.N), wl.ab_scale)
        out.append((a, b))
    return out
