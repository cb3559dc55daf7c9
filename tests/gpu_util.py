"""Helpers shared by the GPU tests: bf16 bit arrays <-> torch tensors, and the oracle
comparison used as the acceptance test."""
import numpy as np

import oracle
from salr_synth import bf16_bits_to_f64


def to_dev(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_close(y_bits, ystar, s, what=""):
    ok, rel, worst = oracle.check_tolerance(y_bits, ystar, s)
    assert ok, f"{what}: rel_fro={rel:.3e} (tol 4e-3), worst elem ratio={worst:.3e} (tol 1e-2)"
    return rel, worst
