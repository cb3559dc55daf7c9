"""The serialised image of an encoded weight, laid out as include/salr.h describes it
(fixed header, offset table, blob) around the oracle's block format.  Test
infrastructure: the expected bytes of salr_save and hand-made inputs of salr_load."""
import math
import struct

import numpy as np

import oracle

HEADER = struct.Struct("<8sIIqqqqfIq")  # 64 bytes, no padding
MAGIC = b"SALRBLK1"


def image(w_bits: np.ndarray, sparsity: float) -> bytes:
    """Image of W pruned at ``sparsity`` (taken as the float32 the C ABI receives)."""
    s32 = float(np.float32(sparsity))
    n, k = w_bits.shape
    m = oracle.magnitude_mask(w_bits, s32)
    wp = oracle.prune(w_bits, m)
    offs, blob = oracle.encode_format(wp, m)
    keep = oracle.keep_count(k, s32)
    return pack(n, k, keep, n * keep, s32, offs, blob)


def pack(n, k, keep, nnz, sparsity, offs, blob, version=2, header_bytes=64, magic=MAGIC,
         zero=0) -> bytes:
    head = HEADER.pack(magic, version, header_bytes, n, k, keep, nnz, sparsity, zero,
                       len(blob))
    table = np.asarray(offs, dtype="<u4").tobytes()
    table += b"\x00" * ((-len(table)) % 16)
    return head + table + bytes(np.asarray(blob, dtype=np.uint8))


def split(img: bytes):
    """(header fields, offsets uint32 array, blob uint8 array) of an image."""
    f = HEADER.unpack_from(img, 0)
    n, k = f[3], f[4]
    nb = (n // 128) * (k // 64)
    table = 64 + math.ceil((nb + 1) * 4 / 16) * 16
    offs = np.frombuffer(img, dtype="<u4", count=nb + 1, offset=64).copy()
    blob = np.frombuffer(img, dtype=np.uint8, count=f[9], offset=table).copy()
    return f, offs, blob
