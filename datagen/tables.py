"""Counter-based synthetic embedding tables.

Value of table ``t`` at element ``e = row * D + col`` for a given seed:

* 32-bit hashing with the MurmurHash3 finaliser ``fmix32`` (Appleby, MurmurHash3,
  public domain): ``a = fmix32(lo32(e) ^ fmix32(hi32(e) ^ base))`` and
  ``b = fmix32(a ^ 0x68E31DA4)`` with ``base = fmix32(seed * 0x9E3779B9 + t * 0x632BE5AB + 1)``.
* Irwin-Hall approximation of a normal: the four 16-bit halves of ``a`` and ``b`` are
  summed and centred, ``s = sum - 131070`` (an exact integer below 2^24),
* ``value = fp32(s) * fp32(0.02 / 37837.2...)`` -- one correctly rounded fp32 multiply,
  so std 0.02 -- then rounded to the table's storage type (bf16 by round-to-nearest-even).

Every step is either integer arithmetic or a single IEEE-754 operation, so the host
(numpy) and device (torch) versions below produce bit-identical tables.  The host
version evaluates only the rows a test needs, so no host copy of a 52M-row table is
ever made.  Multiplication is split into 16-bit halves so that no intermediate
exceeds 2^49 on either side.
"""
from __future__ import annotations

import numpy as np

M32 = 0xFFFFFFFF
_C1 = 0x85EBCA6B
_C2 = 0xC2B2AE35
_STD4 = float(np.sqrt((65536.0 ** 2 - 1.0) / 12.0) * 2.0)   # std of a sum of four U{0..65535}
SCALE = np.float32(0.02 / _STD4)


def _fmix32_int(h: int) -> int:
    h &= M32
    h ^= h >> 16
    h = (h * _C1) & M32
    h ^= h >> 13
    h = (h * _C2) & M32
    h ^= h >> 16
    return h


def table_base(seed: int, table: int) -> int:
    return _fmix32_int((seed * 0x9E3779B9 + table * 0x632BE5AB + 1) & M32)


# ----------------------------------------------------------------------------- numpy

def _mul32_np(h: np.ndarray, k: int) -> np.ndarray:
    lo = (h & 0xFFFF) * np.uint64(k)
    hi = ((h >> np.uint64(16)) * np.uint64(k)) & np.uint64(0xFFFF)
    return (lo + (hi << np.uint64(16))) & np.uint64(M32)


def _fmix32_np(h: np.ndarray) -> np.ndarray:
    h = h ^ (h >> np.uint64(16))
    h = _mul32_np(h, _C1)
    h = h ^ (h >> np.uint64(13))
    h = _mul32_np(h, _C2)
    h = h ^ (h >> np.uint64(16))
    return h


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32."""
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return (r.astype(np.uint32) << np.uint32(16)).view(np.float32)


def table_elements_host(seed: int, table: int, elems: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 values (exactly representable in ``dtype``) of the given flat element indices."""
    e = np.asarray(elems, dtype=np.uint64)
    base = np.uint64(table_base(seed, table))
    a = _fmix32_np((e & np.uint64(M32)) ^ _fmix32_np((e >> np.uint64(32)) ^ base))
    b = _fmix32_np(a ^ np.uint64(0x68E31DA4))
    s = ((a & np.uint64(0xFFFF)) + (a >> np.uint64(16)) + (b & np.uint64(0xFFFF))
         + (b >> np.uint64(16))).astype(np.int64) - 131070
    v = s.astype(np.float32) * SCALE
    if dtype == "bf16":
        v = f32_to_bf16_rne(v)
    return v


def table_rows_host(seed: int, table: int, rows: np.ndarray, D: int, dtype: str) -> np.ndarray:
    """Rows ``rows`` of table ``table`` as an fp32 array [len(rows), D]."""
    rows = np.asarray(rows, dtype=np.int64)
    elems = rows[:, None] * D + np.arange(D, dtype=np.int64)[None, :]
    return table_elements_host(seed, table, elems.reshape(-1), dtype).reshape(len(rows), D)


# ----------------------------------------------------------------------------- torch

def fill_table_device(out, seed: int, table: int, chunk: int = 1 << 25, start_elem: int = 0) -> None:
    """Fill a contiguous torch tensor (fp32 or bf16, any device) with the table values of
    flat elements start_elem, start_elem + 1, ... (start_elem = 0 fills a whole table)."""
    import torch

    flat = out.view(-1)
    n = flat.numel()
    base = table_base(seed, table)
    dev = out.device

    def mul32(h, k):
        lo = (h & 0xFFFF) * k
        hi = ((h >> 16) * k) & 0xFFFF
        return (lo + (hi << 16)) & M32

    def fmix(h):
        h = h ^ (h >> 16)
        h = mul32(h, _C1)
        h = h ^ (h >> 13)
        h = mul32(h, _C2)
        return h ^ (h >> 16)

    scale = torch.tensor(float(SCALE), dtype=torch.float32, device=dev)
    for s0 in range(0, n, chunk):
        s1 = min(n, s0 + chunk)
        e = torch.arange(start_elem + s0, start_elem + s1, dtype=torch.int64, device=dev)
        a = fmix((e & M32) ^ fmix((e >> 32) ^ base))
        del e
        b = fmix(a ^ 0x68E31DA4)
        s = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16) - 131070
        del a, b
        v = s.to(torch.float32) * scale
        flat[s0:s1] = v.to(out.dtype)
        del s, v
