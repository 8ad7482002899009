"""Seeded stand-alone inputs for testing one stage at a time (tokens, field tokens).

Values are drawn from N(0, std) and rounded to the storage type, so both
implementations read identical numbers.  No arithmetic of the method lives here.
"""
from __future__ import annotations

import numpy as np

from .tables import f32_to_bf16_rne


def rand_matrix(seed: int, shape, std: float, dtype: str) -> np.ndarray:
    v = np.random.default_rng(seed).normal(0.0, std, size=shape).astype(np.float32)
    if dtype == "bf16":
        v = f32_to_bf16_rne(v.reshape(-1)).reshape(shape)
    return v
