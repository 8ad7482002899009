"""Decodes a user K/V cache from the layout documented in include/tr.h (test helper)."""
import numpy as np


def decode_kv(raw: np.ndarray, dtype: str, n_layer: int, L_u: int, D: int):
    """raw: uint8 bytes of the cache -> (K, V) float64 [n_layer, L_u, D] (fp32 model: fp32
    rows; bf16 model: fp16 core-matrix images)."""
    if dtype == "f32":
        a = raw[: n_layer * 2 * L_u * D * 4].view(np.float32).reshape(n_layer, 2, L_u, D).astype(np.float64)
        return a[:, 0], a[:, 1]
    Lp = (L_u + 15) // 16 * 16
    f = raw[: n_layer * 2 * Lp * D * 2].view(np.float16).reshape(n_layer, 2, Lp * D).astype(np.float64)
    K = np.zeros((n_layer, Lp, D))
    V = np.zeros((n_layer, Lp, D))
    j = np.arange(Lp)[:, None]
    d = np.arange(D)[None, :]
    kidx = ((d // 8) * (Lp // 8) + j // 8) * 64 + (j % 8) * 8 + d % 8
    vidx = ((j // 8) * (D // 8) + d // 8) * 64 + (d % 8) * 8 + j % 8
    for l in range(n_layer):
        K[l] = f[l, 0][kidx]
        V[l] = f[l, 1][vidx]
    return K[:, :L_u], V[:, :L_u], K[:, L_u:], V[:, L_u:]
