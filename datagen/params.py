"""Seeded random-init parameters of a TransRetrieval backbone and target compressor.

Shapes follow TransRetrieval §3.3-§3.4: per layer Q/K/V/O projections (D x D), a ReLU
FFN D -> 2D -> D, Pre-LN LayerNorms, a learned domain embedding s_d per domain, a
3-layer target compressor with PReLU + LayerNorm between layers, and a linear score
head on a final LayerNorm.  Linear layers are stored as ``W [in, out]`` with ``y = x W + b``.

Init: matrices, biases, LayerNorm shifts, domain embeddings and the head ~ N(0, 0.02);
LayerNorm gains ~ 1 + N(0, 0.02); PReLU slopes ~ 0.25 + N(0, 0.02).  For the bf16 model
every parameter is rounded to bf16 (nearest, ties to even) so that both implementations
read exactly the same values.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .configs import ModelDims, Workload
from .tables import f32_to_bf16_rne

Params = Dict[str, np.ndarray]


def make_params(dims: ModelDims, seed: int, init: str = "paper") -> Params:
    """``init="paper"`` is the N(0, 0.02) recipe above.  ``init="wide"`` draws matrices
    from N(0, 1/fan_in), gains from U(0.5, 1.5), slopes from U(-0.5, 0.5) and the other
    vectors from N(0, 0.3): attention is then far from uniform and candidates differ
    strongly, which makes kernel-level comparisons sharper."""
    rng = np.random.default_rng(np.random.SeedSequence(seed).spawn(4)[0])
    D, H = dims.D, dims.ffn_hidden
    P: Params = {}

    def nrm(*shape):
        return rng.normal(0.0, 0.02, size=shape)

    P["domain_emb"] = nrm(dims.n_domains, D)
    for l in range(dims.n_layer):
        p = f"l{l}."
        P[p + "ln1_g"] = 1.0 + nrm(D)
        P[p + "ln1_b"] = nrm(D)
        for m in "qkvo":
            P[p + "W" + m] = nrm(D, D)
            P[p + "b" + m] = nrm(D)
        P[p + "ln2_g"] = 1.0 + nrm(D)
        P[p + "ln2_b"] = nrm(D)
        P[p + "W1"] = nrm(D, H)
        P[p + "b1"] = nrm(H)
        P[p + "W2"] = nrm(H, D)
        P[p + "b2"] = nrm(D)
    P["lnf_g"] = 1.0 + nrm(D)
    P["lnf_b"] = nrm(D)
    P["w_head"] = nrm(D)
    P["b_head"] = nrm(1)
    c = dims.comp_dims
    for i in range(3):
        P[f"c{i}.W"] = nrm(c[i], c[i + 1])
        P[f"c{i}.b"] = nrm(c[i + 1])
        if i < 2:
            P[f"c{i}.prelu"] = 0.25 + nrm(c[i + 1])
            P[f"c{i}.ln_g"] = 1.0 + nrm(c[i + 1])
            P[f"c{i}.ln_b"] = nrm(c[i + 1])
    if init == "wide":
        wr = np.random.default_rng(seed + 7919)
        for k, v in P.items():
            if v.ndim == 2 and k != "domain_emb":
                P[k] = wr.normal(0.0, 1.0 / np.sqrt(v.shape[0]), size=v.shape)
            elif k.endswith("_g"):
                P[k] = wr.uniform(0.5, 1.5, size=v.shape)
            elif k.endswith("prelu"):
                P[k] = wr.uniform(-0.5, 0.5, size=v.shape)
            else:
                P[k] = wr.normal(0.0, 0.3, size=v.shape)
    elif init != "paper":
        raise ValueError(init)
    for k in P:
        v = P[k].astype(np.float32)
        P[k] = f32_to_bf16_rne(v).reshape(v.shape) if dims.dtype == "bf16" else v
    return P


def workload_params(w: Workload) -> Params:
    return make_params(w.dims, w.seed)
