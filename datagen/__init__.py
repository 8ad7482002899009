"""Seeded synthetic inputs shared by the oracle-side tests and the GPU path.

Holds workload sizes, parameter init, bag generation and the counter-based table
values, and nothing of the scoring arithmetic itself.  Table numbering for the value
hash: user tables are 0 .. user_tables-1, target tables follow them.
"""
from __future__ import annotations

import numpy as np

from .configs import WORKLOADS, ModelDims, Workload, scaled
from .bags import Bags, Request, make_requests, make_target_bags, scale_weights
from .params import Params, make_params, workload_params
from .tables import fill_table_device, table_rows_host, f32_to_bf16_rne
from .stage_inputs import rand_matrix


def user_table_id(w: Workload, t: int) -> int:
    return t


def target_table_id(w: Workload, t: int) -> int:
    return w.user_tables + t


def compact_rows(w: Workload, bags: Bags, side: str):
    """Touched rows of a bag set as one compact table plus keys remapped into it.

    Returns (rows fp32 [U, D], compact_keys int64 [nnz]).  Only the rows the bags read
    are evaluated, so this works for tables of any size.
    """
    D = w.dims.D
    tab_of_key = np.repeat(bags.bag_table.astype(np.int64), np.diff(bags.offsets))
    tid = np.array([user_table_id(w, t) if side == "user" else target_table_id(w, t)
                    for t in range(w.user_tables if side == "user" else len(w.target_rows))],
                   dtype=np.int64)[tab_of_key]
    pair = tid * (1 << 32) + bags.keys.astype(np.int64)
    uniq, inv = np.unique(pair, return_inverse=True)
    rows = np.empty((len(uniq), D), dtype=np.float32)
    ut = uniq >> 32
    ur = uniq & 0xFFFFFFFF
    for t in np.unique(ut):
        sel = ut == t
        rows[sel] = table_rows_host(w.seed, int(t), ur[sel], D, w.dims.dtype)
    return rows, inv.astype(np.int64)


__all__ = [
    "WORKLOADS", "ModelDims", "Workload", "scaled", "Bags", "Request", "make_requests", "make_target_bags",
    "scale_weights", "Params", "make_params", "workload_params", "fill_table_device",
    "table_rows_host", "f32_to_bf16_rne", "rand_matrix", "user_table_id", "target_table_id", "compact_rows",
]
