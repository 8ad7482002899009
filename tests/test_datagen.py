"""Seeded input generators: host and torch table values agree bit for bit; bags are
well-formed and reproducible."""
import numpy as np
import torch

import datagen
from datagen import tables


def test_table_host_and_torch_agree_bitwise():
    for dtype, tdt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        t = torch.empty(3000, 32, dtype=tdt)
        tables.fill_table_device(t, seed=5, table=3, chunk=20_000)
        host = tables.table_rows_host(5, 3, np.arange(3000), 32, dtype)
        assert np.array_equal(t.float().numpy().view(np.uint32), host.view(np.uint32))


def test_table_rows_beyond_2_32_elements():
    rows = np.array([33_554_432, 40_000_000, 51_999_999])      # flat index > 2^32 at D = 128
    host = tables.table_rows_host(4, 16, rows, 128, "bf16")
    for i, r in enumerate(rows):
        t = torch.empty(128, dtype=torch.bfloat16)
        tables.fill_table_device(t, 4, 16, start_elem=int(r) * 128)
        assert np.array_equal(t.float().numpy().view(np.uint32), host[i].view(np.uint32))


def test_table_value_distribution():
    v = tables.table_elements_host(0, 0, np.arange(200_000), "f32")
    assert abs(v.mean()) < 2e-4 and abs(v.std() - 0.02) < 2e-4
    assert np.array_equal(tables.f32_to_bf16_rne(np.array([1.0 + 2 ** -8], np.float32)),
                          np.array([1.0], np.float32))          # tie to even
    assert np.array_equal(tables.f32_to_bf16_rne(np.array([1.0 + 3 * 2 ** -8], np.float32)),
                          np.array([1.0 + 2 ** -6], np.float32))


def test_bags_well_formed_and_reproducible():
    w = datagen.WORKLOADS["packed"].with_(n_cand_per_request=50)
    a = datagen.make_requests(w)
    b = datagen.make_requests(w)
    assert len(a) == 16
    for ra, rb in zip(a, b):
        assert 16 <= ra.L_u <= 128 and ra.user.n_bags == ra.L_u
        assert np.array_equal(ra.target.keys, rb.target.keys)
        assert ra.target.n_bags == 50 * 8
        nf = np.diff(ra.target.offsets)
        assert nf.min() >= 1 and nf.max() <= 8
        assert ra.user.keys.max() < w.user_rows and ra.target.keys.min() >= 0
        assert np.all((ra.target.weights >= 0.1) & (ra.target.weights < 1.0))


def test_params_bf16_representable():
    P = datagen.make_params(datagen.configs.DIMS_64D3L, 1)
    for v in P.values():
        assert np.array_equal(tables.f32_to_bf16_rne(v.reshape(-1)), v.reshape(-1))
