"""The no-allocation user side (tr_prefill_user_noalloc) against tr_prefill_user.

Some callers cannot allocate device memory when a request's user side runs: an open CUDA
stream capture, or a serving engine whose allocator owns all of the GPU.  The no-allocation
entry point keeps its scratch in a fixed device array instead of the library's cudaMalloc'd
workspace.  Here it is called through the C ABI twice in a row, with different inputs, and
each result is compared with the regular entry point's on the same inputs; a request larger
than the fixed array must be refused.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import datagen
from common import check_close
from kvdecode import decode_kv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from transformer_candidate_scoring_b200 import build
    build.build()
    assert torch.cuda.is_available()
    yield


def _kv(tr, m, dims, L_u, fn, U, domain):
    kv = torch.zeros(tr.kv_cache_bytes(m, L_u), dtype=torch.uint8, device="cuda")
    fn(m, torch.from_numpy(U).cuda(), L_u, domain, kv)
    torch.cuda.synchronize()
    return decode_kv(kv.cpu().numpy(), dims.dtype, dims.n_layer, L_u, dims.D)


@pytest.mark.parametrize("name,init", [("tiny", "paper"), ("128d5l", "wide")])
def test_noalloc_matches_regular_user_side_on_two_calls_in_a_row(name, init):
    import transformer_candidate_scoring_b200 as tr
    dims = datagen.WORKLOADS[name].dims
    P = datagen.make_params(dims, 8, init)
    m = tr.Model(dims, P)
    for call, (L_u, seed) in enumerate([(64 if dims.D == 128 else 8, 31), (37 if dims.D == 128 else 5, 32)]):
        U = datagen.rand_matrix(seed, (L_u, dims.D), 0.3 if init == "wide" else 0.01, "f32")
        ref = _kv(tr, m, dims, L_u, tr.prefill_user, U, 1)
        got = _kv(tr, m, dims, L_u, tr.prefill_user_noalloc, U, 1)
        for l in range(dims.n_layer):
            check_close(got[0][l], ref[0][l], dims.dtype, f"call {call} K layer {l}", kind="intermediate")
            check_close(got[1][l], ref[1][l], dims.dtype, f"call {call} V layer {l}", kind="intermediate")
        if dims.dtype == "bf16":
            assert np.all(got[2] == 0) and np.all(got[3] == 0)


def test_noalloc_refuses_requests_beyond_its_scratch():
    import transformer_candidate_scoring_b200 as tr
    from transformer_candidate_scoring_b200 import _lib as L
    dims = datagen.ModelDims(D=128, n_layer=1, n_head=8, ffn_hidden=512, n_target_fields=8,
                             comp_dims=(1024, 512, 256, 128), n_domains=2, dtype="bf16")
    m = tr.Model(dims, datagen.make_params(dims, 0))
    L_u = 256            # 256 * (6*128 + 512) * 4 bytes > TR_NOALLOC_SCRATCH_BYTES
    U = torch.zeros(L_u, 128, dtype=torch.float32, device="cuda")
    kv = torch.zeros(tr.kv_cache_bytes(m, L_u), dtype=torch.uint8, device="cuda")
    with pytest.raises(tr.TrError) as e:
        tr.prefill_user_noalloc(m, U, L_u, 0, kv)
    assert e.value.status == L.TR_ERR_INVALID_ARG and "scratch" in str(e.value)
    assert int(kv.abs().sum()) == 0
