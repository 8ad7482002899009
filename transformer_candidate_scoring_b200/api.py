"""Python binding of libtr: the C ABI's calls under the same names.

Argument marshalling only: torch tensors are passed by device pointer on the current
CUDA stream; every step of the computation runs in libtr's kernels.
"""
from __future__ import annotations

import ctypes as C
from typing import Dict, Sequence

import numpy as np
import torch

from . import _lib as L


class TrError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libtr status {status}: {msg}")
        self.status = status


def _check(status: int) -> None:
    if status != L.TR_OK:
        raise TrError(status, L.load().tr_last_error().decode())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: torch.Tensor | None) -> C.c_void_p:
    if t is None:
        return C.c_void_p(0)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def dtype_code(dt) -> int:
    if dt in (torch.float32, "f32"):
        return L.TR_F32
    if dt in (torch.bfloat16, "bf16"):
        return L.TR_BF16
    raise ValueError(f"unsupported dtype {dt}")


def torch_dtype(code_or_name) -> torch.dtype:
    return torch.bfloat16 if code_or_name in (L.TR_BF16, "bf16") else torch.float32


def kernel_launches() -> int:
    """Kernels libtr has launched so far in this process."""
    return int(L.load().tr_kernel_launches())


def version() -> str:
    return L.load().tr_version().decode()


class Model:
    """A model handle (tr_model_create / tr_model_destroy) built from named fp32 arrays.

    ``params`` uses the names of ``datagen.params``: domain_emb, l{i}.{ln1_g, ..., b2},
    lnf_g, lnf_b, w_head, b_head, c{i}.{W, b, prelu, ln_g, ln_b}.
    """

    def __init__(self, dims, params: Dict[str, np.ndarray]):
        lib = L.load()
        self.dims = dims
        keep = []

        def fp(name):
            a = np.ascontiguousarray(params[name], dtype=np.float32)
            keep.append(a)
            return a.ctypes.data_as(L._fp)

        desc = L.ModelDesc(dims.D, dims.n_layer, dims.n_head, dims.ffn_hidden, dims.n_target_fields,
                           (C.c_int * 4)(*dims.comp_dims), dims.n_domains, dtype_code(dims.dtype))
        layers = (L.LayerWeights * dims.n_layer)()
        for l in range(dims.n_layer):
            for f, _ in L.LayerWeights._fields_:
                setattr(layers[l], f, fp(f"l{l}.{f}"))
        w = L.ModelWeights()
        w.domain_emb = fp("domain_emb")
        w.layers = layers
        w.lnf_g, w.lnf_b, w.w_head = fp("lnf_g"), fp("lnf_b"), fp("w_head")
        w.b_head = float(np.asarray(params["b_head"]).reshape(-1)[0])
        for i in range(3):
            w.comp_W[i] = fp(f"c{i}.W")
            w.comp_b[i] = fp(f"c{i}.b")
        for i in range(2):
            w.comp_prelu[i] = fp(f"c{i}.prelu")
            w.comp_ln_g[i] = fp(f"c{i}.ln_g")
            w.comp_ln_b[i] = fp(f"c{i}.ln_b")
        h = C.c_void_p()
        _check(lib.tr_model_create(C.byref(desc), C.byref(w), C.byref(h)))
        self._h = h

    @property
    def handle(self) -> C.c_void_p:
        return self._h

    def close(self) -> None:
        if getattr(self, "_h", None) and self._h.value:
            L.load().tr_model_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


AGG_MODES = {"mean": 0, "sum": 1, "max": 2}
AGG_POST_LN = 0x100


def aggregate(tables: Sequence[torch.Tensor], bag_table: torch.Tensor, offsets: torch.Tensor,
              keys: torch.Tensor, weights: torch.Tensor, out: torch.Tensor, stream=None, mode: str = "mean",
              post_ln: bool = False) -> torch.Tensor:
    """tr_aggregate (mode "mean", no LayerNorm) or tr_aggregate_ex: one token per bag into
    out [n_bags, D]."""
    n = len(tables)
    arr = (L.Table * max(n, 1))()
    for i, t in enumerate(tables):
        arr[i] = L.Table(t.data_ptr(), t.shape[0], dtype_code(t.dtype))
    D = out.shape[-1]
    n_bags = offsets.numel() - 1
    if mode == "mean" and not post_ln:
        _check(L.load().tr_aggregate(arr, n, _ptr(bag_table), _ptr(offsets), _ptr(keys), _ptr(weights),
                                     n_bags, D, dtype_code(out.dtype), _ptr(out), _stream(stream)))
    else:
        code = AGG_MODES[mode] | (AGG_POST_LN if post_ln else 0)
        _check(L.load().tr_aggregate_ex(arr, n, _ptr(bag_table), _ptr(offsets), _ptr(keys), _ptr(weights),
                                        n_bags, D, dtype_code(out.dtype), code, _ptr(out), _stream(stream)))
    return out


def kv_cache_bytes(model: Model, L_u: int) -> int:
    return int(L.load().tr_kv_cache_bytes(model.handle, L_u))


def prefill_user(model: Model, user_tokens: torch.Tensor, L_u: int, domain: int, kv: torch.Tensor,
                 stream=None) -> torch.Tensor:
    """tr_prefill_user: fp32 user tokens [L_u, D] -> this request's K/V cache."""
    _check(L.load().tr_prefill_user(model.handle, _ptr(user_tokens), L_u, domain, _ptr(kv), _stream(stream)))
    return kv


def prefill_users(model: Model, user_tokens: Sequence[torch.Tensor], L_u: Sequence[int], domain: Sequence[int],
                  kv: Sequence[torch.Tensor], stream=None) -> None:
    """tr_prefill_users: the user sides of R requests in one call (fp32 user tokens [L_u, D]
    of each request -> its K/V cache)."""
    R = len(L_u)
    ut = (C.c_void_p * R)(*[(t.data_ptr() if int(l) else 0) for t, l in zip(user_tokens, L_u)])
    kvp = (C.c_void_p * R)(*[(k.data_ptr() if int(l) else 0) for k, l in zip(kv, L_u)])
    lu = (C.c_int32 * R)(*[int(x) for x in L_u])
    dm = (C.c_int32 * R)(*[int(x) for x in domain])
    for t in list(user_tokens) + list(kv):
        if not t.is_cuda:
            raise ValueError("expected CUDA tensors")
    _check(L.load().tr_prefill_users(model.handle, ut, lu, dm, kvp, R, _stream(stream)))


def prefill_user_noalloc(model: Model, user_tokens: torch.Tensor, L_u: int, domain: int, kv: torch.Tensor,
                         stream=None) -> torch.Tensor:
    """tr_prefill_user_noalloc: the user side with no device allocation, for callers that
    cannot allocate (open stream capture, an engine that owns all device memory)."""
    _check(L.load().tr_prefill_user_noalloc(model.handle, _ptr(user_tokens), L_u, domain, _ptr(kv),
                                            _stream(stream)))
    return kv


def compress_targets(model: Model, x: torch.Tensor, tokens: torch.Tensor, stream=None) -> torch.Tensor:
    """tr_compress_targets: x [n, F*D] (model dtype) -> tokens [n, D] fp32."""
    if tokens.dtype != torch.float32:
        raise ValueError("compressed tokens are fp32")
    _check(L.load().tr_compress_targets(model.handle, _ptr(x), x.shape[0], _ptr(tokens), _stream(stream)))
    return tokens


def compress_target_bags(model: Model, tables: Sequence[torch.Tensor], bag_table: torch.Tensor,
                         offsets: torch.Tensor, keys: torch.Tensor, weights: torch.Tensor, tokens: torch.Tensor,
                         stream=None) -> torch.Tensor:
    """tr_compress_target_bags: the target side in one launch, n = tokens.shape[0]
    candidates whose F field bags are c*F .. c*F+F-1 -> tokens [n, D] fp32."""
    if tokens.dtype != torch.float32:
        raise ValueError("compressed tokens are fp32")
    n = len(tables)
    arr = (L.Table * max(n, 1))()
    for i, t in enumerate(tables):
        arr[i] = L.Table(t.data_ptr(), t.shape[0], dtype_code(t.dtype))
    _check(L.load().tr_compress_target_bags(model.handle, arr, n, _ptr(bag_table), _ptr(offsets), _ptr(keys),
                                            _ptr(weights), tokens.shape[0], _ptr(tokens), _stream(stream)))
    return tokens


def score_candidates(model: Model, tokens: torch.Tensor, req_offsets: Sequence[int], kv: Sequence[torch.Tensor],
                     L_u: Sequence[int], domain: Sequence[int], scores: torch.Tensor, stream=None) -> torch.Tensor:
    """tr_score_candidates over packed requests: tokens [n, D] fp32; scores [n] fp32."""
    if tokens.dtype != torch.float32:
        raise ValueError("candidate tokens are fp32")
    R = len(L_u)
    off = (C.c_int64 * (R + 1))(*[int(x) for x in req_offsets])
    kvp = (C.c_void_p * R)(*[(k.data_ptr() if k is not None and k.numel() else 0) for k in kv])
    lu = (C.c_int32 * R)(*[int(x) for x in L_u])
    dm = (C.c_int32 * R)(*[int(x) for x in domain])
    _check(L.load().tr_score_candidates(model.handle, _ptr(tokens), int(req_offsets[-1]), off, kvp, lu, dm, R,
                                        _ptr(scores), _stream(stream)))
    return scores


def score_candidates_uncompressed(model: Model, tokens: torch.Tensor, L_t: int, req_offsets: Sequence[int],
                                  kv: Sequence[torch.Tensor], L_u: Sequence[int], domain: Sequence[int],
                                  scores: torch.Tensor, stream=None) -> torch.Tensor:
    """tr_score_candidates_uncompressed: candidates of L_t target tokens each (tokens
    [n, L_t, D] or [n*L_t, D]); scores [n] fp32."""
    R = len(L_u)
    off = (C.c_int64 * (R + 1))(*[int(x) for x in req_offsets])
    kvp = (C.c_void_p * R)(*[(k.data_ptr() if k is not None and k.numel() else 0) for k in kv])
    lu = (C.c_int32 * R)(*[int(x) for x in L_u])
    dm = (C.c_int32 * R)(*[int(x) for x in domain])
    _check(L.load().tr_score_candidates_uncompressed(model.handle, _ptr(tokens), int(req_offsets[-1]), int(L_t), off,
                                                     kvp, lu, dm, R, _ptr(scores), _stream(stream)))
    return scores


def topk(scores: torch.Tensor, req_offsets: Sequence[int], k: int, out_idx: torch.Tensor = None,
         out_score: torch.Tensor = None, stream=None):
    """tr_topk: per-request top-k; returns (out_idx int64 [R, k], out_score fp32 [R, k])."""
    R = len(req_offsets) - 1
    off = (C.c_int64 * (R + 1))(*[int(x) for x in req_offsets])
    if out_idx is None:
        out_idx = torch.empty(R, k, dtype=torch.int64, device=scores.device)
    if out_score is None:
        out_score = torch.empty(R, k, dtype=torch.float32, device=scores.device)
    _check(L.load().tr_topk(_ptr(scores), int(req_offsets[-1]), off, R, int(k), _ptr(out_idx), _ptr(out_score),
                            _stream(stream)))
    return out_idx, out_score


def sync_status(stream=None, timeout_ms: int = 10_000) -> int:
    """tr_sync_status; returns the status code (does not raise)."""
    return int(L.load().tr_sync_status(_stream(stream), timeout_ms))


def last_error() -> str:
    return L.load().tr_last_error().decode()
