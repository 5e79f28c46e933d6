"""Thin ctypes binding of libsa.so (include/sa.h).

Argument marshalling only: torch tensors are passed as raw device pointers
with the current CUDA stream; every step runs in the library's kernels.
Importing this module loads libsa.so and raises ImportError if it is missing
(build it with ``python -m top_block_sparse_b200.build``).  There is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libsa.so not found at {_LIB_PATH}; run python -m top_block_sparse_b200.build")
_lib = ctypes.CDLL(_LIB_PATH)

# ---- constants mirrored from sa.h ------------------------------------------
SA_OK, SA_ERR_INVALID, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_INDEX, SA_ERR_CUDA, SA_ERR_TIMEOUT = range(7)
SA_F32, SA_BF16 = 0, 1
SA_POOL_MEAN, SA_POOL_LSA, SA_POOL_OVERLAP = 0, 1, 2
SA_SEL_QUERY0, SA_SEL_TILE_MAX = 0, 1
SA_OP_SCORE_TOPK, SA_OP_GIVEN_IDX, SA_OP_DECODE, SA_OP_PREFILL, SA_OP_VERIFY, SA_OP_COLUMN = 0, 1, 2, 3, 4, 5
SA_OP_BUCKET_DECODE = 6
SA_FLAG_TRUSTED_IDX = 1

EXPORTED = ["sa_version", "sa_workspace_size", "sa_workspace_init", "sa_pool_keys", "sa_score_topk",
            "sa_sparse_attn_given_idx", "sa_sparse_attn_decode", "sa_sparse_attn_prefill",
            "sa_read_status", "sa_status_string", "sa_last_error", "sa_sparse_attn_given_idx_noalloc",
            "sa_decode_launches", "sa_verify_refresh", "sa_column_attn", "sa_append_kv",
            "sa_bucket_build", "sa_bucket_decode"]


class SaParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("ctx_len", ctypes.c_int64), ("kv_capacity", ctypes.c_int64),
        ("n_q", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("pool", ctypes.c_int32), ("pool_stride", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32), ("select", ctypes.c_int32),
        ("sink_keys", ctypes.c_int64), ("window_keys", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float), ("flags", ctypes.c_int32),
        ("pool_kernel", ctypes.c_int32),
    ]


assert ctypes.sizeof(SaParams) == 96

_vp, _sz, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
_P = ctypes.POINTER(SaParams)
_sig = {
    "sa_version": (_i32, []),
    "sa_workspace_size": (_sz, [_P, _i32]),
    "sa_workspace_init": (_i32, [_vp, _sz, _vp]),
    "sa_pool_keys": (_i32, [_P, _vp, _vp, _vp]),
    "sa_score_topk": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_sparse_attn_given_idx": (_i32, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "sa_sparse_attn_decode": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_sparse_attn_prefill": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_sparse_attn_given_idx_noalloc": (_i32, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp]),
    "sa_read_status": (_i32, [_vp, _vp]),
    "sa_status_string": (ctypes.c_char_p, [_i32]),
    "sa_last_error": (ctypes.c_char_p, []),
    "sa_decode_launches": (_i32, [_P]),
    "sa_verify_refresh": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_column_attn": (_i32, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "sa_append_kv": (_i32, [_P, _vp, _vp, _vp, _vp, _vp]),
    "sa_bucket_build": (_i32, [_P, _vp, ctypes.c_int64, _vp, _vp, _vp]),
    "sa_bucket_decode": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class SaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_lib.sa_status_string(status).decode()}: {msg}")
        self.status = status


def _check(st: int):
    if st != SA_OK:
        raise SaError(st, _lib.sa_last_error().decode())


def version() -> int:
    return int(_lib.sa_version())


def make_params(*, batch, num_q_heads, num_kv_heads, ctx_len, n_q, block_size, top_k,
                sink_keys, window_keys, dtype="bf16", out_dtype=None, pool="mean",
                pool_stride=4, pool_kernel=0, kv_capacity=None, prefill=False, softmax_scale=0.0,
                head_dim=128) -> SaParams:
    dt = SA_BF16 if dtype == "bf16" else SA_F32
    odt = dt if out_dtype is None else (SA_BF16 if out_dtype == "bf16" else SA_F32)
    return SaParams(batch=batch, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, ctx_len=ctx_len,
                    kv_capacity=(ctx_len + n_q) if kv_capacity is None else kv_capacity,
                    n_q=n_q, block_size=block_size,
                    pool={"mean": SA_POOL_MEAN, "lsa": SA_POOL_LSA, "overlap": SA_POOL_OVERLAP}[pool],
                    pool_stride=pool_stride, pool_kernel=pool_kernel if pool == "overlap" else 0,
                    top_k=top_k, dtype=dt, out_dtype=odt,
                    select=SA_SEL_TILE_MAX if prefill else SA_SEL_QUERY0,
                    sink_keys=sink_keys, window_keys=window_keys,
                    softmax_scale=softmax_scale, flags=0)


def params_for(w, kv_capacity=None, out_dtype=None) -> SaParams:
    """SaParams for a Workload from top_block_sparse_b200.inputs."""
    return make_params(batch=w.batch, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                       ctx_len=w.ctx_len, n_q=w.n_q, block_size=w.block_size, top_k=w.top_k,
                       sink_keys=w.sink_keys, window_keys=w.window_keys, dtype=w.dtype,
                       out_dtype=out_dtype, pool=w.pool, pool_stride=w.pool_stride,
                       pool_kernel=w.pool_kernel, kv_capacity=kv_capacity,
                       prefill=w.prefill, head_dim=w.head_dim)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libsa must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libsa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(p: SaParams, op: int) -> int:
    return int(_lib.sa_workspace_size(ctypes.byref(p), op))


def alloc_workspace(p: SaParams, op: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size op needs (the status word and the
    self-resetting tickets start at zero)."""
    n = workspace_size(p, op)
    if n == 0:
        _check(SA_ERR_INVALID if _lib.sa_last_error() else SA_ERR_UNSUPPORTED)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.sa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def pool_keys(p: SaParams, K: torch.Tensor, Kc: torch.Tensor, stream=None):
    _check(_lib.sa_pool_keys(ctypes.byref(p), _ptr(K), _ptr(Kc), _stream(stream)))


def append_kv(p: SaParams, K_new, V_new, K, V, stream=None):
    """The new tokens' keys and values [B, Hkv, n_q, d] into cache rows ctx_len.."""
    _check(_lib.sa_append_kv(ctypes.byref(p), _ptr(K_new), _ptr(V_new), _ptr(K), _ptr(V), _stream(stream)))


def score_topk(p: SaParams, Q, Kc, idx, scores=None, ws=None, stream=None):
    _check(_lib.sa_score_topk(ctypes.byref(p), _ptr(Q), _ptr(Kc), _ptr(idx), _ptr(scores),
                              _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def sparse_attn_given_idx(p: SaParams, Q, K, V, idx, O, lse=None, ws=None, stream=None):
    idx_len = 0 if idx is None else int(idx.shape[-1])
    _check(_lib.sa_sparse_attn_given_idx(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                         idx_len, _ptr(O), _ptr(lse), _ptr(ws),
                                         0 if ws is None else ws.numel(), _stream(stream)))


def sparse_attn_given_idx_noalloc(p: SaParams, Q, K, V, idx, O, lse=None, stream=None):
    """sa_sparse_attn_given_idx without a workspace: scratch comes from the
    library's static device array (for callers that cannot allocate)."""
    idx_len = 0 if idx is None else int(idx.shape[-1])
    _check(_lib.sa_sparse_attn_given_idx_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                                 idx_len, _ptr(O), _ptr(lse), _stream(stream)))


def sparse_attn_decode(p: SaParams, Q, K, V, Kc, O, lse=None, idx_out=None, ws=None, stream=None):
    _check(_lib.sa_sparse_attn_decode(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(O),
                                      _ptr(lse), _ptr(idx_out), _ptr(ws),
                                      0 if ws is None else ws.numel(), _stream(stream)))


def sparse_attn_prefill(p: SaParams, Q, K, V, Kc, O, lse=None, idx_out=None, ws=None, stream=None):
    _check(_lib.sa_sparse_attn_prefill(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(O),
                                       _ptr(lse), _ptr(idx_out), _ptr(ws),
                                       0 if ws is None else ws.numel(), _stream(stream)))


def verify_refresh(p: SaParams, Q, K, V, O, mass, lse=None, idx_out=None, ws=None, stream=None):
    """Dense verify of a draft chunk: O, lse, per-block attention mass and the
    top_k blocks by mass (sa_verify_refresh)."""
    _check(_lib.sa_verify_refresh(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(mass),
                                  _ptr(idx_out), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def column_attn(p: SaParams, Q, K, V, cols, O, lse=None, ws=None, stream=None):
    """Column-sparse attention of every 64-token group over its listed key
    columns (sa_column_attn); cols [B, Hkv, groups, n_cols] int32 or None."""
    n_cols = 0 if cols is None else int(cols.shape[-1])
    _check(_lib.sa_column_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(cols), n_cols, _ptr(O), _ptr(lse),
                               _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def bucket_rows(p: SaParams) -> int:
    """Bucket-cache rows per (sequence, KV head): every cluster block the
    cache can hold, block_size / 8 buckets each."""
    return (p.kv_capacity // p.block_size) * (p.block_size // 8)


def bucket_build(p: SaParams, K, centroids, members, first_block=0, stream=None):
    """LSA bucket cache of the complete cluster blocks from first_block on
    (sa_bucket_build): centroids [B, Hkv, R, d] fp32, members [B, Hkv, R,
    16 // pool_stride] int32, R = bucket_rows(p)."""
    _check(_lib.sa_bucket_build(ctypes.byref(p), _ptr(K), int(first_block), _ptr(centroids), _ptr(members),
                                _stream(stream)))


def bucket_decode(p: SaParams, Q, K, V, centroids, members, O, lse=None, sel_out=None, kept_out=None,
                  bucket_keys=0, ws=None, stream=None):
    """Decode / draft chunk with LSA flat bucket retrieval (sa_bucket_decode)."""
    _check(_lib.sa_bucket_decode(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(centroids), _ptr(members),
                                 int(bucket_keys), _ptr(O), _ptr(lse), _ptr(sel_out), _ptr(kept_out), _ptr(ws),
                                 0 if ws is None else ws.numel(), _stream(stream)))


def read_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises and returns (then clears) the device status of the
    workspace: SA_OK, SA_ERR_INDEX or SA_ERR_TIMEOUT."""
    return int(_lib.sa_read_status(_ptr(ws), _stream(stream)))


def decode_launches(p: SaParams) -> int:
    """Kernels one sparse_attn_decode call with `p` launches (1 fused, 2 split)."""
    return int(_lib.sa_decode_launches(ctypes.byref(p)))


def num_blocks(p: SaParams) -> int:
    n = p.n_q if p.select == SA_SEL_TILE_MAX else p.ctx_len
    return n // p.block_size


def raw_call(name: str, *args):
    """Direct access to an exported C function (ctypes-typed as in sa.h)."""
    return getattr(_lib, name)(*args)


def lib_path() -> str:
    return _LIB_PATH
