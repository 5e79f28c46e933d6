"""CPU-only checks of the C ABI: the library loads without a GPU, exports
every symbol include/sa.h declares, the params struct matches, and host-side
validation rejects bad arguments before any launch.  The validation tests
pass fake device pointers, so they are skipped wherever a GPU could run a
kernel on them (only the symbol and layout checks run there)."""
import ctypes
import os
import re

import pytest
import torch

from top_block_sparse_b200 import sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = open(os.path.join(ROOT, "include", "sa.h")).read()

FAKE = ctypes.c_void_p(0x10000)          # 16-byte aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p(0x10008)

# tests that hand the library FAKE addresses run on hosts without a GPU only
host_only = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: host-only test")


def declared_functions():
    body = re.sub(r"/\*.*?\*/", "", HEADER, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", body)))


def test_header_declares_the_abi():
    names = declared_functions()
    for must in ["sa_pool_keys", "sa_score_topk", "sa_sparse_attn_decode", "sa_sparse_attn_prefill",
                 "sa_sparse_attn_given_idx"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sa.lib_path())
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(sa.EXPORTED) | set(declared_functions())
    assert sa.version() == 103


def test_params_struct_layout():
    assert ctypes.sizeof(sa.SaParams) == 96
    assert sa.SaParams.sink_keys.offset == 64
    assert sa.SaParams.softmax_scale.offset == 80


def _p(**kw):
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, ctx_len=4096, n_q=1, block_size=64,
                top_k=8, sink_keys=64, window_keys=128, dtype="bf16")
    base.update(kw)
    return sa.make_params(**base)


def _decode(p, ws_bytes=1 << 30, q=FAKE, kc=FAKE):
    return sa.raw_call("sa_sparse_attn_decode", ctypes.byref(p), q, FAKE, FAKE, kc, FAKE, None, None,
                       FAKE, ws_bytes, None)


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), sa.SA_ERR_UNSUPPORTED),
    (dict(num_q_heads=7), sa.SA_ERR_INVALID),
    (dict(kv_capacity=100), sa.SA_ERR_INVALID),
    (dict(block_size=40), sa.SA_ERR_INVALID),
    (dict(top_k=-1), sa.SA_ERR_INVALID),
    (dict(sink_keys=-1), sa.SA_ERR_INVALID),
    (dict(n_q=0), sa.SA_ERR_INVALID),
    (dict(n_q=5), sa.SA_ERR_UNSUPPORTED),       # 5 tokens x GQA 4 = 20 rows > 16
    (dict(prefill=True), sa.SA_ERR_INVALID),     # decode entry point with the prefill selector
    (dict(batch=2 ** 31 - 1), sa.SA_ERR_UNSUPPORTED),            # pairs past 32-bit counts
    (dict(ctx_len=2 ** 41), sa.SA_ERR_UNSUPPORTED),              # cache rows past 2^40
    (dict(batch=2 ** 20, ctx_len=2 ** 30), sa.SA_ERR_UNSUPPORTED),   # pairs x rows past 2^48
])
def test_validation_rejects(kw, status):
    assert _decode(_p(**kw)) == status
    assert sa.raw_call("sa_last_error").decode() != ""
    # no workspace size for a problem the library refuses
    for op in range(6):
        assert sa.raw_call("sa_workspace_size", ctypes.byref(_p(**kw)), op) == 0


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(pool="overlap", pool_stride=24, pool_kernel=32), sa.SA_ERR_INVALID),   # s does not divide b
    (dict(pool="overlap", pool_stride=16, pool_kernel=8), sa.SA_ERR_INVALID),    # l < s
    (dict(pool="overlap", pool_stride=16, pool_kernel=80), sa.SA_ERR_INVALID),   # l > b
    (dict(pool="overlap", pool_stride=0, pool_kernel=32), sa.SA_ERR_INVALID),
])
def test_overlap_validation_rejects(kw, status):
    assert _decode(_p(**kw)) == status
    assert "pool" in sa.raw_call("sa_last_error").decode()


@host_only
def test_overlap_params_and_workspace():
    """pool_kernel must be 0 outside the overlap mode; the overlap mode runs
    as two kernels (scoring, attention), and its scoring workspace holds one
    score per window, in decode and in prefill (per tile: the windows that
    touch a complete block)."""
    p = _p()
    p.pool_kernel = 8
    assert _decode(p) == sa.SA_ERR_INVALID
    ov = _p(pool="overlap", pool_stride=16, pool_kernel=32)
    assert sa.raw_call("sa_decode_launches", ctypes.byref(ov)) == 2
    assert sa.raw_call("sa_decode_launches", ctypes.byref(_p())) in (1, 2)
    pf = _p(pool="overlap", pool_stride=16, pool_kernel=32, prefill=True, ctx_len=0, n_q=4096,
            num_q_heads=8, num_kv_heads=2)
    pf_mean = _p(prefill=True, ctx_len=0, n_q=4096, num_q_heads=8, num_kv_heads=2)
    nt, nb = 4096 // 64, 4096 // 64
    nc = min((4096 - 32) // 16 + 1, nb * 4)
    for op in (sa.SA_OP_PREFILL, sa.SA_OP_SCORE_TOPK):
        wm = sa.raw_call("sa_workspace_size", ctypes.byref(pf_mean), op)
        wo = sa.raw_call("sa_workspace_size", ctypes.byref(pf), op)
        assert wm > 0 and wo >= wm + 2 * (nt * 4 + 512) * (nc - nb) - 2048
    w_mean = sa.raw_call("sa_workspace_size", ctypes.byref(_p()), sa.SA_OP_SCORE_TOPK)
    w_ovl = sa.raw_call("sa_workspace_size", ctypes.byref(ov), sa.SA_OP_SCORE_TOPK)
    n_c = (4096 - 32) // 16 + 1
    assert w_ovl >= w_mean + 4 * 4 * (n_c - 4096 // 64) - 1024


@host_only
def test_validation_null_and_alignment():
    p = _p()
    assert sa.raw_call("sa_sparse_attn_decode", None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                       1 << 30, None) == sa.SA_ERR_INVALID
    assert _decode(p, q=None) == sa.SA_ERR_INVALID
    assert _decode(p, q=FAKE_ODD) == sa.SA_ERR_INVALID
    p2 = _p()
    p2.flags = 4
    assert _decode(p2) == sa.SA_ERR_INVALID


@host_only
def test_workspace_too_small():
    p = _p()
    need = sa.workspace_size(p, sa.SA_OP_DECODE)
    assert need > 0
    assert _decode(p, ws_bytes=need - 1) == sa.SA_ERR_WORKSPACE
    assert "workspace" in sa.raw_call("sa_last_error").decode()


def test_workspace_sizes_grow_with_the_problem():
    a = sa.workspace_size(_p(), sa.SA_OP_DECODE)
    b = sa.workspace_size(_p(batch=8), sa.SA_OP_DECODE)
    assert 0 < a < b
    assert sa.workspace_size(_p(head_dim=64), sa.SA_OP_DECODE) == 0
    assert sa.workspace_size(_p(), sa.SA_OP_GIVEN_IDX) > 0
    assert sa.workspace_size(_p(), sa.SA_OP_SCORE_TOPK) > 0


@host_only
def test_given_idx_validation():
    p = _p()
    st = sa.raw_call("sa_sparse_attn_given_idx", ctypes.byref(p), FAKE, FAKE, FAKE, None, 4, FAKE, None,
                     FAKE, 1 << 30, None)
    assert st == sa.SA_ERR_INVALID                  # idx NULL with idx_len > 0
    st = sa.raw_call("sa_sparse_attn_given_idx", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, -2, FAKE, None,
                     FAKE, 1 << 30, None)
    assert st == sa.SA_ERR_INVALID


def _verify(p, ws_bytes=1 << 30, mass=FAKE, idx=FAKE):
    return sa.raw_call("sa_verify_refresh", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, mass, idx,
                       FAKE, ws_bytes, None)


@host_only
@pytest.mark.parametrize("kw,status", [
    (dict(dtype="f32"), sa.SA_ERR_UNSUPPORTED),          # tensor cores: bf16 only
    (dict(block_size=32), sa.SA_ERR_UNSUPPORTED),        # mass tiles are 64 keys
    (dict(n_q=5), sa.SA_ERR_UNSUPPORTED),                # 5 tokens x GQA 4 = 20 rows > 16
    (dict(head_dim=64), sa.SA_ERR_UNSUPPORTED),
    (dict(prefill=True), sa.SA_ERR_INVALID),
])
def test_verify_validation_rejects(kw, status):
    assert _verify(_p(**kw)) == status
    assert sa.raw_call("sa_last_error").decode() != ""


@host_only
def test_verify_null_arguments_and_workspace():
    p = _p(n_q=3, num_q_heads=4, num_kv_heads=2)
    assert _verify(p, mass=None) == sa.SA_ERR_INVALID
    assert _verify(p, idx=None) == sa.SA_ERR_INVALID      # top_k > 0 needs idx_out
    need = sa.workspace_size(p, sa.SA_OP_VERIFY)
    assert need > 0
    assert _verify(p, ws_bytes=need - 1) == sa.SA_ERR_WORKSPACE
    # larger batch, larger workspace; the verify workspace holds the rows' lse
    assert sa.workspace_size(_p(n_q=3, num_q_heads=4, num_kv_heads=2, batch=8), sa.SA_OP_VERIFY) > need


def _pcol(**kw):
    base = dict(batch=1, num_q_heads=8, num_kv_heads=2, ctx_len=0, n_q=1000, block_size=64, top_k=70,
                sink_keys=0, window_keys=0, dtype="bf16", prefill=True)
    base.update(kw)
    return sa.make_params(**base)


def _column(p, n_cols=70, cols=FAKE, ws_bytes=1 << 30):
    return sa.raw_call("sa_column_attn", ctypes.byref(p), FAKE, FAKE, FAKE, cols, n_cols, FAKE, None,
                       FAKE, ws_bytes, None)


@host_only
@pytest.mark.parametrize("kw,n_cols,status", [
    (dict(dtype="f32"), 70, sa.SA_ERR_UNSUPPORTED),           # tensor cores: bf16 only
    (dict(num_q_heads=4), 70, sa.SA_ERR_UNSUPPORTED),         # GQA 2: built for multiples of 4 heads
    (dict(num_q_heads=12), 70, sa.SA_ERR_UNSUPPORTED),        # GQA 6 (not a multiple of 4)
    (dict(block_size=128), 70, sa.SA_ERR_UNSUPPORTED),        # the query group is 64 tokens
    (dict(prefill=False), 70, sa.SA_ERR_INVALID),             # sequence-type params needed
    ({}, -1, sa.SA_ERR_INVALID),
])
def test_column_validation_rejects(kw, n_cols, status):
    assert _column(_pcol(**kw), n_cols=n_cols) == status
    assert sa.raw_call("sa_last_error").decode() != ""


@host_only
def test_column_null_table_and_workspace():
    p = _pcol()
    assert _column(p, cols=None) == sa.SA_ERR_INVALID            # n_cols > 0 needs a table
    need = sa.workspace_size(p, sa.SA_OP_COLUMN)
    assert need > 0
    assert _column(p, ws_bytes=need - 1) == sa.SA_ERR_WORKSPACE
    # top_k is the column count for sizing, beyond the selection limit too
    assert sa.workspace_size(_pcol(top_k=13120), sa.SA_OP_COLUMN) > need


def test_status_strings():
    for code, name in [(0, "SA_OK"), (4, "SA_ERR_INDEX"), (6, "SA_ERR_TIMEOUT")]:
        assert sa.raw_call("sa_status_string", code).decode() == name


def test_noalloc_refuses_prefill_tables():
    """The allocation-free entry point takes decode and draft-chunk tables
    only: a prefill table is refused before the pointers are looked at (NULL
    pointers here, so nothing could be launched on any host)."""
    p = _p(prefill=True, ctx_len=0, n_q=4096)
    st = sa.raw_call("sa_sparse_attn_given_idx_noalloc", ctypes.byref(p), None, None, None, None, 8, None, None,
                     None)
    assert st == sa.SA_ERR_UNSUPPORTED
    msg = sa.raw_call("sa_last_error").decode()
    assert "SA_SEL_QUERY0" in msg and "sa_sparse_attn_given_idx" in msg


def _pb(**kw):
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, ctx_len=512 * 6 + 5, n_q=1, block_size=512, top_k=16,
                sink_keys=4, window_keys=512, dtype="bf16", pool="lsa", pool_stride=4)
    base.update(kw)
    return sa.make_params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(pool="mean"), sa.SA_ERR_INVALID),               # buckets are built on LSA pool keys
    (dict(pool_stride=8, block_size=512), sa.SA_ERR_UNSUPPORTED),    # pool keys of 1, 2 or 4 raw keys
    (dict(block_size=1024), sa.SA_ERR_UNSUPPORTED),       # 256 pool keys per cluster block > 128
    (dict(top_k=2048), sa.SA_ERR_UNSUPPORTED),            # 2048 x 4 members > 4096 expansion entries
])
def test_bucket_validation_rejects(kw, status):
    """Host-side checks of the bucket entry points run before any pointer is
    used (NULL pointers here) and agree with the workspace size query."""
    p = _pb(**kw)
    st_b = sa.raw_call("sa_bucket_build", ctypes.byref(p), None, 0, None, None, None)
    st_d = sa.raw_call("sa_bucket_decode", ctypes.byref(p), None, None, None, None, None, 0, None, None, None,
                       None, None, 0, None)
    assert st_b == status
    assert st_d == status
    assert sa.raw_call("sa_workspace_size", ctypes.byref(p), sa.SA_OP_BUCKET_DECODE) == 0


def test_bucket_arguments_and_workspace():
    p = _pb()
    # first_block past the complete cluster blocks; NULL buffers with blocks to build
    assert sa.raw_call("sa_bucket_build", ctypes.byref(p), None, 7, None, None, None) == sa.SA_ERR_INVALID
    assert sa.raw_call("sa_bucket_build", ctypes.byref(p), None, 0, None, None, None) == sa.SA_ERR_INVALID
    # nothing left to build: no launch, no pointer needed
    assert sa.raw_call("sa_bucket_build", ctypes.byref(p), None, 6, None, None, None) == sa.SA_OK
    # bucket_keys must be a multiple of the pool stride
    st = sa.raw_call("sa_bucket_decode", ctypes.byref(p), None, None, None, None, None, 6, None, None, None,
                     None, None, 0, None)
    assert st == sa.SA_ERR_INVALID and "bucket_keys" in sa.raw_call("sa_last_error").decode()
    a = sa.workspace_size(p, sa.SA_OP_BUCKET_DECODE)
    b = sa.workspace_size(_pb(top_k=64), sa.SA_OP_BUCKET_DECODE)
    c = sa.workspace_size(_pb(ctx_len=512 * 60), sa.SA_OP_BUCKET_DECODE)
    assert 0 < a < b and a < c
    # the scores of every bucket of the context: 64 per cluster block, 4 bytes each
    assert c - a >= 2 * 2 * 54 * 64 * 4
    assert sa.bucket_rows(p) == ((512 * 6 + 6) // 512) * 64
    # 5 tokens x GQA 4 = 20 query rows per KV head: the attention is not built
    assert sa.workspace_size(_pb(n_q=5), sa.SA_OP_BUCKET_DECODE) == 0


@host_only
def test_prefill_head_group_sizes():
    """Prefill and column attention take GQA groups of a multiple of 4 query
    heads (4 heads of a tile per work item): groups of 4, 8 and 16 get a
    workspace size, 2 and 6 are refused."""
    for G, ok in ((4, True), (8, True), (16, True), (2, False), (6, False)):
        pf = _p(prefill=True, ctx_len=0, n_q=4096, num_q_heads=2 * G, num_kv_heads=2)
        for op in (sa.SA_OP_PREFILL, sa.SA_OP_SCORE_TOPK, sa.SA_OP_GIVEN_IDX):
            assert (sa.raw_call("sa_workspace_size", ctypes.byref(pf), op) > 0) == ok, (G, op)
        assert (sa.workspace_size(_pcol(num_q_heads=2 * G), sa.SA_OP_COLUMN) > 0) == ok, G
