"""Randomised sa_params (valid and invalid) through the host-side entry
points: every call returns a defined status, with a message whenever it is
not SA_OK, and never crashes; sa_workspace_size is 0 exactly when the shared
validation refuses the problem.  Host only: the pointers are fake, so the
test is skipped wherever a GPU could run a kernel on them."""
import ctypes

import pytest
import torch

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

sa = pytest.importorskip("top_block_sparse_b200.sa")

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: host-only test")

FAKE = ctypes.c_void_p(0x10000)
STATUSES = {sa.SA_OK, sa.SA_ERR_INVALID, sa.SA_ERR_UNSUPPORTED, sa.SA_ERR_WORKSPACE, sa.SA_ERR_INDEX,
            sa.SA_ERR_CUDA, sa.SA_ERR_TIMEOUT}

small = st.integers(min_value=-3, max_value=70)
params = st.fixed_dictionaries(dict(
    batch=st.one_of(small, st.just(2 ** 31 - 1)),
    num_q_heads=st.sampled_from([0, 1, 2, 4, 8, 16, 32, 7]),
    num_kv_heads=st.sampled_from([0, 1, 2, 4, 8]),
    head_dim=st.sampled_from([128, 64, 0]),
    ctx_len=st.one_of(st.integers(min_value=-5, max_value=70000), st.just(2 ** 41)),
    n_q=st.sampled_from([0, 1, 2, 6, 7, 64, 4096]),
    block_size=st.sampled_from([0, 16, 40, 64, 128, 512, 65536]),
    pool=st.sampled_from([0, 1, 2, 3]),
    pool_stride=st.sampled_from([0, 1, 4, 16, 24]),
    pool_kernel=st.sampled_from([0, 8, 32, 64]),
    top_k=st.sampled_from([-1, 0, 1, 8, 64, 4096, 5000]),
    dtype=st.sampled_from([0, 1, 2]),
    out_dtype=st.sampled_from([0, 1, 2]),
    select=st.sampled_from([0, 1, 2]),
    sink_keys=st.sampled_from([-1, 0, 4, 64]),
    window_keys=st.sampled_from([-1, 0, 256, 512]),
    flags=st.sampled_from([0, 1, 2]),
    extra=st.integers(min_value=-1, max_value=40),
))


def _status_ok(st_):
    assert st_ in STATUSES
    if st_ != sa.SA_OK:
        assert sa.raw_call("sa_last_error").decode() != ""


@settings(max_examples=400, deadline=None)
@given(params)
def test_random_params_get_defined_statuses(d):
    extra = d.pop("extra")
    p = sa.SaParams(**{k: v for k, v in d.items()}, kv_capacity=0, softmax_scale=0.0)
    p.kv_capacity = max(p.ctx_len, 0) + max(p.n_q, 0) + extra
    sizes = [sa.raw_call("sa_workspace_size", ctypes.byref(p), op) for op in range(6)]
    assert all(s >= 0 for s in sizes)
    big = ctypes.c_size_t(1 << 40)
    _status_ok(sa.raw_call("sa_pool_keys", ctypes.byref(p), FAKE, FAKE, None))
    _status_ok(sa.raw_call("sa_score_topk", ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, big, None))
    _status_ok(sa.raw_call("sa_sparse_attn_decode", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                           FAKE, big, None))
    _status_ok(sa.raw_call("sa_sparse_attn_given_idx", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, 8, FAKE, None,
                           FAKE, big, None))
    _status_ok(sa.raw_call("sa_append_kv", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None))
    _status_ok(sa.raw_call("sa_sparse_attn_prefill", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                           FAKE, big, None))
    # a problem the decode entry point accepts has a decode workspace size
    st_ = sa.raw_call("sa_sparse_attn_decode", ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                      big, None)
    if st_ in (sa.SA_OK, sa.SA_ERR_CUDA):
        assert sizes[sa.SA_OP_DECODE] > 0
