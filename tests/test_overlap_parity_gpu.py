"""GPU parity of overlapping compressed keys (SA_POOL_OVERLAP) against the
float64 oracle (oracle.sparse_attn_oracle.pool_overlap and
blocks_from_compressed): the window means, the block scores (the max over the
windows that touch a block), the selected sets and the decode output.

Scoring runs in one CTA per (sequence, KV head) when the grid is already
full, else splits a pair's windows over several CTAs whose last one selects;
both forms are covered."""
import numpy as np
import pytest
import torch

from helpers import assert_close, compare_sets, oracle_decode
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")


def _w(**over):
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, ctx_len=64 * 37 + 19, n_needles=3)
    base.update(over)
    return WORKLOADS["decode_32k_overlap"].scaled(**base)


def n_windows(w):
    C, l, s = w.ctx_len, w.pool_kernel, w.pool_stride
    return (C - l) // s + 1 if C >= l else 0


def run_pool(w, inp, p):
    Kc = torch.full((w.batch, w.num_kv_heads, max(n_windows(w), 1), 128), float("nan"), device="cuda")
    sa.pool_keys(p, inp["K"], Kc)
    return Kc


def pairs_of(w, limit=None):
    pairs = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    if limit and len(pairs) > limit:
        pick = np.random.default_rng(5).choice(len(pairs), limit, replace=False)
        pairs = sorted({pairs[i] for i in pick} | {pairs[0], pairs[-1]})
    return pairs


@pytest.mark.parametrize("dtype,b,l,s,C", [
    ("bf16", 64, 32, 16, 64 * 37 + 19),
    ("f32", 64, 48, 16, 64 * 21 + 5),
    ("bf16", 64, 17, 16, 64 * 9 + 40),        # odd window length
    ("bf16", 32, 24, 8, 32 * 40 + 7),
    ("f32", 64, 64, 64, 64 * 12),             # no overlap: plain block means
    ("bf16", 64, 32, 16, 20),                 # shorter than a window: nothing written
])
def test_overlap_pool_parity(dtype, b, l, s, C):
    w = _w(dtype=dtype, block_size=b, pool_kernel=l, pool_stride=s, ctx_len=C, sink_keys=b, window_keys=b)
    inp = make_inputs(w, seed=91, device="cuda")
    Kc = run_pool(w, inp, sa.params_for(w))
    torch.cuda.synchronize()
    n_c = n_windows(w)
    if n_c == 0:
        assert torch.isnan(Kc).all()
        return
    for (bi, h) in pairs_of(w):
        ref = orc.pool_overlap(inp["K"][bi, h, :C].double().cpu().numpy(), l, s)
        assert ref.shape[0] == n_c
        np.testing.assert_allclose(Kc[bi, h, :n_c].double().cpu().numpy(), ref, atol=2e-6, rtol=1e-5)


@pytest.mark.parametrize("over,want_scores", [
    ({}, True),                                                   # several CTAs per pair
    (dict(ctx_len=64 * 3 + 5), True),                              # one CTA per pair, 3 blocks
    (dict(batch=40, num_kv_heads=8, num_q_heads=32, ctx_len=4096 + 77), True),   # grid full: one CTA
    (dict(pool_kernel=64, pool_stride=16, ctx_len=64 * 30 + 63), False),
    (dict(block_size=128, pool_kernel=96, pool_stride=32, ctx_len=128 * 20 + 100, top_k=5), True),
    (dict(top_k=500), True),                                       # k above #candidates
])
def test_overlap_score_topk_parity(over, want_scores):
    w = _w(**over)
    inp = make_inputs(w, seed=92, device="cuda")
    p = sa.params_for(w)
    Kc = run_pool(w, inp, p)
    nb = w.ctx_len // w.block_size
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device="cuda", dtype=torch.int32)
    scores = torch.empty((w.batch, w.num_kv_heads, nb), device="cuda") if want_scores else None
    ws = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK)
    sa.score_topk(p, inp["Q"], Kc, idx, scores, ws)
    assert sa.read_status(ws) == sa.SA_OK
    ref = oracle_decode(w, inp, pairs_of(w, limit=8))
    ties = 0
    for (b, h), r in ref.items():
        if want_scores:
            np.testing.assert_allclose(scores[b, h].double().cpu().numpy(), r["scores"], atol=2e-5, rtol=2e-5)
        v = compare_sets(idx[b, h].cpu().numpy(), r["sel"])
        assert v != "mismatch", (b, h, idx[b, h].tolist(), r["sel"].selected)
        ties += v == "near_tie"
    print(f"\noverlap score/top-k {over}: {len(ref)} pairs, {ties} near-ties")


def check_decode(w, seed, out_dtype=torch.float32, limit=None):
    inp = make_inputs(w, seed=seed, device="cuda")
    p = sa.params_for(w, out_dtype="bf16" if out_dtype == torch.bfloat16 else "f32")
    assert sa.decode_launches(p) == 2
    Kc = run_pool(w, inp, p)
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device="cuda", dtype=out_dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device="cuda")
    idx = torch.empty((w.batch, w.num_kv_heads, max(w.top_k, 1)), device="cuda", dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_DECODE)
    sa.sparse_attn_decode(p, inp["Q"], inp["K"], inp["V"], Kc, O, lse, idx, ws)
    assert sa.read_status(ws) == sa.SA_OK
    G = w.group
    ref = oracle_decode(w, inp, pairs_of(w, limit))
    n_tie = 0
    for (b, h), r in ref.items():
        v = compare_sets(idx[b, h, :w.top_k].cpu().numpy(), r["sel"])
        assert v != "mismatch", (b, h, idx[b, h].tolist(), r["sel"].selected)
        if v == "near_tie":
            n_tie += 1
            continue
        dt = "f32" if (w.dtype == "f32" and out_dtype == torch.float32) else "bf16"
        assert_close(O[b, :, h * G:(h + 1) * G], r["O"], dt, f"O pair {(b, h)}")
        err = np.abs(lse[b, :, h * G:(h + 1) * G].double().cpu().numpy() - r["lse"]).max()
        assert err < (2e-5 if w.dtype == "f32" else 2e-4), err
    print(f"\n{w.name} {w.ctx_len}: {len(ref)} pairs, {n_tie} near-ties")
    return inp, idx


@pytest.mark.parametrize("over", [
    {},
    dict(dtype="f32", ctx_len=64 * 25 + 33),
    dict(n_q=6, num_q_heads=16, num_kv_heads=8, batch=3, ctx_len=64 * 50 + 1),   # draft chunk
    dict(ctx_len=40),                                                             # no complete block
])
def test_overlap_decode_parity(over):
    check_decode(_w(**over), seed=93)


def test_overlap_decode_needles_bf16_output():
    w = _w(ctx_len=8192, n_needles=6)
    inp, idx = check_decode(w, seed=94, out_dtype=torch.bfloat16)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            assert set(inp["needles"][b, h].tolist()) <= set(idx[b, h].tolist())


def test_overlap_decode_full_size_sampled():
    """The 32k decode workload with windows of 32 keys every 16 keys, at
    full size; the oracle checks a sample of pairs."""
    check_decode(WORKLOADS["decode_32k_overlap"], seed=95, out_dtype=torch.bfloat16, limit=6)
    torch.cuda.empty_cache()
