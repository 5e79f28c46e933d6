"""GPU parity of the causal prefill with LSA centroids and with overlapping
compressed keys against the float64 oracle, tile by tile.

LSA (LSA review §2.2-2.3): each query row's GQA-summed index query is
normalised, the tile score of a block is the largest row cosine against its
centroid.  Overlapping windows (SparDA "方法"): the tile takes the max over
its rows of every window complete inside its context, and a block the max
over the windows that share a key with it.

Bars as for the mean-pooled prefill: block scores within 2e-5; selected
sets identical except oracle near-ties; outputs within max abs 5e-3 and
relative L2 1e-2 (fp32 outputs, so no bf16 rounding relief applies).
"""
import numpy as np
import pytest
import torch

from helpers import assert_close, compare_sets, oracle_params
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")

# (pool, pool_stride, pool_kernel)
MODES = [("lsa", 4, 0), ("overlap", 16, 32), ("overlap", 32, 64), ("overlap", 8, 24), ("overlap", 64, 64)]


def pf(T, mode, Hkv=2, k=8, **kw):
    pool, s, l = mode
    return WORKLOADS["prefill_64k"].scaled(n_q=T, num_kv_heads=Hkv, num_q_heads=4 * Hkv, top_k=k,
                                           n_needles=min(k, 4), pool=pool, pool_stride=s,
                                           pool_kernel=l, **kw)


def kc_rows(w):
    if w.pool == "overlap":
        return (w.n_q - w.pool_kernel) // w.pool_stride + 1 if w.n_q >= w.pool_kernel else 0
    return w.n_q // 64


def head_arrays(inp, h, w):
    q = inp["Q"][0, :, 4 * h:4 * h + 4].double().cpu().numpy()     # [T, G, d]
    K = inp["K"][0, h, :w.n_q].double().cpu().numpy()
    V = inp["V"][0, h, :w.n_q].double().cpu().numpy()
    return q, K, V


@pytest.mark.parametrize("mode", MODES)
def test_prefill_pooled_scores_and_selection(mode):
    """sa_score_topk on a ragged prefill: the block scores of every
    candidate and the selected sets of every tile."""
    w = pf(64 * 40 + 17, mode)
    inp = make_inputs(w, seed=71, device="cuda")
    p = sa.params_for(w)
    T = w.n_q
    nb, nt = T // 64, (T + 63) // 64
    Kc = torch.empty((1, w.num_kv_heads, kc_rows(w), 128), device="cuda")
    sa.pool_keys(p, inp["K"], Kc)
    idx = torch.empty((1, w.num_kv_heads, nt, w.top_k), device="cuda", dtype=torch.int32)
    scores = torch.full((1, w.num_kv_heads, nt, nb), float("nan"), device="cuda")
    ws = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK)
    sa.score_topk(p, inp["Q"], Kc, idx, scores, ws)
    assert sa.read_status(ws) == sa.SA_OK
    op = oracle_params(w)
    ties = 0
    for h in range(w.num_kv_heads):
        q, K, V = head_arrays(inp, h, w)
        Kc_all = orc.compress(K, op)
        np.testing.assert_allclose(Kc[0, h].double().cpu().numpy(), Kc_all, atol=2e-6, rtol=1e-5)
        sel = orc.prefill_head_selection(q, Kc_all, op, range(nt))
        for i in range(nt):
            cand = orc.candidate_blocks(64 * i, op)
            if cand:
                ref = orc.prefill_tile_scores(q[i * 64:(i + 1) * 64], Kc_all[:orc.context_rows(64 * i, op)],
                                              op, 64 * i)
                got = scores[0, h, i, cand].double().cpu().numpy()
                np.testing.assert_allclose(got, ref[cand], atol=2e-5, rtol=2e-5)
            v = compare_sets(idx[0, h, i].cpu().numpy(), sel[i])
            assert v != "mismatch", (h, i, idx[0, h, i].tolist(), sel[i].selected)
            ties += v == "near_tie"
    print(f"\n{mode}: near-ties {ties}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("T,k", [(64 * 24, 8), (64 * 13 + 33, 3), (100, 8), (40, 4)])
def test_prefill_pooled_end_to_end(mode, T, k):
    """sa_sparse_attn_prefill: pooling, scoring, selection and attention of
    every tile, including a ragged tail, a sequence with one complete block
    and one with none."""
    w = pf(T, mode, k=k)
    inp = make_inputs(w, seed=72, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    nt = (T + 63) // 64
    Kc = torch.empty((1, w.num_kv_heads, max(kc_rows(w), 1), 128), device="cuda")
    O = torch.empty((1, T, w.num_q_heads, 128), device="cuda")
    lse = torch.empty((1, T, w.num_q_heads), device="cuda")
    idx = torch.empty((1, w.num_kv_heads, nt, w.top_k), device="cuda", dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_PREFILL)
    sa.sparse_attn_prefill(p, inp["Q"], inp["K"], inp["V"], Kc, O, lse, idx, ws)
    assert sa.read_status(ws) == sa.SA_OK
    op = oracle_params(w)
    ties = 0
    for h in range(w.num_kv_heads):
        q, K, V = head_arrays(inp, h, w)
        Kc_all = orc.compress(K, op)
        for i in range(nt):
            rows = slice(i * 64, min((i + 1) * 64, T))
            r = orc.prefill_tile(q[rows], K, V, i, op, Kc_all)
            v = compare_sets(idx[0, h, i].cpu().numpy(), r["sel"])
            assert v != "mismatch", (h, i, idx[0, h, i].tolist(), r["sel"].selected)
            if v == "near_tie":
                ties += 1
                continue
            assert_close(O[0, rows, 4 * h:4 * h + 4], r["O"], "bf16", f"head {h} tile {i}")
            lerr = np.abs(lse[0, rows, 4 * h:4 * h + 4].double().cpu().numpy() - r["lse"]).max()
            assert lerr < 2e-3, (h, i, lerr)
    print(f"\n{mode} T={T}: near-ties {ties}")


def test_prefill_overlap_needles_selected():
    """Needle blocks placed for the last tile's query win the max of their
    own windows: the last tile selects every one of them."""
    w = pf(64 * 48, ("overlap", 16, 32), Hkv=1, k=8)
    inp = make_inputs(w, seed=73, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    nt = w.n_q // 64
    Kc = torch.empty((1, 1, kc_rows(w), 128), device="cuda")
    O = torch.empty((1, w.n_q, 4, 128), device="cuda")
    idx = torch.empty((1, 1, nt, w.top_k), device="cuda", dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_PREFILL)
    sa.sparse_attn_prefill(p, inp["Q"], inp["K"], inp["V"], Kc, O, None, idx, ws)
    assert sa.read_status(ws) == sa.SA_OK
    assert set(inp["needles"][0, 0].tolist()) <= set(idx[0, 0, nt - 1].tolist())
