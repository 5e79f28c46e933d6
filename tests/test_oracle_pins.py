"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against a closed form, an invariant the
definitions imply, a library routine the definition reduces to in a special
case, brute force on tiny inputs, or the hand-worked examples in
tests/golden/hand_worked.json.  No expected value here comes from the CUDA
library.  A final group plants plausible mistakes in (a copy of) the oracle
and checks that some pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = json.load(open(os.path.join(HERE, "golden", "hand_worked.json")))["cases"]


def P(w, **kw):
    p = orc.OracleParams(block_size=w.block_size, top_k=w.top_k,
                         sink_keys=w.sink_keys, window_keys=w.window_keys,
                         pool=w.pool, pool_stride=w.pool_stride, pool_kernel=w.pool_kernel)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- golden ---

def _case(name):
    return next(c for c in GOLD if c["name"] == name)


@pytest.mark.parametrize("name", ["decode_k1", "decode_k2", "decode_tie"])
def test_hand_worked_decode(name):
    c = _case(name)
    pr = c["params"]
    p = orc.OracleParams(block_size=pr["block_size"], top_k=pr["top_k"],
                         sink_keys=pr["sink_keys"], window_keys=pr["window_keys"])
    K = np.array(c["K"], float)
    V = np.array(c["V"], float)
    q = np.array(c["q"], float)[None]          # [n_q=1, G=1, d]
    r = orc.decode_pair(q, K, V, pr["C"], p)
    e = c["expect"]
    if "Kc" in e:
        np.testing.assert_allclose(r["Kc"], e["Kc"], atol=1e-15)
    if "scores" in e:
        np.testing.assert_allclose(r["scores"], e["scores"], atol=1e-15)
    if "candidates" in e:
        assert r["candidates"] == e["candidates"]
    assert r["sel"].selected == e["selected"]
    if "positions" in e:
        assert r["positions"][0].tolist() == e["positions"]
    np.testing.assert_allclose(r["O"][0, 0], e["O"], rtol=1e-14, atol=1e-14)
    assert abs(r["lse"][0, 0] - e["lse"]) < 1e-14


def test_hand_worked_lsa_centroid():
    c = _case("lsa_centroid")
    K = np.array(c["K"], float)
    cent = orc.pool_lsa(K, c["params"]["block_size"], c["params"]["pool_stride"])
    np.testing.assert_allclose(cent[0], c["expect"]["centroid"], atol=1e-15)
    p = orc.OracleParams(block_size=8, top_k=1, sink_keys=0, window_keys=0, pool="lsa")
    s = orc.block_scores(np.array(c["qbar"], float), cent, p)
    assert abs(s[0] - c["expect"]["score"]) < 1e-15


# ----------------------------------------------------------- compression ---

def test_pool_mean_equals_library_avg_pool():
    """Non-overlapping mean pooling is avg_pool1d with kernel = stride = b
    (a partial trailing block is dropped by both)."""
    K = rng(1).standard_normal((1000, 16))
    ref = torch.nn.functional.avg_pool1d(torch.from_numpy(K).T[None], 64, 64)[0].T
    got = orc.pool_mean(K, 64)
    assert got.shape == (15, 16)
    np.testing.assert_allclose(got, ref.numpy(), atol=1e-14)


def test_pool_mean_invariants():
    r = rng(2)
    K = r.standard_normal((256, 8))
    base = orc.pool_mean(K, 32)
    # permuting keys inside a block leaves the compressed key unchanged
    Kp = K.copy()
    for j in range(8):
        Kp[j * 32:(j + 1) * 32] = Kp[j * 32 + r.permutation(32)]
    np.testing.assert_allclose(orc.pool_mean(Kp, 32), base, atol=1e-14)
    # a block of identical keys compresses to that key; b = 1 is the identity
    x = r.standard_normal(8)
    assert np.allclose(orc.pool_mean(np.tile(x, (32, 1)), 32)[0], x, atol=1e-15)
    np.testing.assert_array_equal(orc.pool_mean(K, 1), K)


def test_pool_lsa_invariants():
    r = rng(3)
    K = r.standard_normal((2048, 16))
    c = orc.pool_lsa(K, 512, 4)
    assert c.shape == (4, 16)
    np.testing.assert_allclose(np.linalg.norm(c, axis=1), 1.0, atol=1e-14)
    # step (1) normalises every raw key: positive per-key scaling changes nothing
    a = r.uniform(0.01, 100.0, size=(2048, 1))
    np.testing.assert_allclose(orc.pool_lsa(K * a, 512, 4), c, atol=1e-13)
    # the pool-key sums are plain sums: centroid = normalise(sum of unit keys)
    unit = K / np.linalg.norm(K, axis=1, keepdims=True)
    direct = unit.reshape(4, 512, 16).sum(1)
    direct /= np.linalg.norm(direct, axis=1, keepdims=True)
    np.testing.assert_allclose(c, direct, atol=1e-13)
    # keys all pointing one way -> that direction; negation flips the sign
    x = r.standard_normal(16)
    same = np.outer(r.uniform(0.5, 2, 512), x)
    np.testing.assert_allclose(orc.pool_lsa(same, 512)[0], x / np.linalg.norm(x), atol=1e-14)
    np.testing.assert_allclose(orc.pool_lsa(-K, 512, 4), -c, atol=1e-13)


# --------------------------------------------------------------- scoring ---

def test_scores_brute_force_loops():
    """s_j = scale * (1/b) * sum_{t in block j} sum_h q_h . K_t, written as
    explicit Python loops over heads, keys and coordinates."""
    r = rng(4)
    G, d, b, T = 3, 8, 4, 32
    q = r.standard_normal((G, d))
    K = r.standard_normal((T, d))
    p = orc.OracleParams(block_size=b, top_k=2, sink_keys=0, window_keys=0)
    s = orc.block_scores(orc.index_query(q), orc.pool_mean(K, b), p)
    scale = 1 / math.sqrt(d)
    for j in range(T // b):
        acc = 0.0
        for t in range(j * b, (j + 1) * b):
            for h in range(G):
                for c in range(d):
                    acc += q[h, c] * K[t, c]
        assert abs(s[j] - scale * acc / b) < 1e-13


def test_lsa_scores_are_cosines():
    r = rng(5)
    K = r.standard_normal((4096, 16))
    p = orc.OracleParams(block_size=512, top_k=2, sink_keys=4, window_keys=512, pool="lsa")
    c = orc.compress(K, p)
    qbar = r.standard_normal(16)
    s = orc.block_scores(qbar, c, p)
    assert np.all(np.abs(s) <= 1 + 1e-15)
    np.testing.assert_allclose(orc.block_scores(7.5 * qbar, c, p), s, atol=1e-15)
    assert abs(orc.block_scores(c[2] * 3.0, c, p)[2] - 1.0) < 1e-14


# -------------------------------------------------- candidates and top-k ---

def _candidates_by_key_enumeration(C, p):
    b = p.block_size
    s_end, w_begin = min(p.sink_keys, C), max(C - p.window_keys, 0)
    return [j for j in range(C // b)
            if any(not (t < s_end or t >= w_begin) for t in range(j * b, (j + 1) * b))]


@pytest.mark.parametrize("C,b,S,W", [(4096, 64, 64, 128), (1000, 64, 64, 256), (640, 64, 100, 70),
                                     (300, 64, 0, 0), (64, 64, 64, 64), (2048, 512, 4, 512),
                                     (130, 64, 200, 10)])
def test_candidates_match_key_enumeration(C, b, S, W):
    p = orc.OracleParams(block_size=b, top_k=1, sink_keys=S, window_keys=W)
    assert orc.candidate_blocks(C, p) == _candidates_by_key_enumeration(C, p)


def test_candidate_counts_of_workloads():
    w = WORKLOADS
    assert len(orc.candidate_blocks(4096, P(w["tiny_decode"]))) == 61
    c1 = orc.candidate_blocks(32768, P(w["decode_32k"]))
    assert len(c1) == 507 and c1[0] == 1 and c1[-1] == 507
    c3 = orc.candidate_blocks(1048576, P(w["decode_1m"]))
    assert len(c3) == 2047 and c3[0] == 0          # block 0 only partly sink
    assert len(orc.candidate_blocks(16384, P(w["draft_chunk_16k"]))) == 251
    pp = P(w["prefill_64k"])
    for i in [0, 5, 6, 7, 100, 1023]:
        assert len(orc.candidate_blocks(64 * i, pp)) == max(0, i - 5)


def test_topk_matches_exhaustive_rank_count():
    """Selected iff fewer than k candidates beat it, where i beats j when
    s_i > s_j or (s_i == s_j and i < j); scores drawn with many exact ties."""
    r = rng(6)
    for trial in range(300):
        nb = int(r.integers(1, 13))
        s = r.integers(-3, 4, size=nb).astype(float) / 2.0
        cand = sorted(r.choice(nb, size=int(r.integers(0, nb + 1)), replace=False).tolist())
        for k in range(0, nb + 2):
            sel = orc.select_topk(s, cand, k).selected
            want = [j for j in cand
                    if sum(1 for i in cand if s[i] > s[j] or (s[i] == s[j] and i < j)) < k]
            assert sel == sorted(want)


def test_topk_subset_maximises_score_sum():
    """Brute force over all k-subsets: the chosen set has the largest total
    score (distinct scores, so the optimum is unique)."""
    r = rng(7)
    for trial in range(50):
        nb = 9
        s = r.standard_normal(nb)
        cand = list(range(nb))
        for k in range(1, 5):
            best = max(itertools.combinations(cand, k), key=lambda c: sum(s[list(c)]))
            assert orc.select_topk(s, cand, k).selected == sorted(best)


def test_near_tie_flag():
    s = np.array([1.0, 0.99999999, 0.5, 2.0])
    sel = orc.select_topk(s, [0, 1, 2, 3], 1)
    assert sel.selected == [3] and sel.near_tie is False and sel.gap == 1.0
    sel = orc.select_topk(s, [0, 1, 2, 3], 2)
    assert sel.selected == [0, 3] and sel.near_tie is True
    sel = orc.select_topk(s, [0, 1, 2], 1)
    assert sel.selected == [0] and sel.near_tie is True
    sel = orc.select_topk(s, [0, 1, 2], 3)
    assert sel.selected == [0, 1, 2] and sel.gap is None and sel.near_tie is False


# ----------------------------------------------------------- attention ---

def _slab(inp, b, h, G, dt=np.float64):
    q = inp["Q"][b, :, h * G:(h + 1) * G].double().numpy()
    K = inp["K"][b, h].double().numpy()
    V = inp["V"][b, h].double().numpy()
    return q, K, V


def _sdpa(q, K, V, n_keys):
    """Library dense attention of one query over keys [0, n_keys)."""
    qt = torch.from_numpy(q)[None, None, None]          # [1,1,1,d]
    kt = torch.from_numpy(K[:n_keys])[None, None]
    vt = torch.from_numpy(V[:n_keys])[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, 0, 0].numpy()


def test_needles_selected_tiny_decode():
    w = WORKLOADS["tiny_decode"]
    inp = make_inputs(w, seed=11)
    q, K, V = _slab(inp, 0, 0, w.group)
    r = orc.decode_pair(q, K, V, w.ctx_len, P(w))
    assert set(inp["needles"][0, 0].tolist()) <= set(r["sel"].selected)
    assert len(r["sel"].selected) == 8
    assert all(len(pz) == 705 for pz in r["positions"])       # (8+1+2)*64 + 1


def test_needles_selected_decode_32k_slab():
    w = WORKLOADS["decode_32k"].scaled(batch=1, num_q_heads=8, num_kv_heads=2)
    inp = make_inputs(w, seed=12)
    for h in range(2):
        q, K, V = _slab(inp, 0, h, w.group)
        r = orc.decode_pair(q, K, V, w.ctx_len, P(w))
        assert set(inp["needles"][0, h].tolist()) <= set(r["sel"].selected)
        assert len(r["positions"][0]) == 2369                 # (32+1+4)*64 + 1
        np.testing.assert_allclose(r["wsum"], 1.0, atol=1e-12)


def test_sink_window_always_attended_and_chunk_causal():
    w = WORKLOADS["draft_chunk_16k"].scaled(batch=1, num_kv_heads=1, num_q_heads=2, ctx_len=4096)
    inp = make_inputs(w, seed=13)
    q, K, V = _slab(inp, 0, 0, w.group)
    p = P(w)
    r = orc.decode_pair(q, K, V, w.ctx_len, p)
    C = w.ctx_len
    for j, pos in enumerate(r["positions"]):
        s = set(pos.tolist())
        assert set(range(64)) <= s and set(range(C - 256, C)) <= s
        assert set(range(C, C + j + 1)) <= s and max(s) == C + j
        assert len(pos) == (16 + 1 + 4) * 64 + j + 1


@pytest.mark.parametrize("pool", ["mean", "lsa", "overlap"])
def test_dense_equivalence_when_topk_covers_all(pool):
    """With k >= #candidates the sparse result is dense causal attention
    (the special case S = all-ones causal of the masked softmax)."""
    b = 512 if pool == "lsa" else 64
    w = WORKLOADS["draft_chunk_16k"].scaled(batch=1, num_kv_heads=1, num_q_heads=3,
                                            ctx_len=2048 + 37, block_size=b, pool=pool,
                                            pool_stride=16 if pool == "overlap" else 4,
                                            pool_kernel=32 if pool == "overlap" else 0)
    inp = make_inputs(w, seed=14)
    q, K, V = _slab(inp, 0, 0, w.group)
    p = P(w, top_k=10_000)
    r = orc.decode_pair(q, K, V, w.ctx_len, p)
    for j in range(w.n_q):
        for g in range(w.group):
            ref = _sdpa(q[j, g], K, V, w.ctx_len + j + 1)
            np.testing.assert_allclose(r["O"][j, g], ref, atol=1e-12)
            z = K[:w.ctx_len + j + 1] @ q[j, g] / math.sqrt(128)
            assert abs(r["lse"][j, g] - logsumexp(z)) < 1e-12


def test_block_size_one_full_window_is_dense():
    r_ = rng(8)
    C, d = 50, 8
    K = r_.standard_normal((C + 1, d))
    V = r_.standard_normal((C + 1, d))
    q = r_.standard_normal((1, 2, d))
    p = orc.OracleParams(block_size=1, top_k=0, sink_keys=0, window_keys=C)
    r = orc.decode_pair(q, K, V, C, p)
    for g in range(2):
        np.testing.assert_allclose(r["O"][0, g], _sdpa(q[0, g], K, V, C + 1), atol=1e-13)


def test_constant_values_and_equal_keys():
    w = WORKLOADS["tiny_decode"]
    inp = make_inputs(w, seed=15)
    q, K, V = _slab(inp, 0, 0, w.group)
    p = P(w)
    Vc = np.tile(np.arange(128, dtype=float), (K.shape[0], 1))
    r = orc.decode_pair(q, K, Vc, w.ctx_len, p)
    np.testing.assert_allclose(r["O"], np.broadcast_to(Vc[0], r["O"].shape), atol=1e-12)
    Ke = np.tile(K[0], (K.shape[0], 1))
    r2 = orc.decode_pair(q, Ke, V, w.ctx_len, p)
    pos = r2["positions"][0]
    np.testing.assert_allclose(r2["O"][0, 0], V[pos].mean(axis=0), atol=1e-12)


def test_attention_pure_python_loops():
    """Brute-force softmax with explicit loops on a tiny case."""
    r_ = rng(9)
    C, d = 24, 4
    K = r_.standard_normal((C + 2, d))
    V = r_.standard_normal((C + 2, d))
    q = r_.standard_normal((2, 1, d))
    p = orc.OracleParams(block_size=4, top_k=2, sink_keys=4, window_keys=4)
    r = orc.decode_pair(q, K, V, C, p)
    for j in range(2):
        pos = r["positions"][j].tolist()
        z = [sum(q[j, 0, c] * K[t, c] for c in range(d)) / math.sqrt(d) for t in pos]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        tot = sum(e)
        for c in range(d):
            o = sum(e[i] * V[t, c] for i, t in enumerate(pos)) / tot
            assert abs(o - r["O"][j, 0, c]) < 1e-13
        assert abs(m + math.log(tot) - r["lse"][j, 0]) < 1e-13


# --------------------------------------------------------------- prefill ---

def test_prefill_tile_score_is_max_of_row_scores():
    r_ = rng(10)
    G, d, b = 4, 16, 8
    K = r_.standard_normal((10 * b, d))
    q_tile = r_.standard_normal((b, G, d))
    p = orc.OracleParams(block_size=b, top_k=2, sink_keys=b, window_keys=2 * b)
    Kc = orc.pool_mean(K, b)[:7]
    s = orc.prefill_tile_scores(q_tile, Kc, p)
    for j in range(7):
        rows = [sum(float(q_tile[r, h] @ Kc[j]) for h in range(G)) / math.sqrt(d) for r in range(b)]
        assert abs(s[j] - max(rows)) < 1e-13


def test_prefill_dense_equivalence_and_needles():
    w = WORKLOADS["prefill_64k"].scaled(n_q=1024 + 40, num_q_heads=2, num_kv_heads=1, n_needles=3)
    inp = make_inputs(w, seed=16)
    q = inp["Q"][0, :, 0:2].double().numpy()             # [T, G, d]
    K = inp["K"][0, 0].double().numpy()
    V = inp["V"][0, 0].double().numpy()
    T = w.n_q
    # dense equivalence: k covers every candidate
    p = P(w, top_k=10_000)
    Kc = orc.compress(K, p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(1, 0, 2)[None],
        torch.from_numpy(K)[None, None].expand(1, 2, T, 128),
        torch.from_numpy(V)[None, None].expand(1, 2, T, 128), is_causal=True)[0].permute(1, 0, 2).numpy()
    for i in [0, 3, 7, 16]:
        rows = slice(i * 64, min((i + 1) * 64, T))
        r = orc.prefill_tile(q[rows], K, V, i, p, Kc)
        np.testing.assert_allclose(r["O"], ref[rows], atol=1e-12)
        np.testing.assert_allclose(r["wsum"], 1.0, atol=1e-12)
    # the last (ragged) tile selects every needle with the real k
    p = P(w)
    i = (T - 1) // 64
    r = orc.prefill_tile(q[i * 64:], K, V, i, p, Kc)
    assert set(inp["needles"][0, 0].tolist()) <= set(r["sel"].selected)
    assert len(r["sel"].selected) == min(64, i - 5)


def test_prefill_head_selection_matches_tiles_and_brute_force():
    """The selection-only helper picks, for every tile of a ragged case, the
    same blocks as the full tile computation, and the same blocks as a brute
    force: tile score = max over the rows of the hand-summed group logits,
    candidates by key enumeration, then an exhaustive sort."""
    r_ = rng(61)
    G, d, b = 2, 16, 8
    T = 13 * b + 5
    K = r_.standard_normal((T, d))
    V = r_.standard_normal((T, d))
    q = r_.standard_normal((T, G, d))
    p = orc.OracleParams(block_size=b, top_k=3, sink_keys=b, window_keys=2 * b)
    Kc_all = orc.pool_mean(K, b)
    nt = (T + b - 1) // b
    sels = orc.prefill_head_selection(q, Kc_all, p, range(nt))
    for i in range(nt):
        full = orc.prefill_tile(q[i * b:(i + 1) * b], K, V, i, p, Kc_all)
        assert sels[i].selected == full["sel"].selected, i
        C = i * b
        rows = range(i * b, min((i + 1) * b, T))
        brute = []
        for j in range(C // b):
            keys = range(j * b, (j + 1) * b)
            if all(t < b or t >= C - 2 * b for t in keys):
                continue                                       # wholly inside sink or window
            mean = [sum(K[t, c] for t in keys) / b for c in range(d)]
            s = max(sum(sum(q[rr, g, c] for g in range(G)) * mean[c] for c in range(d)) for rr in rows)
            brute.append((-s / math.sqrt(d), j))
        brute.sort()
        assert sels[i].selected == sorted(j for _, j in brute[:3]), i


@pytest.mark.parametrize("pool", ["mean", "lsa", "overlap"])
def test_compress_without_a_complete_block_is_empty(pool):
    """Fewer keys than one block (or one window) give no compressed key in
    every pooling mode (reading R5: only complete blocks are compressed)."""
    p = orc.OracleParams(block_size=64, top_k=1, sink_keys=0, window_keys=0, pool=pool,
                         pool_stride=16 if pool == "overlap" else 4, pool_kernel=32 if pool == "overlap" else 0)
    short = 31 if pool == "overlap" else 63
    for T in (0, 1, short):
        assert orc.compress(rng(65).standard_normal((T, 8)), p).shape == (0, 8)
    assert orc.compress(rng(65).standard_normal((short + 1, 8)), p).shape == (1, 8)


def _prefill_ovl_brute(q, K, i, b, l, s_, scale):
    """Tile scores of tile i by enumeration: for each complete context block
    j, the max over the tile's rows and over the windows lying wholly inside
    the context [0, i b) that share a key with the block, of the hand-summed
    group logit against the window's hand-averaged keys."""
    C = i * b
    T, G, d = q.shape
    rows = range(i * b, min((i + 1) * b, T))
    out = []
    for j in range(C // b):
        block = set(range(j * b, (j + 1) * b))
        best = -math.inf
        for c in range(C):
            keys = range(c * s_, c * s_ + l)
            if c * s_ + l > C or not block.intersection(keys):
                continue
            mean = [sum(K[t, e] for t in keys) / l for e in range(d)]
            for rr in rows:
                best = max(best, scale * sum(sum(q[rr, g, e] for g in range(G)) * mean[e] for e in range(d)))
        out.append(best)
    return np.array(out)


@pytest.mark.parametrize("b,l,s_", [(8, 6, 2), (8, 8, 4), (8, 4, 4), (16, 12, 4)])
def test_prefill_overlap_tile_scores_brute_force(b, l, s_):
    """Overlapping compression in a causal prefill (readings R2 and R18): the
    oracle's tile scores and selections equal an enumeration over rows,
    windows complete inside the tile's context and blocks; an exhaustive
    sort with candidates by key enumeration gives the same sets."""
    r_ = rng(62 + b + l + s_)
    G, d = 2, 6
    T = 9 * b + 3
    K = r_.standard_normal((T, d))
    V = r_.standard_normal((T, d))
    q = r_.standard_normal((T, G, d))
    p = orc.OracleParams(block_size=b, top_k=2, sink_keys=b, window_keys=b, pool="overlap",
                         pool_stride=s_, pool_kernel=l, scale=0.5)
    Kc_all = orc.compress(K, p)
    nt = (T + b - 1) // b
    sels = orc.prefill_head_selection(q, Kc_all, p, range(nt))
    for i in range(1, nt):
        C = i * b
        ref = _prefill_ovl_brute(q, K, i, b, l, s_, 0.5)
        got = orc.prefill_tile_scores(q[i * b:(i + 1) * b], Kc_all[:orc.context_rows(C, p)], p, C)
        np.testing.assert_allclose(got, ref, atol=1e-12)
        full = orc.prefill_tile(q[i * b:(i + 1) * b], K, V, i, p, Kc_all)
        np.testing.assert_allclose(full["scores"], ref, atol=1e-12)
        cand = [j for j in range(C // b)
                if any(not (t < b or t >= C - b) for t in range(j * b, (j + 1) * b))]
        brute = sorted(sorted(cand, key=lambda j: (-ref[j], j))[:2])
        assert full["sel"].selected == brute == sels[i].selected, i


def test_prefill_overlap_without_overlap_is_mean_prefill():
    """l = s = b: one window per block, so the overlapping prefill gives the
    block-mean prefill's scores, selections and outputs on every tile."""
    w = WORKLOADS["prefill_64k"].scaled(n_q=64 * 11 + 9, num_q_heads=2, num_kv_heads=1, top_k=3, n_needles=2)
    inp = make_inputs(w, seed=63)
    q = inp["Q"][0, :, 0:2].double().numpy()
    K = inp["K"][0, 0].double().numpy()
    V = inp["V"][0, 0].double().numpy()
    p_mean = P(w)
    p_ovl = P(w, pool="overlap", pool_stride=64, pool_kernel=64)
    Kc_m, Kc_o = orc.compress(K, p_mean), orc.compress(K, p_ovl)
    for i in (1, 5, 8, 11):
        rows = slice(i * 64, (i + 1) * 64)
        a = orc.prefill_tile(q[rows], K, V, i, p_mean, Kc_m)
        o = orc.prefill_tile(q[rows], K, V, i, p_ovl, Kc_o)
        np.testing.assert_allclose(o["scores"], a["scores"], atol=1e-13)
        assert o["sel"].selected == a["sel"].selected
        np.testing.assert_allclose(o["O"], a["O"], atol=1e-13)


def test_prefill_lsa_tile_scores_are_row_cosines():
    """LSA pooling in a causal prefill (readings R2 and R7): each row's index
    query is normalised, so scaling a row's group of queries by a positive
    factor leaves the tile scores unchanged, every score is a cosine
    against a unit centroid (|s| <= 1), a tile whose rows all point along
    one centroid scores it 1, and a single-row tile equals the decode score
    of that row."""
    r_ = rng(64)
    G, d, b = 2, 8, 16
    T = 7 * b
    K = r_.standard_normal((T, d))
    q = r_.standard_normal((b, G, d))
    p = orc.OracleParams(block_size=b, top_k=2, sink_keys=0, window_keys=0, pool="lsa", pool_stride=4)
    Kc = orc.compress(K, p)[:6]
    s = orc.prefill_tile_scores(q, Kc, p)
    f = r_.uniform(0.1, 10.0, size=(b, 1, 1))
    np.testing.assert_allclose(orc.prefill_tile_scores(q * f, Kc, p), s, atol=1e-13)
    assert np.all(np.abs(s) <= 1 + 1e-12)
    for j in range(6):
        rows = [float(q[r].sum(0) @ Kc[j]) / math.sqrt(float(q[r].sum(0) @ q[r].sum(0))) for r in range(b)]
        assert abs(s[j] - max(rows)) < 1e-12
    along = np.repeat((3.0 * Kc[4] / G)[None, None], G, axis=1).repeat(b, axis=0)
    assert abs(orc.prefill_tile_scores(along, Kc, p)[4] - 1.0) < 1e-12
    np.testing.assert_allclose(orc.prefill_tile_scores(q[5:6], Kc, p),
                               orc.block_scores(q[5].sum(0), Kc, p), atol=1e-15)


# ------------------------------------------- overlapping compression ---

_OVL_CASES = [(64, 32, 16, 320), (64, 32, 16, 333), (64, 64, 16, 300), (64, 16, 16, 256),
              (32, 24, 8, 200), (64, 64, 64, 256), (64, 48, 16, 64 * 7 + 40)]


def _ovl_params(b, l, s):
    return orc.OracleParams(block_size=b, top_k=1, sink_keys=0, window_keys=0, pool="overlap",
                            pool_stride=s, pool_kernel=l, scale=0.5)


@pytest.mark.parametrize("b,l,s,C", _OVL_CASES)
def test_overlap_pool_is_library_avg_pool(b, l, s, C):
    """Overlapping mean pooling is avg_pool1d with kernel l and stride s
    (windows running past the rows are dropped by both)."""
    K = rng(5).standard_normal((C, 8))
    ref = torch.nn.functional.avg_pool1d(torch.from_numpy(K).T[None], l, s)[0].T.numpy()
    got = orc.compress(K, _ovl_params(b, l, s))
    assert got.shape == ref.shape == ((C - l) // s + 1, 8)
    np.testing.assert_allclose(got, ref, atol=1e-14)


@pytest.mark.parametrize("b,l,s,C", _OVL_CASES)
def test_overlap_block_scores_closed_form(b, l, s, C):
    """Keys on a ramp K_t = +-(t+1) v: compressed key c is
    +-(c*s + (l+1)/2) v, so with qbar.v > 0 a block's score is taken from the
    LAST window touching it on a rising ramp (c = min(n_c-1, ((j+1)b-1)//s):
    complete windows only) and from the FIRST on a falling one
    (c = max(0, ceil((jb-l+1)/s)): the window reaching in from the block
    before counts)."""
    d = 8
    p = _ovl_params(b, l, s)
    n_c = (C - l) // s + 1
    v = rng(6).standard_normal(d)
    qbar = 2.0 * v
    qv = float(qbar @ v) * 0.5
    for sign in (1.0, -1.0):
        K = sign * (np.arange(C)[:, None] + 1.0) * v[None, :]
        S = orc.blocks_from_compressed(orc.block_scores(qbar, orc.compress(K, p), p), C, p)
        assert S.shape == (C // b,)
        for j in range(C // b):
            if sign > 0:
                c = min(n_c - 1, ((j + 1) * b - 1) // s)
            else:
                c = max(0, -(-(j * b - l + 1) // s))
            assert S[j] == pytest.approx(sign * qv * (c * s + (l + 1) / 2), rel=1e-12), (sign, j)


def test_overlap_without_overlap_is_block_mean():
    """l = s = b: one window per block, the plain block-mean scores."""
    r = rng(7)
    K = r.standard_normal((64 * 9 + 5, 16))
    q = r.standard_normal(16)
    p_ovl = _ovl_params(64, 64, 64)
    p_mean = orc.OracleParams(block_size=64, top_k=1, sink_keys=0, window_keys=0, scale=0.5)
    got = orc.blocks_from_compressed(orc.block_scores(q, orc.compress(K, p_ovl), p_ovl), len(K), p_ovl)
    np.testing.assert_allclose(got, orc.block_scores(q, orc.pool_mean(K, 64), p_mean), atol=1e-14)


def test_overlap_needles_selected():
    """Needle blocks (keys pulled towards the index query) win the block
    max of their own windows, so the 32k overlapping decode slab keeps
    them."""
    w = WORKLOADS["decode_32k_overlap"].scaled(batch=1, num_kv_heads=1, num_q_heads=4, ctx_len=8192, n_needles=6)
    inp = make_inputs(w, seed=15)
    q, K, V = _slab(inp, 0, 0, w.group)
    r = orc.decode_pair(q, K, V, w.ctx_len, P(w))
    assert set(inp["needles"][0, 0].tolist()) <= set(r["sel"].selected)


# ------------------------------------------- LSA flat bucket retrieval ---

def _sse(X):
    X = np.asarray(X, float)
    return float(((X - X.mean(axis=0)) ** 2).sum())


def test_ward_cost_is_the_rise_in_sum_of_squares():
    """Ward's criterion: merging A and B raises the within-bucket sum of
    squared distances to the mean by exactly the cost (brute force)."""
    r = rng(21)
    for na, nb in [(1, 1), (1, 3), (2, 2), (3, 4), (5, 1)]:
        A, B = r.standard_normal((na, 16)), r.standard_normal((nb, 16)) + 0.3
        rise = _sse(np.vstack([A, B])) - _sse(A) - _sse(B)
        assert orc.ward_cost(A.sum(0), na, B.sum(0), nb) == pytest.approx(rise, rel=1e-10)


def _bases(n, d, seed):
    return 10.0 * orc._normalise(rng(seed).standard_normal((n, d)))


def test_ward_recovers_planted_pairs_and_quartets():
    """Tight pairs far apart are exactly the 64 buckets; tight groups of four
    (the cap) end as two buckets each, none mixing groups."""
    r = rng(22)
    perm = r.permutation(128)
    pts = np.repeat(_bases(64, 32, 23), 2, axis=0) + 1e-3 * r.standard_normal((128, 32))
    P = np.empty_like(pts)
    P[perm] = pts                                  # point i of pair i // 2 sits at perm[i]
    got = {frozenset(b) for b in orc.ward_buckets(P, 64, 4)}
    want = {frozenset((int(perm[2 * k]), int(perm[2 * k + 1]))) for k in range(64)}
    assert got == want
    pts = np.repeat(_bases(32, 32, 24), 4, axis=0) + 1e-3 * r.standard_normal((128, 32))
    P = np.empty_like(pts)
    P[perm] = pts
    group = {int(perm[i]): i // 4 for i in range(128)}
    out = orc.ward_buckets(P, 64, 4)
    assert len(out) == 64
    per_group = {}
    for b in out:
        assert len({group[m] for m in b}) == 1
        per_group[group[b[0]]] = per_group.get(group[b[0]], 0) + 1
    assert all(v == 2 for v in per_group.values()) and len(per_group) == 32


@pytest.mark.parametrize("seed,n,target,cap", [(25, 128, 64, 4), (26, 128, 64, 4), (27, 40, 20, 8), (28, 33, 17, 2)])
def test_ward_rounds_merge_mutual_cheapest_pairs(seed, n, target, cap):
    """Every round merges only pairs of buckets that are each other's
    cheapest partner within the cap (costs by brute force on the members),
    all such pairs unless that would pass the bucket target (then the
    cheapest); the result partitions the keys into `target` buckets of at
    most `cap`, ordered by their lowest member."""
    P = rng(seed).standard_normal((n, 24))
    hist = []
    out = orc.ward_buckets(P, target, cap, hist)
    for buckets, merged in hist:
        nb = len(buckets)
        cost = np.full((nb, nb), np.inf)
        for a in range(nb):
            for b in range(nb):
                if a != b and len(buckets[a]) + len(buckets[b]) <= cap:
                    cost[a, b] = _sse(P[buckets[a] + buckets[b]]) - _sse(P[buckets[a]]) - _sse(P[buckets[b]])
        best = [int(np.argmin(cost[a])) if np.isfinite(cost[a]).any() else -1 for a in range(nb)]
        mutual = {(a, best[a]) for a in range(nb) if best[a] > a and best[best[a]] == a}
        assert set(merged) <= mutual
        if len(merged) < len(mutual):
            assert nb - len(merged) == target
            worst = max(cost[a, b] for a, b in merged)
            assert all(cost[a, b] >= worst - 1e-12 for a, b in mutual - set(merged))
    flat = sorted(m for b in out for m in b)
    assert flat == list(range(n)) and len(out) == target
    assert all(len(b) <= cap and b == sorted(b) for b in out)
    assert [b[0] for b in out] == sorted(b[0] for b in out)


def _lsa_params(**kw):
    base = dict(block_size=512, top_k=4, sink_keys=4, window_keys=512, pool="lsa", pool_stride=4)
    base.update(kw)
    return orc.OracleParams(**base)


def test_bucket_index_covers_blocks_and_ignores_key_scale():
    """The bucket cache of the complete cluster blocks: every pool key of
    them in exactly one bucket, 64 per block, unit centroids; scaling raw
    keys by positive factors (which the L2 normalisation removes) changes
    nothing."""
    r = rng(29)
    C = 512 * 3 + 100
    K = r.standard_normal((C, 32))
    p = _lsa_params()
    members, cents = orc.lsa_bucket_index(K, C, p)
    assert len(members) == 3 * 64
    assert sorted(m for b in members for m in b) == list(range(3 * 128))
    assert all(len(b) <= 4 for b in members)
    assert np.allclose(np.linalg.norm(cents, axis=1), 1.0)
    members2, cents2 = orc.lsa_bucket_index(K * r.uniform(0.1, 10.0, (C, 1)), C, p)
    assert members2 == members
    np.testing.assert_allclose(cents2, cents, atol=1e-12)


def test_bucket_decode_with_every_bucket_is_dense_attention():
    """With k above the number of candidate buckets and a context of whole
    cluster blocks, the attended set is every key: library dense attention
    (torch SDPA in float64); also for a 3-token chunk."""
    r = rng(30)
    C, d = 512 * 3, 32
    K, V = r.standard_normal((C + 3, d)), r.standard_normal((C + 3, d))
    q = r.standard_normal((3, 2, d))
    res = orc.bucket_decode_pair(q, K, V, C, _lsa_params(top_k=10_000))
    assert len(res["sel"].selected) == len(res["candidates"]) == 2 * 64     # the last block is the window
    for j in range(3):
        for g in range(2):
            np.testing.assert_allclose(res["O"][j, g], _sdpa(q[j, g], K, V, C + j + 1), atol=1e-12)


def test_bucket_decode_selects_a_planted_needle_and_keeps_the_budget():
    """Eight raw keys (two pool keys) pulled towards the query in an early
    cluster block land in the selected buckets; with a budget of N keys only
    the N / 4 member pool keys of best own cosine stay, every kept one at
    least as good as every dropped one."""
    r = rng(31)
    C, d = 512 * 6, 64
    K, V = r.standard_normal((C + 1, d)), r.standard_normal((C + 1, d))
    q = r.standard_normal((1, 4, d))
    u = q[0].mean(axis=0)
    needle = list(range(512 + 100, 512 + 108))
    K[needle] = 0.5 * u * 4 + 0.3 * r.standard_normal((8, d))
    res = orc.bucket_decode_pair(q, K, V, C, _lsa_params(top_k=6))
    assert set(needle) <= set(res["positions"][0].tolist())
    full = res["kept"]
    res2 = orc.bucket_decode_pair(q, K, V, C, _lsa_params(top_k=6, bucket_keys=16))
    kept = res2["kept"]
    assert len(kept) == min(4, len(full)) and set(kept) <= set(full)
    P = orc.lsa_pool_keys(K[:C])
    qhat = orc._normalise(q[0].sum(axis=0))
    own = {m: float(orc._normalise(P[m]) @ qhat) for m in full}
    assert min(own[m] for m in kept) >= max([own[m] for m in set(full) - set(kept)] + [-2.0])


def test_bucket_decode_before_the_first_cluster_block():
    """A context shorter than one cluster block has no pool keys, no buckets
    and nothing to select: with a window covering it, every key is attended
    (library dense attention); with none, only the sink and the chunk."""
    r = rng(62)
    C, d = 300, 16
    K, V = r.standard_normal((C + 2, d)), r.standard_normal((C + 2, d))
    q = r.standard_normal((2, 2, d))
    assert orc.lsa_pool_keys(K[:0]).shape == (0, d)
    res = orc.bucket_decode_pair(q, K, V, C, _lsa_params(top_k=8))
    assert res["members"] == [] and res["kept"] == [] and res["sel"].selected == []
    for j in range(2):
        for g in range(2):
            np.testing.assert_allclose(res["O"][j, g], _sdpa(q[j, g], K, V, C + j + 1), atol=1e-12)
    res = orc.bucket_decode_pair(q, K, V, C, _lsa_params(top_k=8, window_keys=0))
    assert res["positions"][1].tolist() == [0, 1, 2, 3, C, C + 1]


@pytest.mark.parametrize("stride", [2, 4, 8])
def test_bucket_candidates_by_key_enumeration(stride):
    """A bucket is a candidate iff one of its raw keys lies outside sink and
    window, for any pool stride: expected sets built key by key (raw key t
    belongs to pool key t // stride, which belongs to one bucket), with a
    sink and a window that cut through buckets."""
    r = rng(60 + stride)
    b, d = 512, 16
    C = 3 * b
    K, V = r.standard_normal((C + 1, d)), r.standard_normal((C + 1, d))
    q = r.standard_normal((1, 2, d))
    p = _lsa_params(pool_stride=stride, sink_keys=6, window_keys=300, top_k=10_000)
    res = orc.bucket_decode_pair(q, K, V, C, p)
    owner = {}
    for g, ids in enumerate(res["members"]):
        for m in ids:
            owner[m] = g
    expected = set()
    for t in range(C):
        if 6 <= t < C - 300:
            expected.add(owner[t // stride])
    assert sorted(expected) == res["candidates"]
    assert all(len(ids) <= 16 // stride for ids in res["members"])
    # every candidate selected: every key of the context is attended (dense)
    for g in range(2):
        np.testing.assert_allclose(res["O"][0, g], _sdpa(q[0, g], K, V, C + 1), atol=1e-12)


# ---------------------------------------------- planted-mistake checks ---

# ------------------------------------------------------------ dense verify ---

def _verify_case(seed=21, C=2048 + 37, n_q=3, G=2):
    w = WORKLOADS["draft_chunk_16k"].scaled(batch=1, num_kv_heads=1, num_q_heads=G, n_q=n_q,
                                            ctx_len=C, top_k=5)
    inp = make_inputs(w, seed=seed)
    q, K, V = _slab(inp, 0, 0, w.group)
    return w, inp, q, K, V


def test_verify_mass_equals_library_softmax_block_sums():
    """Block mass = block sums of the weights torch.softmax gives each
    (token, head) over its causally visible keys (a library routine of the
    same definition); O and lse equal library dense attention."""
    w, inp, q, K, V = _verify_case()
    C, b = w.ctx_len, w.block_size
    r = orc.verify_pair(q, K, V, C, P(w))
    nb = C // b
    mass = torch.zeros(nb, dtype=torch.float64)
    Kt, scale = torch.from_numpy(K), 1.0 / math.sqrt(128)
    for j in range(w.n_q):
        n = C + j + 1
        for g in range(w.group):
            z = Kt[:n] @ torch.from_numpy(q[j, g]) * scale
            wt = torch.softmax(z, dim=0)
            mass += wt[:nb * b].reshape(nb, b).sum(dim=1)
            np.testing.assert_allclose(r["O"][j, g], _sdpa(q[j, g], K, V, n), atol=1e-12)
            assert abs(r["lse"][j, g] - logsumexp(z.numpy())) < 1e-12
    np.testing.assert_allclose(r["mass"], mass.numpy(), atol=1e-12, rtol=0)


def test_verify_mass_total_needle_and_full_k():
    """Weights of every (token, head) sum to one, so the block masses plus the
    weight on the keys past the complete blocks total n_q * G; a block whose
    keys point along the chunk's queries takes the most mass and is
    selected; k >= #candidates selects every candidate."""
    w, inp, q, K, V = _verify_case(seed=22)
    C, b = w.ctx_len, w.block_size
    jn = 17
    K = K.copy()
    K[jn * b:(jn + 1) * b] += 3.0 * q.reshape(-1, 128).mean(axis=0)
    r = orc.verify_pair(q, K, V, C, P(w))
    assert abs(r["mass"].sum() + r["wtail"].sum() - w.n_q * w.group) < 1e-12
    assert int(np.argmax(r["mass"])) == jn and jn in r["sel"].selected
    assert len(r["sel"].selected) == 5
    r_all = orc.verify_pair(q, K, V, C, P(w, top_k=10_000))
    assert r_all["sel"].selected == orc.candidate_blocks(C, P(w))


# ------------------------------------------------------------ column-sparse ---

_COLP = orc.OracleParams(block_size=64, top_k=0, sink_keys=0, window_keys=0)


def _col_case(seed=31, T=300, G=4):
    r = rng(seed)
    q = r.standard_normal((64, G, 128))
    K = r.standard_normal((T, 128))
    V = r.standard_normal((T, 128))
    return q, K, V


def test_column_attention_all_columns_is_library_bidirectional_attention():
    """Every key kept: plain bidirectional attention (torch SDPA without a
    mask), whatever the order of the list or its duplicates."""
    q, K, V = _col_case()
    T = len(K)
    cols = list(range(T))[::-1] + [5, 5, -1]
    r = orc.column_attention_group(q, K, V, cols, _COLP)
    for i in (0, 17, 63):
        for g in range(4):
            np.testing.assert_allclose(r["O"][i, g], _sdpa(q[i, g], K, V, T), atol=1e-12)
            z = K @ q[i, g] / math.sqrt(128)
            assert abs(r["lse"][i, g] - logsumexp(z)) < 1e-12


def test_column_attention_subset_and_edge_cases():
    """A subset of columns equals library attention over those rows only
    (keys after the query included); one column gives that column's V; an
    empty list gives O = 0 and lse = -inf."""
    q, K, V = _col_case(seed=32)
    cols = [3, 250, 7, 299, 120, 64]
    r = orc.column_attention_group(q, K, V, cols, _COLP)
    sub = sorted(cols)
    for i in (0, 40):
        for g in (0, 3):
            ref = _sdpa(q[i, g], K[sub], V[sub], len(sub))
            np.testing.assert_allclose(r["O"][i, g], ref, atol=1e-12)
    one = orc.column_attention_group(q, K, V, [42], _COLP)
    np.testing.assert_allclose(one["O"][5, 1], V[42], atol=1e-12)
    assert abs(one["lse"][5, 1] - float(K[42] @ q[5, 1]) / math.sqrt(128)) < 1e-12
    none = orc.column_attention_group(q, K, V, [-1, -1], _COLP)
    assert np.all(none["O"] == 0) and np.all(np.isneginf(none["lse"]))


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible mistake planted in the oracle makes some pin fail."""
    orig_pool_ovl = orc.pool_overlap
    mistakes = {
        "mean instead of sum over the GQA group":
            ("index_query", lambda qg: np.asarray(qg, float).mean(axis=0),
             test_scores_brute_force_loops),
        "LSA pooling without key normalisation":
            ("pool_lsa", lambda K, b, stride=4: orc._normalise(
                np.asarray(K, float)[:(len(K) // b) * b].reshape(len(K) // b, b, -1).sum(1)),
             test_pool_lsa_invariants),
        "ties broken towards the higher index":
            ("select_topk", lambda s, c, k: orc.Selection(
                sorted(sorted(c, key=lambda j: (-float(s[j]), -j))[:min(k, len(c))]), len(c), None, None, False),
             test_topk_matches_exhaustive_rank_count),
        "window dropped from the attended set":
            ("attended_positions", lambda C, p, sel, last: np.flatnonzero(np.isin(
                np.arange(last + 1),
                list(range(min(p.sink_keys, C))) + [t for j in sel for t in range(j * p.block_size, (j + 1) * p.block_size)]
                + list(range(C, last + 1)))),
             test_sink_window_always_attended_and_chunk_causal),
    }
    for what, (name, bad, pin) in mistakes.items():
        with monkeypatch.context() as m:
            m.setattr(orc, name, bad)
            assert _fails(pin), f"no pin caught: {what}"
    # scale 1/d instead of 1/sqrt(d): the hand-worked example catches it
    with monkeypatch.context() as m:
        m.setattr(orc, "softmax_scale", lambda d, p: 1.0 / d)
        assert _fails(lambda: test_hand_worked_decode("decode_k1"))
    # verify mass of the first token only, or without the causal mask
    orig_verify = orc.verify_pair

    def mass_first_token(q, K, V, C, p):
        r = orig_verify(q, K, V, C, p)
        r["mass"] = orig_verify(q[:1], K, V, C, p)["mass"]
        return r
    for bad in (mass_first_token,
                lambda q, K, V, C, p: _verify_noncausal(q, K, V, C, p)):
        with monkeypatch.context() as m:
            m.setattr(orc, "verify_pair", bad)
            assert _fails(test_verify_mass_equals_library_softmax_block_sums)
    # a causal mask applied to the column-sparse attention
    orig_col = orc.column_attention_group

    def causal_cols(q, K, V, cols, p):
        r = orig_col(q, K, V, [c for c in cols if 0 <= c <= 63], p)
        return r
    with monkeypatch.context() as m:
        m.setattr(orc, "column_attention_group", causal_cols)
        assert _fails(test_column_attention_subset_and_edge_cases)
    # overlapping compression: windows inside the block only, incomplete
    # windows kept, the sum over the stride instead of the mean over the window
    orig_b2c = orc.blocks_from_compressed

    def contained_only(sigma, C, p):
        b, l, s_ = p.block_size, p.pool_kernel, p.pool_stride
        st = np.arange(len(sigma)) * s_
        return np.array([np.max(np.asarray(sigma)[(st >= j * b) & (st + l <= (j + 1) * b)])
                         for j in range(C // b)])

    def with_partial(K, kernel, stride):
        K = np.asarray(K, float)
        return np.stack([K[c:c + kernel].mean(0) for c in range(0, len(K) - stride + 1, stride)])
    ovl = lambda: [test_overlap_block_scores_closed_form(*c) for c in _OVL_CASES]
    for name, bad in (("blocks_from_compressed", contained_only),
                      ("pool_overlap", with_partial),
                      ("pool_overlap", lambda K, l, s_: orig_pool_ovl(K, l, s_) * l / s_)):
        with monkeypatch.context() as m:
            m.setattr(orc, name, bad)
            assert _fails(ovl), name
    assert orig_b2c is orc.blocks_from_compressed
    # prefill with overlapping windows: the context's windows counted like
    # its blocks, or windows reaching past the context kept
    for bad in (lambda C, p: C // p.block_size,
                lambda C, p: (C - p.pool_stride) // p.pool_stride + 1 if p.pool == "overlap" else C // p.block_size):
        with monkeypatch.context() as m:
            m.setattr(orc, "context_rows", bad)
            assert _fails(lambda: test_prefill_overlap_tile_scores_brute_force(8, 6, 2)), "context_rows"
    # Ward clustering: centroid distance without the size weights; every
    # bucket merging with its cheapest partner whether or not that is mutual;
    # the size cap ignored
    with monkeypatch.context() as m:
        m.setattr(orc, "ward_cost", lambda sa, na, sb, nb: float(((sa / na - sb / nb) ** 2).sum()))
        assert _fails(test_ward_cost_is_the_rise_in_sum_of_squares)
    orig_wb = orc.ward_buckets

    def greedy(P, n_buckets, cap, history=None):
        P = np.asarray(P, float)
        buckets = [[i] for i in range(len(P))]
        while len(buckets) > n_buckets:
            nb = len(buckets)
            used, merged = set(), []
            for a in range(nb):
                if a in used:
                    continue
                cands = [b for b in range(nb) if b != a and b not in used and len(buckets[a]) + len(buckets[b]) <= cap]
                if not cands or nb - len(merged) <= n_buckets:
                    continue
                b = min(cands, key=lambda b: (orc.ward_cost(P[buckets[a]].sum(0), len(buckets[a]), P[buckets[b]].sum(0), len(buckets[b])), b))
                used.update((a, b))
                merged.append((a, b))
            if history is not None:
                history.append(([list(x) for x in buckets], merged))
            buckets = sorted([bk for i, bk in enumerate(buckets) if i not in used]
                             + [sorted(buckets[a] + buckets[b]) for a, b in merged], key=lambda x: x[0])
        return buckets
    for bad in (greedy, lambda P, n, cap, history=None: orig_wb(P, n, 10 ** 6, history)):
        with monkeypatch.context() as m:
            m.setattr(orc, "ward_buckets", bad)
            assert _fails(lambda: test_ward_rounds_merge_mutual_cheapest_pairs(25, 128, 64, 4))
    # summed chunk queries instead of the chunk's first query for selection
    with monkeypatch.context() as m:
        m.setattr(orc, "index_query", lambda qg: np.asarray(qg, float).sum(axis=0) * 0.0)
        assert _fails(test_needles_selected_tiny_decode)


def _verify_noncausal(q, K, V, C, p):
    """verify_pair with every token seeing the whole chunk (a planted mistake)."""
    n_q, G, d = q.shape
    b = p.block_size
    nb = C // b
    scale = orc.softmax_scale(d, p)
    O, lse, mass = np.zeros((n_q, G, d)), np.zeros((n_q, G)), np.zeros(nb)
    pos = np.arange(C + n_q)
    for j in range(n_q):
        for g in range(G):
            O[j, g], lse[j, g], wt = orc.masked_softmax_attention(q[j, g], K, V, pos, scale)
            mass += wt[:nb * b].reshape(nb, b).sum(axis=1)
    return dict(O=O, lse=lse, mass=mass, wtail=None, candidates=None, sel=None)
