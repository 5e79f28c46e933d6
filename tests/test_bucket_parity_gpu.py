"""GPU parity of LSA flat bucket retrieval (sa_bucket_build, sa_bucket_decode)
against the float64 oracle (LSA review §2.2-2.3, reading R19).

Bucket partitions are compared exactly, block by block; a block may differ
only where one of the oracle's own Ward decisions is a near-tie (two partner
costs, or the last round's cut, within 1e-5 relative), and such blocks are
counted.  Selected buckets follow the selection rule of the block path (a
near-tie is a k-th / (k+1)-th score gap below 1e-4 |s_k|), kept pool keys the
same rule on their own cosines at the cut.  Outputs: fp32 inputs max abs
<= 1e-5, bf16 inputs max abs <= 5e-3 and relative L2 <= 1e-2 (fp32 outputs).
"""
import math

import numpy as np
import pytest
import torch

from helpers import assert_close, compare_sets, oracle_params, slab
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")

WARD_TIE_REL = 1e-5


def ward_min_gap(P, n_buckets, cap):
    """Smallest relative gap among the decisions of the oracle's Ward rounds
    on one block: each bucket's cheapest against its second-cheapest allowed
    partner, and, in a round that merges only part of its mutual pairs, the
    last merged pair against the first one left out."""
    hist = []
    orc.ward_buckets(P, n_buckets, cap, history=hist)
    gap = math.inf
    for buckets, merged in hist:
        nb = len(buckets)
        sums = np.stack([P[b].sum(axis=0) for b in buckets])
        size = np.array([len(b) for b in buckets], dtype=np.float64)
        cost = orc.ward_cost(sums[:, None, :], size[:, None], sums[None, :, :], size[None, :])
        cost = np.where((size[:, None] + size[None, :] <= cap) & ~np.eye(nb, dtype=bool), cost, math.inf)
        best = []
        for a in range(nb):
            row = np.sort(cost[a][np.isfinite(cost[a])])
            if len(row) >= 2:
                gap = min(gap, (row[1] - row[0]) / max(row[0], 1e-30))
            best.append(int(np.argmin(cost[a])) if len(row) else -1)
        mutual = sorted((float(cost[a, best[a]]), a) for a in range(nb)
                        if best[a] > a and best[best[a]] == a)
        if len(mutual) > len(merged) > 0:
            c0, c1 = mutual[len(merged) - 1][0], mutual[len(merged)][0]
            gap = min(gap, (c1 - c0) / max(c0, 1e-30))
    return gap


def build(w, inp, p):
    R = sa.bucket_rows(p)
    mcap = 16 // w.pool_stride
    cents = torch.full((w.batch, w.num_kv_heads, R, 128), float("nan"), device="cuda")
    members = torch.full((w.batch, w.num_kv_heads, R, mcap), -7, device="cuda", dtype=torch.int32)
    sa.bucket_build(p, inp["K"], cents, members)
    return cents, members


def gpu_buckets(members, b, h, nblk, nbk):
    rows = members[b, h, :nblk * nbk].cpu().numpy()
    return [[int(x) for x in r if x >= 0] for r in rows]


def check_partitions(w, inp, cents, members, pairs):
    """Per pair: the GPU buckets of every complete cluster block against the
    oracle's Ward clustering; centroids of matching blocks within 2e-6."""
    b, stride = w.block_size, w.pool_stride
    m, nbk, mcap = b // stride, b // 8, 16 // stride
    nblk = w.ctx_len // b
    near = 0
    for (bi, h) in pairs:
        K = inp["K"][bi, h, :nblk * b].double().cpu().numpy()
        P = orc.lsa_pool_keys(K, stride)
        got = gpu_buckets(members, bi, h, nblk, nbk)
        for c in range(nblk):
            Pc = P[c * m:(c + 1) * m]
            ref = [[c * m + i for i in bk] for bk in orc.ward_buckets(Pc, nbk, mcap)]
            mine = got[c * nbk:(c + 1) * nbk]
            if mine != ref:
                gap = ward_min_gap(Pc, nbk, mcap)
                assert gap < WARD_TIE_REL, (bi, h, c, gap)
                near += 1
                continue
            ref_c = orc._normalise(np.stack([P[ids].sum(axis=0) for ids in ref]))
            got_c = cents[bi, h, c * nbk:(c + 1) * nbk].double().cpu().numpy()
            np.testing.assert_allclose(got_c, ref_c, atol=2e-6)
    return near


@pytest.mark.parametrize("dtype,stride,b", [("bf16", 4, 512), ("f32", 4, 512), ("bf16", 2, 256),
                                            ("bf16", 1, 128)])
def test_bucket_build_matches_oracle_partitions(dtype, stride, b):
    w = WORKLOADS["decode_1m_buckets"].scaled(batch=1, num_q_heads=8, num_kv_heads=2, ctx_len=4 * b + 37,
                                              dtype=dtype, block_size=b, pool_stride=stride, n_needles=1,
                                              top_k=8)
    cap = 6 * b
    inp = make_inputs(w, seed=40 + stride, device="cuda", kv_capacity=cap)
    p = sa.params_for(w, kv_capacity=cap)
    cents, members = build(w, inp, p)
    torch.cuda.synchronize()
    near = check_partitions(w, inp, cents, members, [(0, 0), (0, 1)])
    print(f"\nbuckets {dtype} stride {stride} b {b}: {near} near-tie blocks of 8")
    # rows of cluster blocks past the context are left untouched
    nbk = b // 8
    assert bool(torch.isnan(cents[:, :, 4 * nbk:]).all())
    assert bool((members[:, :, 4 * nbk:] == -7).all())
    # every complete block: a partition of its pool keys into b / 8 buckets
    mm = members[:, :, :4 * nbk].cpu().numpy()
    m = b // stride
    for bi in range(1):
        for h in range(2):
            for c in range(4):
                ids = mm[bi, h, c * nbk:(c + 1) * nbk].ravel()
                assert sorted(int(x) for x in ids if x >= 0) == list(range(c * m, (c + 1) * m))


def test_bucket_build_streams_block_by_block():
    """Blocks built later (first_block > 0, after the context grew) equal a
    single build of the whole context, and earlier rows are left alone."""
    w = WORKLOADS["decode_1m_buckets"].scaled(batch=1, num_q_heads=4, num_kv_heads=2, ctx_len=5 * 512 + 11,
                                              n_needles=1)
    cap = 8 * 512
    inp = make_inputs(w, seed=44, device="cuda", kv_capacity=cap)
    p_all = sa.params_for(w, kv_capacity=cap)
    c_all, m_all = build(w, inp, p_all)
    p_two = sa.params_for(w.scaled(ctx_len=2 * 512 + 5), kv_capacity=cap)
    c_inc, m_inc = build(w, inp, p_two)
    sa.bucket_build(p_all, inp["K"], c_inc, m_inc, first_block=2)
    torch.cuda.synchronize()
    assert torch.equal(m_inc[:, :, :5 * 64], m_all[:, :, :5 * 64])
    assert torch.equal(c_inc[:, :, :5 * 64], c_all[:, :, :5 * 64])


def own_gap(K, C, p, q, full, keep):
    """Relative gap of the oracle's own cosines at the expansion cut."""
    P = orc.lsa_pool_keys(K[:(C // p.block_size) * p.block_size], p.pool_stride)
    qhat = orc._normalise(orc.index_query(q[0]))
    own = sorted((float(orc._normalise(P[m]) @ qhat) for m in full), reverse=True)
    if len(own) <= keep:
        return math.inf
    return (own[keep - 1] - own[keep]) / max(abs(own[keep - 1]), 1e-30)


def run_bucket_decode(w, inp, p, cents, members, bucket_keys, out_dtype=torch.float32):
    mcap = 16 // w.pool_stride
    n_ent = w.top_k * mcap
    kcap = min(bucket_keys // w.pool_stride, n_ent) if bucket_keys > 0 else n_ent
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device="cuda", dtype=out_dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device="cuda")
    sel = torch.empty((w.batch, w.num_kv_heads, w.top_k), device="cuda", dtype=torch.int32)
    kept = torch.empty((w.batch, w.num_kv_heads, kcap), device="cuda", dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_BUCKET_DECODE)
    sa.bucket_decode(p, inp["Q"], inp["K"], inp["V"], cents, members, O, lse, sel, kept, bucket_keys, ws)
    assert sa.read_status(ws) == sa.SA_OK
    return O, lse, sel, kept


def check_bucket_decode(w, seed, bucket_keys, pairs=None):
    inp = make_inputs(w, seed=seed, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    cents, members = build(w, inp, p)
    O, lse, sel, kept = run_bucket_decode(w, inp, p, cents, members, bucket_keys)
    torch.cuda.synchronize()
    G = w.group
    op = oracle_params(w, bucket_keys=bucket_keys)
    nblk, nbk = w.ctx_len // w.block_size, w.block_size // 8
    pairs = pairs or [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    stats = dict(match=0, near=0)
    for (bi, h) in pairs:
        q, K, V = slab(inp, bi, h, G, w.kv_len)
        res = orc.bucket_decode_pair(q, K, V, w.ctx_len, op)
        if gpu_buckets(members, bi, h, nblk, nbk) != res["members"]:
            stats["near"] += 1                      # partition near-tie (checked in the build tests)
            continue
        verdict = compare_sets(sel[bi, h].cpu().numpy(), res["sel"])
        assert verdict != "mismatch", (bi, h, sel[bi, h].tolist(), res["sel"].selected)
        if verdict == "near_tie":
            stats["near"] += 1
            continue
        got_kept = [int(x) for x in kept[bi, h].tolist() if x >= 0]
        assert got_kept == sorted(set(got_kept))
        if got_kept != res["kept"]:
            full = sorted(mm for g in res["sel"].selected for mm in res["members"][g])
            gap = own_gap(K, w.ctx_len, op, q, full, bucket_keys // w.pool_stride)
            assert gap < 1e-4, (bi, h, gap)
            stats["near"] += 1
            continue
        assert_close(O[bi, :, h * G:(h + 1) * G], res["O"], w.dtype, f"O pair {(bi, h)}")
        lse_err = np.abs(lse[bi, :, h * G:(h + 1) * G].double().cpu().numpy() - res["lse"]).max()
        assert lse_err < (2e-5 if w.dtype == "f32" else 2e-4), lse_err
        stats["match"] += 1
    print(f"\n{w.name} bucket decode: {stats}")
    assert stats["match"] >= len(pairs) // 2
    return stats


@pytest.mark.parametrize("dtype,n_q,bucket_keys", [("bf16", 1, 64), ("bf16", 1, 0), ("f32", 1, 64),
                                                   ("bf16", 3, 64), ("f32", 2, 0)])
def test_bucket_decode_matches_oracle(dtype, n_q, bucket_keys):
    """Selection, expansion and attention against the oracle on contexts of
    8 cluster blocks plus a ragged tail (the window cuts the last block, the
    4-key sink lies inside a bucket of the first)."""
    w = WORKLOADS["decode_1m_buckets"].scaled(batch=2, num_q_heads=8, num_kv_heads=2, n_q=n_q,
                                              ctx_len=512 * 8 + 37, dtype=dtype, top_k=12, n_needles=2)
    check_bucket_decode(w, seed=50 + n_q, bucket_keys=bucket_keys)


def test_bucket_decode_every_bucket_is_dense():
    """top_k above the number of candidate buckets and a window covering the
    tail: every key is attended, so the result is the library-independent
    dense attention of the oracle (and no bucket selection is a near-tie)."""
    w = WORKLOADS["decode_1m_buckets"].scaled(batch=1, num_q_heads=4, num_kv_heads=1, ctx_len=512 * 4,
                                              dtype="f32", top_k=1024 // 4, n_needles=0, sink_keys=4,
                                              window_keys=512)
    inp = make_inputs(w, seed=57, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    cents, members = build(w, inp, p)
    O, lse, sel, kept = run_bucket_decode(w, inp, p, cents, members, 0)
    torch.cuda.synchronize()
    q, K, V = slab(inp, 0, 0, w.group, w.kv_len)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0])[None, :, None], torch.from_numpy(K)[None, None].expand(1, w.group, -1, -1),
        torch.from_numpy(V)[None, None].expand(1, w.group, -1, -1))[0, :, 0].numpy()     # library, float64
    assert_close(O[0, 0], ref, "f32", "dense")
    # every candidate is selected: the buckets of the first three blocks
    # except one holding only the 4 sink keys (the last block is the window)
    res = orc.bucket_decode_pair(q, K, V, w.ctx_len, oracle_params(w))
    assert [int(x) for x in sel[0, 0].tolist() if x >= 0] == res["sel"].selected == res["candidates"]
    assert len(res["candidates"]) in (3 * 64 - 1, 3 * 64)


def test_bucket_decode_without_buckets():
    """top_k = 0, and a context without a complete cluster block: the
    attended set is sink, window and the chunk."""
    for over in (dict(top_k=0, ctx_len=512 * 3 + 9), dict(top_k=8, ctx_len=300)):
        w = WORKLOADS["decode_1m_buckets"].scaled(batch=1, num_q_heads=4, num_kv_heads=2, n_q=2, dtype="f32",
                                                  n_needles=0, **over)
        inp = make_inputs(w, seed=58, device="cuda")
        p = sa.params_for(w, out_dtype="f32")
        cents, members = build(w, inp, p)
        O, lse, sel, kept = run_bucket_decode(w, inp, p, cents, members, 64)
        torch.cuda.synchronize()
        for h in range(2):
            q, K, V = slab(inp, 0, h, w.group, w.kv_len)
            res = orc.bucket_decode_pair(q, K, V, w.ctx_len, oracle_params(w, bucket_keys=64))
            assert res["kept"] == []
            assert_close(O[0, :, h * w.group:(h + 1) * w.group], res["O"], "f32", f"{over} head {h}")


def _ward_block(args):
    Pc, n_buckets, cap = args
    return orc.ward_buckets(Pc, n_buckets, cap)


def test_bucket_decode_full_size_sampled():
    """The 1M-token bucket workload at full size (4 sequences x 8 KV heads,
    2048 cluster blocks each): every block's buckets form a partition of its
    pool keys; for one sampled pair the oracle clusters all 2048 blocks (in
    spawned worker processes) and the partitions, the selected buckets, the
    kept pool keys and the outputs are compared as in the small cases."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os

    w = WORKLOADS["decode_1m_buckets"]
    inp = make_inputs(w, seed=59, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    cents, members = build(w, inp, p)
    bucket_keys = 2048
    O, lse, sel, kept = run_bucket_decode(w, inp, p, cents, members, bucket_keys)
    torch.cuda.synchronize()
    b, stride = w.block_size, w.pool_stride
    m, nbk, mcap = b // stride, b // 8, 16 // stride
    nblk = w.ctx_len // b
    # partitions of every block of every pair (a property that holds at any size)
    mm = members[:, :, :nblk * nbk].reshape(w.batch * w.num_kv_heads, nblk, nbk * mcap)
    srt = torch.sort(mm, dim=-1).values[..., nbk * mcap - m:]
    base = (torch.arange(nblk, device="cuda") * m)[None, :, None]
    assert bool((srt.long() == base + torch.arange(m, device="cuda")[None, None, :]).all())
    n_kept = (kept >= 0).sum(-1)
    assert bool((sel >= 0).all()) and bool((n_kept > 0).all()) and bool((n_kept <= bucket_keys // stride).all())
    # one pair against the oracle
    bi, h = 2, 5
    q, K, V = slab(inp, bi, h, w.group, w.kv_len)
    P = orc.lsa_pool_keys(K[:nblk * b], stride)
    jobs = [(P[c * m:(c + 1) * m], nbk, mcap) for c in range(nblk)]
    with cf.ProcessPoolExecutor(max_workers=min(32, os.cpu_count() or 1),
                                mp_context=mp.get_context("spawn")) as ex:
        blocks = list(ex.map(_ward_block, jobs, chunksize=16))
    ref_members = [[c * m + i for i in bk] for c, bks in enumerate(blocks) for bk in bks]
    got = gpu_buckets(members, bi, h, nblk, nbk)
    differ = [c for c in range(nblk) if got[c * nbk:(c + 1) * nbk] != ref_members[c * nbk:(c + 1) * nbk]]
    for c in differ:
        assert ward_min_gap(P[c * m:(c + 1) * m], nbk, mcap) < WARD_TIE_REL, c
    print(f"\n1M buckets, pair {(bi, h)}: {len(differ)} of {nblk} blocks differ at Ward near-ties")
    if differ:
        return
    ref_cents = orc._normalise(np.stack([P[ids].sum(axis=0) for ids in ref_members]))
    np.testing.assert_allclose(cents[bi, h, :nblk * nbk].double().cpu().numpy(), ref_cents, atol=2e-6)
    op = oracle_params(w, bucket_keys=bucket_keys)
    res = orc.bucket_decode_pair(q, K, V, w.ctx_len, op, index=(ref_members, ref_cents))
    verdict = compare_sets(sel[bi, h].cpu().numpy(), res["sel"])
    assert verdict != "mismatch"
    if verdict == "near_tie":
        return
    got_kept = [int(x) for x in kept[bi, h].tolist() if x >= 0]
    if got_kept != res["kept"]:
        full = sorted(x for g in res["sel"].selected for x in res["members"][g])
        assert own_gap(K, w.ctx_len, op, q, full, bucket_keys // stride) < 1e-4
        return
    G = w.group
    assert_close(O[bi, :, h * G:(h + 1) * G], res["O"], "bf16", "1M bucket decode")
