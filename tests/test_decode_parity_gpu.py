"""GPU parity of the decode / draft-chunk path against the float64 oracle.

Every case draws seeded inputs on the GPU, runs the CUDA library through the
C ABI, copies the same inputs to the host and runs the oracle on them.
Bars (bf16 inputs, fp32 accumulation): max abs <= 5e-3 and relative L2 <=
1e-2; fp32 inputs: max abs <= 1e-5.  Selected block sets must be identical
except where the oracle's k-th/(k+1)-th gap is a near-tie (< 1e-4 |s_k|);
such pairs are counted and reported.
"""
import numpy as np
import pytest
import torch

from helpers import (assert_close, compare_sets, errors, oracle_decode, oracle_params, slab)
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")


def dev_inputs(w, seed, kv_capacity=None):
    return make_inputs(w, seed=seed, device="cuda", kv_capacity=kv_capacity)


def run_pool(w, inp, p):
    nb = w.ctx_len // w.block_size
    Kc = torch.empty((w.batch, w.num_kv_heads, nb, 128), device="cuda", dtype=torch.float32)
    sa.pool_keys(p, inp["K"], Kc)
    return Kc


def run_decode(w, inp, p, Kc, out_dtype=torch.float32):
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device="cuda", dtype=out_dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device="cuda", dtype=torch.float32)
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device="cuda", dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_DECODE)
    sa.sparse_attn_decode(p, inp["Q"], inp["K"], inp["V"], Kc, O, lse, idx, ws)
    assert sa.read_status(ws) == sa.SA_OK
    return O, lse, idx, ws


def all_pairs(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


def check_decode(w, seed, pairs=None, out_dtype=torch.float32, p_over=None):
    inp = dev_inputs(w, seed)
    p = sa.params_for(w, out_dtype="bf16" if out_dtype == torch.bfloat16 else "f32")
    if p_over:
        for k, v in p_over.items():
            setattr(p, k, v)
    Kc = run_pool(w, inp, p)
    O, lse, idx, _ = run_decode(w, inp, p, Kc, out_dtype)
    torch.cuda.synchronize()
    pairs = pairs or all_pairs(w)
    op = oracle_params(w, **({"top_k": p_over["top_k"]} if p_over and "top_k" in p_over else {}))
    ref = oracle_decode(w, inp, pairs, op)
    G = w.group
    n_match = n_tie = 0
    for (b, h), r in ref.items():
        # compressed keys
        np.testing.assert_allclose(Kc[b, h].double().cpu().numpy(), r["Kc"], atol=2e-6, rtol=1e-5)
        verdict = compare_sets(idx[b, h].cpu().numpy(), r["sel"])
        assert verdict != "mismatch", (b, h, idx[b, h].tolist(), r["sel"].selected)
        if verdict == "near_tie":
            n_tie += 1
            continue
        n_match += 1
        dt = "f32" if (w.dtype == "f32" and out_dtype == torch.float32) else "bf16"
        assert_close(O[b, :, h * G:(h + 1) * G], r["O"], dt, f"O pair {(b, h)}")
        lse_err = np.abs(lse[b, :, h * G:(h + 1) * G].double().cpu().numpy() - r["lse"]).max()
        assert lse_err < (2e-5 if w.dtype == "f32" else 2e-4), lse_err
    print(f"\n{w.name}: {n_match} pairs matched, {n_tie} near-ties")
    return inp, p, Kc, O, lse, idx


# ------------------------------------------------------------------ pooling --

@pytest.mark.parametrize("dtype,pool,b,C", [("bf16", "mean", 64, 64 * 37 + 19), ("f32", "mean", 64, 64 * 21),
                                            ("bf16", "lsa", 512, 512 * 9 + 100), ("f32", "lsa", 128, 128 * 5),
                                            ("bf16", "mean", 16, 16 * 50 + 3)])
def test_pool_keys_parity(dtype, pool, b, C):
    w = WORKLOADS["decode_32k"].scaled(batch=2, num_q_heads=8, num_kv_heads=2, ctx_len=C, dtype=dtype,
                                       pool=pool, block_size=b, n_needles=2, sink_keys=b, window_keys=b)
    inp = dev_inputs(w, 21)
    p = sa.params_for(w)
    Kc = run_pool(w, inp, p)
    torch.cuda.synchronize()
    for (bi, h) in all_pairs(w):
        K = inp["K"][bi, h, :C].double().cpu().numpy()
        ref = orc.pool_lsa(K, b, 4) if pool == "lsa" else orc.pool_mean(K, b)
        np.testing.assert_allclose(Kc[bi, h].double().cpu().numpy(), ref, atol=2e-6, rtol=1e-5)


# ------------------------------------------------------------- score + top-k --

@pytest.mark.parametrize("name,over", [
    ("tiny_decode", {}),
    ("decode_32k", dict(batch=2)),
    ("draft_chunk_16k", dict(batch=2)),
    ("decode_1m", dict(batch=1, ctx_len=512 * 300 + 77, num_kv_heads=2, num_q_heads=8)),
])
def test_score_topk_parity(name, over):
    w = WORKLOADS[name].scaled(**over)
    inp = dev_inputs(w, 31)
    p = sa.params_for(w)
    Kc = run_pool(w, inp, p)
    nb = w.ctx_len // w.block_size
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device="cuda", dtype=torch.int32)
    scores = torch.empty((w.batch, w.num_kv_heads, nb), device="cuda", dtype=torch.float32)
    ws = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK)
    sa.score_topk(p, inp["Q"], Kc, idx, scores, ws)
    torch.cuda.synchronize()
    ref = oracle_decode(w, inp, all_pairs(w))
    ties = 0
    for (b, h), r in ref.items():
        np.testing.assert_allclose(scores[b, h].double().cpu().numpy(), r["scores"], atol=2e-5, rtol=2e-5)
        v = compare_sets(idx[b, h].cpu().numpy(), r["sel"])
        assert v != "mismatch", (b, h)
        ties += v == "near_tie"
        if w.n_needles <= w.top_k:
            assert set(inp["needles"][b, h].tolist()) <= set(idx[b, h].tolist())
    print(f"\n{name}: near-ties {ties}/{len(ref)}")


# ----------------------------------- scorer chunking and the two selectors --

@pytest.mark.parametrize("B,Hkv,nb,k,dup", [
    (1, 1, 2100, 32, False),      # one pair over many CTAs, CTA-wide selection
    (1, 1, 16384, 200, False),    # the largest table the selector takes
    (38, 8, 2100, 32, False),     # one CTA per pair, CTA-wide selection
    (38, 8, 600, 32, False),      # one CTA per pair, warp selection
    (1, 4, 600, 48, False),       # several CTAs per pair, warp selection
    (1, 2, 3000, 64, True),       # duplicated rows: exact ties go to the lower id
    (2, 2, 2500, 3000, False),    # k above the number of candidates
])
def test_score_topk_given_compressed_keys(B, Hkv, nb, k, dup):
    C = nb * 64 + 17
    w = WORKLOADS["decode_32k"].scaled(batch=B, num_kv_heads=Hkv, num_q_heads=4 * Hkv, ctx_len=C, top_k=k)
    p = sa.params_for(w)
    g = torch.Generator().manual_seed(1000 * nb + k)
    Kc = torch.randn((B, Hkv, nb, 128), generator=g) * 0.125     # the spread of 64-key means
    if dup:
        Kc[:, :, 1::2] = Kc[:, :, 0::2]
    Q = torch.randn((B, 1, 4 * Hkv, 128), generator=g).to(torch.bfloat16)
    idx = torch.empty((B, Hkv, k), device="cuda", dtype=torch.int32)
    scores = torch.empty((B, Hkv, nb), device="cuda")
    ws = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK)
    sa.score_topk(p, Q.cuda(), Kc.cuda(), idx, scores, ws)
    torch.cuda.synchronize()
    op = oracle_params(w)
    cand = orc.candidate_blocks(C, op)
    idx_h, sc_h = idx.cpu().numpy(), scores.cpu().double().numpy()
    ties = 0
    for b in range(B):
        for h in range(Hkv):
            qbar = orc.index_query(Q[b, 0, 4 * h:4 * h + 4].double().numpy())
            ref = orc.block_scores(qbar, Kc[b, h].double().numpy(), op)
            np.testing.assert_allclose(sc_h[b, h], ref, atol=2e-5, rtol=2e-5)
            sel = orc.select_topk(ref, cand, k)
            v = compare_sets(idx_h[b, h], sel)
            assert v != "mismatch", (b, h)
            ties += v == "near_tie"
            if dup:
                got = set(int(j) for j in idx_h[b, h] if j >= 0)
                for j in got:
                    if j % 2 == 1 and (j - 1) in cand:
                        assert j - 1 in got, (b, h, j)
    print(f"\nnb={nb} k={k} pairs={B * Hkv}: near-ties {ties}")


# -------------------------------------------------------- given index table --

@pytest.mark.parametrize("name,over", [
    ("tiny_decode", {}),
    ("decode_32k", dict(batch=2)),
    ("draft_chunk_16k", dict(batch=2, ctx_len=4096 + 5)),
    ("decode_1m", dict(batch=1, ctx_len=512 * 64 + 300, num_kv_heads=2, num_q_heads=8)),
])
def test_given_idx_with_oracle_indices(name, over):
    """The attention step alone, fed the oracle's own selection."""
    w = WORKLOADS[name].scaled(**over)
    inp = dev_inputs(w, 41)
    pairs = all_pairs(w)
    ref = oracle_decode(w, inp, pairs)
    idx = torch.full((w.batch, w.num_kv_heads, w.top_k), -1, dtype=torch.int32)
    for (b, h), r in ref.items():
        s = r["sel"].selected
        idx[b, h, :len(s)] = torch.tensor(s, dtype=torch.int32)
    idx = idx.cuda()
    p = sa.params_for(w, out_dtype="f32")
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device="cuda", dtype=torch.float32)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device="cuda", dtype=torch.float32)
    ws = sa.alloc_workspace(p, sa.SA_OP_GIVEN_IDX)
    sa.sparse_attn_given_idx(p, inp["Q"], inp["K"], inp["V"], idx, O, lse, ws)
    assert sa.read_status(ws) == sa.SA_OK
    G = w.group
    worst = (0.0, 0.0)
    for (b, h), r in ref.items():
        e = assert_close(O[b, :, h * G:(h + 1) * G], r["O"], w.dtype, f"pair {(b, h)}")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        assert np.abs(lse[b, :, h * G:(h + 1) * G].double().cpu().numpy() - r["lse"]).max() < 2e-4
    print(f"\n{name}: worst max-abs {worst[0]:.2e} rel-L2 {worst[1]:.2e}")


# ------------------------------------------------------------ end to end ----

@pytest.mark.parametrize("name,over", [
    ("tiny_decode", {}),
    ("decode_32k", dict(batch=2)),
    ("draft_chunk_16k", dict(batch=2)),
    ("decode_1m", dict(batch=1, ctx_len=512 * 200, num_kv_heads=2, num_q_heads=8)),
    # LSA centroids past 512 blocks: the fused step, each CTA publishing the
    # top k of its own score chunks and the last of a pair merging them
    ("decode_1m", dict(batch=2, ctx_len=512 * 1500 + 77, num_kv_heads=4, num_q_heads=16)),
    ("decode_1m", dict(batch=1, ctx_len=512 * 2000 + 300, num_kv_heads=1, num_q_heads=4, top_k=8)),
    # 8 and 16 query rows per KV head (n_q tokens x G heads): the tensor-core
    # kernel's other row-count instantiations
    ("draft_chunk_16k", dict(batch=3, n_q=2, num_q_heads=32, num_kv_heads=8, ctx_len=4096 + 77)),
    ("draft_chunk_16k", dict(batch=2, n_q=4, num_q_heads=32, num_kv_heads=8, ctx_len=8192 + 5)),
    ("draft_chunk_16k", dict(batch=2, n_q=3, num_q_heads=40, num_kv_heads=8, ctx_len=2048 + 64)),
])
def test_decode_end_to_end(name, over):
    check_decode(WORKLOADS[name].scaled(**over), seed=51)


def test_decode_bf16_output():
    check_decode(WORKLOADS["decode_32k"].scaled(batch=1), seed=52, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("over", [
    dict(top_k=0),                                      # sink + window + new token only
    dict(top_k=600),                                    # k above #candidates: dense equivalence
    dict(ctx_len=40),                                   # no complete block
    dict(ctx_len=0),                                    # the new token attends itself only
    dict(ctx_len=64 * 33 + 7, sink_keys=100, window_keys=70),   # ragged sink / window / context
    dict(num_q_heads=2, num_kv_heads=2),                # GQA 1
    dict(num_q_heads=16, num_kv_heads=2, n_q=2),        # GQA 8 x 2 tokens = 16 rows
    dict(num_q_heads=4, num_kv_heads=2, n_q=6, top_k=5),  # draft chunk, 12 rows
    dict(block_size=128, top_k=3),
])
def test_decode_edge_cases(over):
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, ctx_len=4096, n_needles=2)
    base.update(over)
    w = WORKLOADS["decode_32k"].scaled(**base)
    if w.top_k > 64 or w.ctx_len < 4096:
        w = w.scaled(n_needles=0)
    check_decode(w, seed=61)


@pytest.mark.parametrize("batch,n_q", [
    (74, 3),      # 148 pairs, 6 rows: one whole pair per CTA on a 148-SM B200, nothing split
    (74, 6),      # the same with 12 rows per KV head (draft chunk)
    (149, 1),     # 298 pairs, 2 rows: two whole pairs per CTA, two split over every CTA
    (150, 6),     # 300 pairs: two whole pairs per CTA, four split
])
def test_attention_whole_pairs_then_split(batch, n_q):
    """The attention kernel gives each CTA floor(pairs / SMs) whole pairs and
    splits the rest evenly; at these pair counts (all above what the fused
    launch takes, so scoring and attention run as two kernels) every output
    row is checked (2 KV heads, a 2085-key context)."""
    assert sa.decode_launches(sa.params_for(WORKLOADS["decode_32k"].scaled(batch=batch, num_q_heads=4,
                                                                           num_kv_heads=2, n_q=n_q))) == 2
    w = WORKLOADS["decode_32k"].scaled(batch=batch, num_q_heads=4, num_kv_heads=2, ctx_len=2048 + 37,
                                       n_q=n_q, top_k=5, n_needles=0)
    check_decode(w, seed=67, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dtype,n_q", [("bf16", 1), ("bf16", 6), ("f32", 3)])
def test_append_kv(dtype, n_q):
    """sa_append_kv puts the new tokens' rows at rows ctx_len.. of every
    pair, bit for bit, and leaves every other row of the cache as it was."""
    w = WORKLOADS["decode_32k"].scaled(batch=3, num_q_heads=8, num_kv_heads=2, ctx_len=1000, n_q=n_q,
                                       dtype=dtype, n_needles=0)
    cap = w.kv_len + 37
    inp = make_inputs(w, seed=69, device="cuda", kv_capacity=cap)
    K, V = inp["K"], inp["V"]
    K0, V0 = K.clone(), V.clone()
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    Kn = torch.randn((w.batch, w.num_kv_heads, n_q, 128), device="cuda", generator=g).to(K.dtype)
    Vn = torch.randn((w.batch, w.num_kv_heads, n_q, 128), device="cuda", generator=g).to(K.dtype)
    sa.append_kv(sa.params_for(w, kv_capacity=cap), Kn, Vn, K, V)
    torch.cuda.synchronize()
    C = w.ctx_len
    assert torch.equal(K[:, :, C:C + n_q], Kn) and torch.equal(V[:, :, C:C + n_q], Vn)
    keep = torch.ones(cap, dtype=torch.bool, device="cuda")
    keep[C:C + n_q] = False
    assert torch.equal(K[:, :, keep], K0[:, :, keep]) and torch.equal(V[:, :, keep], V0[:, :, keep])


def test_decode_fp32_dense_equivalence_torch():
    """k covering every candidate: the GPU result equals dense attention
    computed by torch in float64 (a library routine, independent of both)."""
    w = WORKLOADS["tiny_decode"].scaled(top_k=100, ctx_len=1500)
    inp = dev_inputs(w, 62)
    p = sa.params_for(w)
    Kc = run_pool(w, inp, p)
    O, lse, idx, _ = run_decode(w, inp, p, Kc)
    q = inp["Q"][0, 0].double()                    # [4, d]
    K = inp["K"][0, 0, :w.kv_len].double()
    V = inp["V"][0, 0, :w.kv_len].double()
    ref = torch.nn.functional.scaled_dot_product_attention(q[:, None], K[None].expand(4, -1, -1),
                                                           V[None].expand(4, -1, -1))[:, 0]
    assert (O[0, 0].double() - ref).abs().max().item() <= 1e-5


def test_workspace_reuse_is_deterministic():
    w = WORKLOADS["decode_32k"].scaled(batch=2)
    inp = dev_inputs(w, 71)
    p = sa.params_for(w, out_dtype="f32")
    Kc = run_pool(w, inp, p)
    O1, lse1, idx1, ws = run_decode(w, inp, p, Kc)
    O2 = torch.empty_like(O1)
    lse2 = torch.empty_like(lse1)
    idx2 = torch.empty_like(idx1)
    for _ in range(3):
        sa.sparse_attn_decode(p, inp["Q"], inp["K"], inp["V"], Kc, O2, lse2, idx2, ws)
    assert sa.read_status(ws) == sa.SA_OK
    assert torch.equal(idx1, idx2) and torch.equal(O1, O2) and torch.equal(lse1, lse2)


def test_trusted_table_flag_gives_the_checked_result():
    """SA_FLAG_TRUSTED_IDX only skips the checking pass: with a valid table
    (here the library's own selection) both paths agree bit for bit."""
    w = WORKLOADS["decode_32k"].scaled(batch=2)
    inp = dev_inputs(w, 73)
    p = sa.params_for(w, out_dtype="f32")
    Kc = run_pool(w, inp, p)
    _, _, idx, _ = run_decode(w, inp, p, Kc)
    outs = []
    for flags in (0, sa.SA_FLAG_TRUSTED_IDX):
        p.flags = flags
        O = torch.empty((w.batch, 1, w.num_q_heads, 128), device="cuda")
        ws = sa.alloc_workspace(p, sa.SA_OP_GIVEN_IDX)
        sa.sparse_attn_given_idx(p, inp["Q"], inp["K"], inp["V"], idx, O, None, ws)
        assert sa.read_status(ws) == sa.SA_OK
        outs.append(O)
    assert torch.equal(outs[0], outs[1])


def test_given_idx_bad_entries_are_reported_and_skipped():
    w = WORKLOADS["decode_32k"].scaled(batch=1, num_kv_heads=2, num_q_heads=8, ctx_len=4096, top_k=6,
                                       n_needles=0)
    inp = dev_inputs(w, 81)
    nb = w.ctx_len // 64
    rows = [[3, 9, 9, 20, -1, -1],            # repeated id
            [5, 2, 30, nb + 4, 40, -1]]       # descending pair and an out-of-range id
    keep = [[3, 9, 20], [5, 30, 40]]
    idx = torch.tensor(rows, dtype=torch.int32, device="cuda")[None]
    p = sa.params_for(w, out_dtype="f32")
    O = torch.empty((1, 1, 8, 128), device="cuda")
    ws = sa.alloc_workspace(p, sa.SA_OP_GIVEN_IDX)
    sa.sparse_attn_given_idx(p, inp["Q"], inp["K"], inp["V"], idx, O, None, ws)
    assert sa.read_status(ws) == sa.SA_ERR_INDEX
    assert sa.read_status(ws) == sa.SA_OK            # the status word was cleared
    op = oracle_params(w)
    for h in range(2):
        q, K, V = slab(inp, 0, h, 4, w.kv_len)
        pos = orc.attended_positions(w.ctx_len, op, keep[h], w.ctx_len)
        for g in range(4):
            ref, _, _ = orc.masked_softmax_attention(q[0, g], K, V, pos, 1 / np.sqrt(128))
            err = np.abs(O[0, 0, h * 4 + g].double().cpu().numpy() - ref).max()
            assert err < 5e-3


# ------------------------------------------------------- full-size samples --

def _sampled(w):
    return sorted({(0, 0), (w.batch - 1, w.num_kv_heads - 1), (w.batch // 2, w.num_kv_heads // 2),
                   (1 % w.batch, (3 % w.num_kv_heads)), (w.batch // 3, w.num_kv_heads - 1)})


@pytest.mark.parametrize("name", ["decode_32k", "draft_chunk_16k", "decode_1m"])
def test_full_size_sampled(name):
    """The benchmark's launch configuration at full size; the oracle checks a
    sample of (sequence, KV head) pairs one by one."""
    w = WORKLOADS[name]
    check_decode(w, seed=91, pairs=_sampled(w), out_dtype=torch.bfloat16)
    torch.cuda.empty_cache()


def test_full_size_sampled_fp32_output():
    """decode_32k at full size in the benchmark's launch configuration (the
    fused cooperative launch) with fp32 outputs: the sampled pairs meet max
    abs <= 5e-3 and relative L2 <= 1e-2 on the plain error, with nothing
    discounted for an output format."""
    w = WORKLOADS["decode_32k"]
    assert sa.decode_launches(sa.params_for(w, out_dtype="f32")) == 1
    check_decode(w, seed=92, pairs=_sampled(w), out_dtype=torch.float32)
    torch.cuda.empty_cache()


def test_fused_empty_tiles_after_score_chunks():
    """A 3-block window plus the new key gives an odd number of
    index-independent tiles, so the last unit of each pair's run has an
    empty second tile; at full batch every CTA first scores several chunks
    of compressed keys through the same ring stages.  The empty tile's V rows
    must read as zeros, not as whatever the stage last held: every output is
    finite and sampled pairs match the oracle."""
    w = WORKLOADS["decode_32k"].scaled(window_keys=192)
    assert sa.decode_launches(sa.params_for(w)) == 1
    _, _, _, O, lse, _ = check_decode(w, seed=93, pairs=_sampled(w), out_dtype=torch.bfloat16)
    assert torch.isfinite(O.float()).all() and torch.isfinite(lse).all()
    torch.cuda.empty_cache()


def test_decode_32k_runs_as_one_launch():
    """The batched-decode and 1M-token workloads take the fused path (scores,
    top-k and attention in one cooperative launch) on this device, LSA
    pooling too, past 512 blocks for k <= 8; draft chunks (12 query rows per
    KV head), more than two pairs per SM, fp32, overlapping windows and more
    than 512 blocks with k > 8 take the scoring kernel and then the
    attention kernel."""
    n = lambda w: sa.decode_launches(sa.params_for(w))
    assert n(WORKLOADS["decode_32k"]) == 1
    assert n(WORKLOADS["draft_chunk_16k"]) == 2
    assert n(WORKLOADS["draft_chunk_16k"].scaled(n_q=2)) == 2        # 512 pairs
    assert n(WORKLOADS["draft_chunk_16k"].scaled(n_q=2, batch=16)) == 1
    assert n(WORKLOADS["tiny_decode"]) == 2                            # fp32
    assert n(WORKLOADS["decode_32k_overlap"]) == 2                     # windows
    assert n(WORKLOADS["decode_1m"]) == 1                              # 2048 blocks, k = 4
    assert n(WORKLOADS["decode_1m"].scaled(top_k=9)) == 2              # 2048 blocks, k > 8
    assert n(WORKLOADS["decode_1m"].scaled(ctx_len=512 * 512, top_k=64)) == 1
    assert n(WORKLOADS["decode_1m"].scaled(ctx_len=512 * 513, top_k=64)) == 2


@pytest.mark.parametrize("nb,k,pool,launches", [(500, 8, "lsa", 1), (400, 32, "lsa", 1), (450, 6, "mean", 1),
                                                 (2048, 4, "lsa", 1), (1500, 6, "mean", 1), (1500, 12, "mean", 2)])
def test_decode_selection_with_exact_ties(nb, k, pool, launches):
    """The decode step's selection (the fused step's warp bit search up to
    512 blocks, its per-CTA candidates and merge past them for k <= 8, the
    scoring kernel's CTA radix select otherwise) on compressed keys whose
    odd rows repeat the even rows: exact ties go to the lower block id, so a
    selected odd block always comes with its even twin; the sets and outputs
    match the oracle's."""
    b = 512 if pool == "lsa" else 64
    C = nb * b + 33
    base = WORKLOADS["decode_1m"] if pool == "lsa" else WORKLOADS["decode_32k"]
    w = base.scaled(batch=2, num_kv_heads=2, num_q_heads=8, ctx_len=C, top_k=k, n_needles=0)
    p = sa.params_for(w, out_dtype="f32")
    assert sa.decode_launches(p) == launches
    inp = dev_inputs(w, seed=97)
    Kc = run_pool(w, inp, p)
    Kc[:, :, 1::2] = Kc[:, :, 0::2]
    O, lse, idx, _ = run_decode(w, inp, p, Kc, torch.float32)
    torch.cuda.synchronize()
    op = oracle_params(w)
    cand = orc.candidate_blocks(C, op)
    for bi in range(w.batch):
        for h in range(w.num_kv_heads):
            q, K, V = slab(inp, bi, h, w.group, w.kv_len)
            ref = orc.block_scores(orc.index_query(q[0]), Kc[bi, h].double().cpu().numpy(), op)
            sel = orc.select_topk(ref, cand, k)
            v = compare_sets(idx[bi, h].cpu().numpy(), sel)
            assert v != "mismatch", (bi, h, idx[bi, h].tolist(), sel.selected)
            got = set(int(j) for j in idx[bi, h] if j >= 0)
            for j in got:
                if j % 2 == 1 and (j - 1) in cand:
                    assert j - 1 in got, (bi, h, j, sorted(got))
            if v == "match":
                pos = orc.attended_positions(C, op, sel.selected, C)
                Oref, lref, _ = orc.masked_softmax_attention(q[0, 0], K, V, pos, orc.softmax_scale(128, op))
                assert_close(O[bi, 0, h * w.group], Oref[None], "bf16", f"pair {(bi, h)}")
