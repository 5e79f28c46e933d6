"""The algorithmic byte and FLOP counts behind the benchmark's roofline
figures, derived here independently from the workload shapes: keys
attended per query (sink + k blocks + window + the new keys), the bytes of
one decode step (retained K and V rows, compressed keys, Q and O) and the
algorithmic FLOPs of the causal prefill."""
import bench
from top_block_sparse_b200.inputs import WORKLOADS


def _keys(S, k, b, W, n_new):
    return S + k * b + W + n_new


def test_decode_step_bytes():
    # 32k decode: 64 sink + 32 blocks of 64 + 256 window + the new key
    w = WORKLOADS["decode_32k"]
    by = bench.decode_bytes(w)
    pairs = 32 * 8
    assert by["keys_per_query"] == _keys(64, 32, 64, 256, 1) == 2369
    assert by["kv"] == pairs * 2369 * 128 * 2 * 2                # 310.5 MB
    assert by["kc"] == pairs * (32768 // 64) * 128 * 4           # 67.1 MB
    qo = 32 * 1 * 32 * 128 * 2
    assert by["step"] == by["kv"] + by["kc"] + 2 * qo + qo
    assert abs(by["step"] / 1e6 - 378.4) < 0.1
    # draft chunk: 16 blocks, 6 new keys; 1M-token LSA: 4 sink keys, 4 blocks of 512, 512 window
    assert bench.decode_bytes(WORKLOADS["draft_chunk_16k"])["keys_per_query"] == _keys(64, 16, 64, 256, 6) == 1350
    d1m = bench.decode_bytes(WORKLOADS["decode_1m"])
    assert d1m["keys_per_query"] == _keys(4, 4, 512, 512, 1) == 2565
    assert d1m["kc"] == 4 * 8 * 2048 * 128 * 4
    assert bench.decode_bytes(WORKLOADS["tiny_decode"])["keys_per_query"] == _keys(64, 8, 64, 128, 1) == 705


def test_prefill_flops():
    """Tile i of 64 queries (context C = 64 i) attends the sink block, the
    top-64 of its max(0, i - 5) candidate blocks, the 4 window blocks before
    it and its own keys causally; QK^T and PV are 4 d FLOP per (query, key,
    head).  Scoring: each (tile, candidate block) pair costs 64 rows x 2 d
    per KV head."""
    w = WORKLOADS["prefill_64k"]
    d, Hq, Hkv = 128, 32, 8
    attn = score = 0
    for i in range(65536 // 64):
        C = 64 * i
        sink = min(64, C)
        window = C - max(C - 256, sink)
        cand = max(0, i - 5)
        ctx_keys = sink + 64 * min(64, cand) + window
        attn += Hq * 4 * d * (64 * ctx_keys + 64 * 65 // 2)
        score += Hkv * cand * 64 * 2 * d
    c = bench.prefill_counts(w)
    assert c["attn_alg"] == attn and abs(attn / 1e12 - 4.61) < 0.01
    assert c["score_alg"] == score and abs(score / 1e9 - 68.0) < 0.1
    assert c["attn_exec"] >= c["attn_alg"] and c["score_exec"] >= c["score_alg"]


def test_prefill_report_fractions():
    """The prefill line's headline fractions count algorithmic FLOPs; the
    executed-FLOP fractions are separate fields, and the scoring call also
    reports Q and Kc read once against the HBM peak."""
    w = WORKLOADS["prefill_64k"]
    c = bench.prefill_counts(w)
    pk = (6000.0, 1500.0, 1400.0, "test")
    rep = bench.prefill_report(w, [5.0, 5.2], [0.25, 0.27], [4.9, 4.7], pk)
    a, s = rep["attention"], rep["scoring"]
    assert abs(a["ms"] - 4.8) < 1e-12 and abs(s["ms"] - 0.26) < 1e-12
    assert abs(a["frac_of_bf16_peak"] - c["attn_alg"] / 4.8e-3 / 1e12 / 1500.0) < 1e-12
    assert abs(a["exec_frac_of_bf16_peak"] - c["attn_exec"] / 4.8e-3 / 1e12 / 1500.0) < 1e-12
    assert abs(s["frac_of_bf16_peak"] - c["score_alg"] / 0.26e-3 / 1e12 / 1500.0) < 1e-12
    assert abs(s["exec_frac_of_bf16_peak"] - c["score_exec"] / 0.26e-3 / 1e12 / 1500.0) < 1e-12
    # split precision: three bf16 products per fp32 product, so executed > 3x algorithmic
    assert s["exec_frac_of_bf16_peak"] > 3 * s["frac_of_bf16_peak"]
    q_bytes = 65536 * 32 * 128 * 2
    kc_bytes = 8 * 1024 * 128 * 4
    assert s["hbm_bytes"] == q_bytes + kc_bytes
    assert abs(s["hbm_frac"] - (q_bytes + kc_bytes) / 0.26e-3 / 1e9 / 6000.0) < 1e-12
    assert rep["ms_spread"]["min"] == 5.0 and rep["ms_spread"]["max"] == 5.2


def test_step_spread():
    sp = bench.spread([3.0, 1.0, 2.0, 10.0, 4.0, 5.0, 6.0, 7.0, 8.0, 9.0])
    assert sp["min"] == 1.0 and sp["max"] == 10.0 and sp["median"] == 5.5
    assert sp["p90"] == 9.0 and sp["n"] == 10 and abs(sp["mean"] - 5.5) < 1e-12


def test_parity_tally_counts_and_errors():
    """The benchmark's per-config parity record: sets counted as matching,
    near-tie or mismatching; errors only over matching pairs; a bf16 output's
    format rounding reported apart from the plain max abs."""
    import numpy as np
    import torch
    from oracle.sparse_attn_oracle import Selection

    t = bench.ParityTally()
    sel = Selection([1, 4], 10, 0.5, 0.2, False)
    tie = Selection([1, 5], 10, 0.5, 1e-9, True)
    assert t.sets([1, 4], sel) and not t.sets([1, 6], tie) and not t.sets([2, 4], sel)
    ref = np.array([[1.0, -2.0], [0.5, 0.25]])
    t.out(torch.tensor(ref + 1e-3, dtype=torch.float32), ref)
    r = t.report("test", 4.0)
    assert (r["checked"], r["sets_match"], r["near_ties"], r["mismatches"]) == (3, 1, 1, 1)
    assert abs(r["max_abs"] - 1e-3) < 1e-7 and abs(r["max_abs_beyond_bf16_rounding"] - 1e-3) < 1e-7
    assert abs(r["rel_l2"] - 2e-3 / np.sqrt((ref ** 2).sum())) < 1e-7
    t2 = bench.ParityTally()
    t2.out(torch.tensor(ref, dtype=torch.bfloat16), ref + 4e-4)    # within half a bf16 step (>= 2^-10 here)
    assert t2.max_abs > 0 and t2.max_abs_fmt == 0.0


def test_even_pairs_sampling():
    w = WORKLOADS["decode_1m"]
    ps = bench.even_pairs(w, 4)
    assert len(ps) == 4 and ps[0] == (0, 0) and len(set(ps)) == 4
    assert bench.even_pairs(w, 100) == [(b, h) for b in range(4) for h in range(8)]
