"""GPU parity of column-sparse attention (sa_column_attn) against the float64
oracle (oracle.sparse_attn_oracle.column_attention_group): every 64-token
group of a (sequence, KV head) attends to its listed key columns, both
before and after it."""
import numpy as np
import pytest
import torch

from helpers import assert_close, oracle_params
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_columns, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")


def _w(**over):
    base = dict(n_q=64 * 5 + 17, num_q_heads=8, num_kv_heads=2, top_k=70)
    base.update(over)
    return WORKLOADS["column_64k"].scaled(**base)


def run_column(w, inp, cols, out_dtype=torch.float32, trusted=True):
    p = sa.params_for(w, out_dtype="bf16" if out_dtype == torch.bfloat16 else "f32")
    if trusted:
        p.flags = sa.SA_FLAG_TRUSTED_IDX
    dev = torch.device("cuda")
    Q, K, V = (inp[k].to(dev) for k in ("Q", "K", "V"))
    O = torch.full((w.batch, w.n_q, w.num_q_heads, 128), float("nan"), device=dev, dtype=out_dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev)
    n_cols = 0 if cols is None else cols.shape[-1]
    p.top_k = n_cols
    ws = sa.alloc_workspace(p, sa.SA_OP_COLUMN, device=dev)
    sa.column_attn(p, Q, K, V, None if cols is None else cols.to(dev).contiguous(), O, lse, ws)
    status = sa.read_status(ws)
    return O, lse, status


def check_groups(w, inp, cols, O, lse, groups, kept=None, out_dtype=torch.float32):
    """Compare the listed (sequence, KV head, group) items with the oracle."""
    p = oracle_params(w)
    G = w.group
    T = w.n_q
    dt = "bf16"
    for (b, h, t) in groups:
        lo, hi = t * 64, min(t * 64 + 64, T)
        q = inp["Q"][b, lo:hi, h * G:(h + 1) * G].double().numpy()
        K = inp["K"][b, h, :T].double().numpy()
        V = inp["V"][b, h, :T].double().numpy()
        lst = kept(b, h, t) if kept else cols[b, h, t].tolist()
        r = orc.column_attention_group(q, K, V, lst, p)
        got = O[b, lo:hi, h * G:(h + 1) * G]
        if len(r["positions"]) == 0:
            assert torch.all(got == 0) and torch.all(torch.isneginf(lse[b, lo:hi, h * G:(h + 1) * G]))
            continue
        assert_close(got, r["O"], dt, f"O {(b, h, t)}")
        err = np.abs(lse[b, lo:hi, h * G:(h + 1) * G].double().cpu().numpy() - r["lse"]).max()
        assert err < 2e-4, ((b, h, t), err)


def _all_groups(w):
    return [(b, h, t) for b in range(w.batch) for h in range(w.num_kv_heads) for t in range((w.n_q + 63) // 64)]


@pytest.mark.parametrize("over,n_cols", [
    ({}, 70),                                           # two chunks, the second partial; ragged last group
    (dict(n_q=256), 64),                                # one full chunk per group
    (dict(n_q=64 * 3, batch=2), 200),                   # lists longer than the sequence: -1 padding
    (dict(n_q=128), 1),                                 # one column
    (dict(num_q_heads=16), 70),                         # 8 query heads per KV head: two head groups per item
])
def test_column_parity(over, n_cols):
    w = _w(**over)
    inp = make_inputs(w, seed=81, device="cpu")
    cols = make_columns(w, seed=82, n_cols=n_cols)
    O, lse, st = run_column(w, inp, cols)
    assert st == sa.SA_OK
    check_groups(w, inp, cols, O, lse, _all_groups(w))


def test_column_all_keys_is_dense_bidirectional_attention():
    """Every position listed: plain attention without a mask (torch SDPA,
    a library routine independent of both sides)."""
    w = _w(n_q=200)
    inp = make_inputs(w, seed=83, device="cpu")
    groups = (w.n_q + 63) // 64
    cols = torch.arange(w.n_q, dtype=torch.int32).expand(w.batch, w.num_kv_heads, groups, w.n_q).contiguous()
    O, lse, st = run_column(w, inp, cols)
    assert st == sa.SA_OK
    G = w.group
    for h in range(w.num_kv_heads):
        q = inp["Q"][0, :, h * G:(h + 1) * G].double().permute(1, 0, 2)      # [G, T, d]
        K = inp["K"][0, h, :w.n_q].double()[None].expand(G, -1, -1)
        V = inp["V"][0, h, :w.n_q].double()[None].expand(G, -1, -1)
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V).permute(1, 0, 2)
        assert_close(O[0, :, h * G:(h + 1) * G], ref.numpy(), "bf16", f"head {h}")


def test_column_empty_lists_and_bf16_output():
    """No column: O = 0 and lse = -inf; a bf16 output on a normal table."""
    w = _w(n_q=128)
    inp = make_inputs(w, seed=84, device="cpu")
    O, lse, st = run_column(w, inp, None)
    assert st == sa.SA_OK
    assert torch.all(O == 0) and torch.all(torch.isneginf(lse))
    cols = make_columns(w, seed=85, n_cols=96)
    O, lse, st = run_column(w, inp, cols, out_dtype=torch.bfloat16)
    assert st == sa.SA_OK
    check_groups(w, inp, cols, O, lse, _all_groups(w), out_dtype=torch.bfloat16)


def test_column_untrusted_table_is_checked():
    """Out-of-range, repeated and descending entries are dropped (status
    SA_ERR_INDEX); the kept entries - each above every earlier kept one -
    give the oracle's result."""
    w = _w(n_q=192)
    inp = make_inputs(w, seed=86, device="cpu")
    cols = make_columns(w, seed=87, n_cols=80)
    cols[0, 0, 0, :6] = torch.tensor([10, 5, 10, 900, -7, 40], dtype=torch.int32)
    cols[0, 1, 2, 3] = 100000
    O, lse, st = run_column(w, inp, cols, trusted=False)
    assert st == sa.SA_ERR_INDEX

    def kept(b, h, t):
        out, last = [], -1
        for c in cols[b, h, t].tolist():
            if 0 <= c < w.n_q and c > last:
                out.append(c)
                last = c
        return out
    check_groups(w, inp, cols, O, lse, _all_groups(w), kept=kept)


def test_column_full_size_sampled():
    """The 64k-token workload at full size (20% of the columns per group);
    the oracle checks a sample of groups."""
    w = WORKLOADS["column_64k"]
    inp = make_inputs(w, seed=88, device="cpu")
    cols = make_columns(w, seed=89)
    O, lse, st = run_column(w, inp, cols, out_dtype=torch.bfloat16)
    assert st == sa.SA_OK
    check_groups(w, inp, cols, O, lse, [(0, 0, 0), (0, 7, 1023), (0, 3, 511), (0, 5, 77)],
                 out_dtype=torch.bfloat16)
    torch.cuda.empty_cache()
