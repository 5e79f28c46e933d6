"""The bounded cross-CTA wait of the fused decode step runs out and is
reported, without a GPU fault.

The fused decode kernel (one cooperative launch) publishes each (sequence,
KV head) pair's index table with a ready flag that the CTAs attending the
pair's selected blocks wait for, with a limit of about 2 s.  A workspace
that breaks the zero-fill precondition in one pair's score counter makes
that pair's count never complete, so nothing ever sets its flag: the waits
must give up, the call must come back with the device status word reading
SA_ERR_TIMEOUT, and a later call on a properly zero-filled workspace must be
exact again.  The workspace layout used here: a 256-byte header holding the
status word, then one 32-bit score counter per pair.
"""
import time

import pytest
import torch

from helpers import assert_close, oracle_decode
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")


def _decode(p, w, inp, Kc, ws):
    O = torch.empty((w.batch, 1, w.num_q_heads, 128), device="cuda")
    lse = torch.empty((w.batch, 1, w.num_q_heads), device="cuda")
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device="cuda", dtype=torch.int32)
    sa.sparse_attn_decode(p, inp["Q"], inp["K"], inp["V"], Kc, O, lse, idx, ws)
    return O, lse, idx


def test_fused_decode_wait_gives_up_and_reports_timeout():
    w = WORKLOADS["decode_32k"].scaled(batch=2, ctx_len=8192, n_needles=4)
    inp = make_inputs(w, seed=71, device="cuda")
    p = sa.params_for(w, out_dtype="f32")
    assert sa.decode_launches(p) == 1                     # the fused cooperative launch
    nb = w.ctx_len // w.block_size
    Kc = torch.empty((w.batch, w.num_kv_heads, nb, 128), device="cuda")
    sa.pool_keys(p, inp["K"], Kc)
    ref_ws = sa.alloc_workspace(p, sa.SA_OP_DECODE)
    O_ref, _, idx_ref = _decode(p, w, inp, Kc, ref_ws)
    assert sa.read_status(ref_ws) == sa.SA_OK

    bad = sa.alloc_workspace(p, sa.SA_OP_DECODE)
    bad.view(torch.int32)[256 // 4 + 3] = 1               # pair 3's score counter starts at 1
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    _decode(p, w, inp, Kc, bad)
    st = sa.read_status(bad)
    dt = time.perf_counter() - t0
    assert st == sa.SA_ERR_TIMEOUT, sa.raw_call("sa_status_string", st)
    assert 1.0 < dt < 60.0, dt                            # the ~2 s limit ran out, nothing hung

    # the context is still usable: a zero-filled workspace gives the exact result again
    good = sa.alloc_workspace(p, sa.SA_OP_DECODE)
    O, _, idx = _decode(p, w, inp, Kc, good)
    assert sa.read_status(good) == sa.SA_OK
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref)
    assert torch.equal(O, O_ref)
    ref = oracle_decode(w, inp, [(0, 3)])[(0, 3)]
    G = w.group
    if [int(x) for x in idx[0, 3].tolist() if x >= 0] == ref["sel"].selected:
        assert_close(O[0, :, 3 * G:4 * G], ref["O"], "bf16", "pair 3 after the timeout")
