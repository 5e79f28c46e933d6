"""GPU parity of the dense verify (sa_verify_refresh) against the float64
oracle (oracle.sparse_attn_oracle.verify_pair): O and lse of the dense causal
attention, the per-block attention mass and the refreshed top-k table."""
import numpy as np
import pytest
import torch

from helpers import assert_close, compare_sets, oracle_params, slab
from oracle import sparse_attn_oracle as orc
from top_block_sparse_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("top_block_sparse_b200.sa")

# Each weight exp(z - lse) is off by the relative error of z - lse: the
# logit from bf16 inputs with fp32 accumulation (~1e-6 of |z|), the fp32 lse
# of the dense pass (~1e-6) and ex2.approx (2^-22); the mass sums at most
# 16 rows x b weights in fp32.  2e-5 leaves a margin of ten over that.
MASS_REL = 2e-5


def run_verify(w, inp, out_dtype=torch.float32):
    p = sa.params_for(w, out_dtype="bf16" if out_dtype == torch.bfloat16 else "f32")
    dev = torch.device("cuda")
    Q, K, V = (inp[k].to(dev) for k in ("Q", "K", "V"))
    nb = w.ctx_len // w.block_size
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev, dtype=out_dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev, dtype=torch.float32)
    mass = torch.full((w.batch, w.num_kv_heads, max(nb, 1)), float("nan"), device=dev, dtype=torch.float32)
    idx = torch.empty((w.batch, w.num_kv_heads, max(w.top_k, 1)), device=dev, dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_VERIFY, device=dev)
    sa.verify_refresh(p, Q, K, V, O, mass, lse=lse, idx_out=idx if w.top_k > 0 else None, ws=ws)
    assert sa.read_status(ws) == sa.SA_OK
    return O, lse, mass[..., :nb], idx[..., :w.top_k]


def check_verify(w, seed, pairs=None, out_dtype=torch.float32):
    inp = make_inputs(w, seed=seed, device="cpu")
    O, lse, mass, idx = run_verify(w, inp, out_dtype)
    torch.cuda.synchronize()
    p = oracle_params(w)
    pairs = pairs or [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    G = w.group
    worst_mass = 0.0
    n_tie = 0
    for (b, h) in pairs:
        q, K, V = slab(inp, b, h, G, w.kv_len)
        r = orc.verify_pair(q, K, V, w.ctx_len, p)
        dt = "f32" if (w.dtype == "f32" and out_dtype == torch.float32) else "bf16"
        assert_close(O[b, :, h * G:(h + 1) * G], r["O"], dt, f"O pair {(b, h)}")
        lse_err = np.abs(lse[b, :, h * G:(h + 1) * G].double().cpu().numpy() - r["lse"]).max()
        assert lse_err < 2e-4, lse_err
        m = mass[b, h].double().cpu().numpy()
        err = np.abs(m - r["mass"])
        assert np.all(err <= MASS_REL * r["mass"] + 1e-7), (b, h, float(err.max()))
        if len(m):
            worst_mass = max(worst_mass, float((err / np.maximum(r["mass"], 1e-30)).max()))
        if w.top_k > 0:
            verdict = compare_sets(idx[b, h].cpu().numpy(), r["sel"])
            assert verdict != "mismatch", (b, h, idx[b, h].tolist(), r["sel"].selected)
            n_tie += verdict == "near_tie"
    print(f"\n{w.name} verify: worst relative mass error {worst_mass:.2e}, {n_tie} near-ties")
    return inp, O, lse, mass, idx


def _chunk(**over):
    base = dict(batch=2, num_q_heads=4, num_kv_heads=2, n_q=7, ctx_len=2048 + 37, top_k=8)
    base.update(over)
    return WORKLOADS["draft_chunk_16k"].scaled(**base)


@pytest.mark.parametrize("over", [
    {},                                                  # 7 tokens x GQA 2 = 14 rows, ragged context
    dict(n_q=1, num_q_heads=16, num_kv_heads=2),         # 8 rows
    dict(ctx_len=64 * 40),                               # context a whole number of blocks
    dict(top_k=500),                                     # k above #candidates
    dict(block_size=128, top_k=3),                       # two 64-key tiles per block
    dict(ctx_len=40),                                    # no complete block: empty mass, -1 table
    dict(top_k=0),                                       # mass only
    dict(sink_keys=100, window_keys=70, ctx_len=64 * 33 + 7),
])
def test_verify_parity(over):
    check_verify(_chunk(**over), seed=71)


def test_verify_bf16_output_and_needles():
    """Planted needle blocks of the draft-chunk inputs take the most mass,
    so the refreshed table keeps them."""
    w = _chunk(ctx_len=4096, n_needles=3)
    inp, O, lse, mass, idx = check_verify(w, seed=72, out_dtype=torch.bfloat16)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            assert set(inp["needles"][b, h].tolist()) <= set(idx[b, h].tolist())


def test_verify_mass_totals():
    """Per pair, block masses plus the weight on the keys past the complete
    blocks total n_q * G (every row's weights sum to one)."""
    w = _chunk()
    inp = make_inputs(w, seed=73, device="cpu")
    O, lse, mass, idx = run_verify(w, inp)
    p = oracle_params(w)
    for (b, h) in [(0, 0), (1, 1)]:
        q, K, V = slab(inp, b, h, w.group, w.kv_len)
        r = orc.verify_pair(q, K, V, w.ctx_len, p)
        tot = float(mass[b, h].double().sum()) + float(r["wtail"].sum())
        assert abs(tot - w.n_q * w.group) < 1e-3 * w.n_q * w.group


def test_verify_full_size_sampled():
    """The draft-chunk workload at full size (64 sequences, 8 KV heads,
    16k context) with the chunk plus its bonus token, n_q = 7; the oracle
    checks a sample of pairs."""
    w = WORKLOADS["draft_chunk_16k"].scaled(n_q=7)
    pairs = sorted({(0, 0), (w.batch - 1, w.num_kv_heads - 1), (w.batch // 2, 3), (17, 5)})
    check_verify(w, seed=74, pairs=pairs, out_dtype=torch.bfloat16)
    torch.cuda.empty_cache()
