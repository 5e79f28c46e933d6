"""Helpers shared by the GPU parity tests: run the float64 oracle on the same
seeded inputs, compare index sets with the near-tie allowance, and measure
output errors."""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

from oracle import sparse_attn_oracle as orc

# Tolerances (bf16 inputs with fp32 accumulation / fp32 inputs).
BF16_MAX_ABS = 5e-3
BF16_REL_L2 = 1e-2
F32_MAX_ABS = 1e-5


def oracle_params(w, **kw) -> orc.OracleParams:
    p = orc.OracleParams(block_size=w.block_size, top_k=w.top_k, sink_keys=w.sink_keys,
                         window_keys=w.window_keys, pool=w.pool, pool_stride=w.pool_stride,
                         pool_kernel=w.pool_kernel)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def slab(inp, b: int, h: int, G: int, T: Optional[int] = None):
    """float64 numpy copies of one (sequence, KV head) slab."""
    q = inp["Q"][b, :, h * G:(h + 1) * G].double().cpu().numpy()
    K = inp["K"][b, h, :T].double().cpu().numpy()
    V = inp["V"][b, h, :T].double().cpu().numpy()
    return q, K, V


def oracle_decode(w, inp, pairs: List[tuple], p: Optional[orc.OracleParams] = None) -> Dict:
    p = p or oracle_params(w)
    out = {}
    for (b, h) in pairs:
        q, K, V = slab(inp, b, h, w.group, w.kv_len)
        out[(b, h)] = orc.decode_pair(q, K, V, w.ctx_len, p)
    return out


@dataclass
class SetReport:
    pairs: int = 0
    matched: int = 0
    near_ties: int = 0
    mismatched: List[tuple] = field(default_factory=list)


def compare_sets(gpu_idx_row: np.ndarray, sel: orc.Selection) -> str:
    """'match', 'near_tie' (differs but the oracle's k-th gap is a near-tie)
    or 'mismatch'.  Also checks the GPU row is well formed."""
    row = [int(x) for x in gpu_idx_row]
    k = len(row)
    valid = [x for x in row if x >= 0]
    assert valid == sorted(set(valid)), f"GPU ids not strictly ascending: {row}"
    assert all(x == -1 for x in row[len(valid):]), f"GPU -1 padding not at the end: {row}"
    assert len(valid) == min(k, sel.n_candidates), (len(valid), k, sel.n_candidates)
    if valid == sel.selected:
        return "match"
    return "near_tie" if sel.near_tie else "mismatch"


def bf16_half_step(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers around |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def errors(got: torch.Tensor, ref: np.ndarray):
    """Max abs and relative L2 error against the float64 reference.  For a
    bf16 output the max abs error is counted beyond half a bf16 step of the
    exact value (the output format cannot come closer), so the bar measures
    the kernel's arithmetic, not the format."""
    g = got.double().cpu().numpy().reshape(ref.shape)
    d = g - ref
    if got.dtype == torch.bfloat16:
        excess = np.maximum(np.abs(d) - bf16_half_step(ref), 0.0)
        max_abs = float(excess.max()) if d.size else 0.0
    else:
        max_abs = float(np.abs(d).max()) if d.size else 0.0
    den = float(np.sqrt((ref * ref).sum()))
    rel = float(np.sqrt((d * d).sum()) / den) if den > 0 else float(np.sqrt((d * d).sum()))
    return max_abs, rel


def assert_close(got, ref, dtype: str, what: str = ""):
    max_abs, rel = errors(got, ref)
    if dtype == "f32":
        assert max_abs <= F32_MAX_ABS, f"{what}: max abs {max_abs:.3e} > {F32_MAX_ABS}"
    else:
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, \
            f"{what}: max abs {max_abs:.3e} (<= {BF16_MAX_ABS}), rel L2 {rel:.3e} (<= {BF16_REL_L2})"
    return max_abs, rel
