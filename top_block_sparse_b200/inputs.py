"""Seeded synthetic inputs and the workload shapes they are drawn at.

This module builds inputs only: it holds none of the sparse-attention
arithmetic (no pooling, scoring, selection or softmax), so both the CUDA
library's tests/benchmark and the float64 oracle may draw from it.

Recipe (every workload):
  * Q [B, n_q, Hq, d], K and V [B, Hkv, C + n_q, d] are i.i.d. N(0, 1) in fp32
    from torch generators with fixed seeds (one generator per tensor slab, so
    the result does not depend on the batch being generated in pieces).
  * Needle blocks imitate long-context retrieval (needle-in-a-haystack style
    tasks): u = mean of the defining query over the GQA group (the new token,
    the chunk's first token, or for prefill the last token); for
    ``n_needles`` distinct blocks drawn uniformly from the blocks that lie
    after the sink and wholly before the window, every key of the block
    becomes 0.5*u + (its own N(0,1) noise).
  * bf16 workloads then round Q, K, V to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int              # new query tokens per sequence (prefill: T)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    ctx_len: int          # C: keys cached before the new tokens (prefill: 0)
    dtype: str            # "f32" | "bf16"
    block_size: int       # b
    pool: str             # "mean" | "lsa"
    top_k: int
    sink_keys: int
    window_keys: int
    n_needles: int
    prefill: bool = False
    pool_stride: int = 4  # LSA: raw keys per pool key; overlap: keys between window starts
    pool_kernel: int = 0  # overlap: keys per compressed key

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def kv_len(self) -> int:
        return self.ctx_len + self.n_q

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # batch 1, GQA 4 (4 query heads / 1 KV head), fp32, C = 4096
    "tiny_decode": Workload("tiny_decode", 1, 1, 4, 1, 128, 4096, "f32",
                            64, "mean", 8, 64, 128, 4),
    # batch 32, 32 query heads / 8 KV heads, C = 32768, bf16
    "decode_32k": Workload("decode_32k", 32, 1, 32, 8, 128, 32768, "bf16",
                           64, "mean", 32, 64, 256, 16),
    # causal prefill of T = 65536 tokens, 32 / 8 heads, bf16
    "prefill_64k": Workload("prefill_64k", 1, 65536, 32, 8, 128, 0, "bf16",
                            64, "mean", 64, 64, 256, 16, prefill=True),
    # batch 4, C = 1,048,576, LSA pooling (4 -> 1, 128 pool keys per block)
    "decode_1m": Workload("decode_1m", 4, 1, 32, 8, 128, 1048576, "bf16",
                          512, "lsa", 4, 4, 512, 32),
    # decode_32k with overlapping compressed keys: windows of 32 keys every
    # 16 keys (two windows per half block, neighbours sharing half their keys)
    "decode_32k_overlap": Workload("decode_32k_overlap", 32, 1, 32, 8, 128, 32768, "bf16",
                                   64, "overlap", 32, 64, 256, 16, pool_stride=16, pool_kernel=32),
    # decode_1m with LSA flat bucket retrieval: 64 Ward buckets per 512-key
    # cluster block, top-256 buckets by centroid cosine, expanded to the 2048
    # long-range keys of best own cosine (sa_bucket_decode, bucket_keys 2048)
    "decode_1m_buckets": Workload("decode_1m_buckets", 4, 1, 32, 8, 128, 1048576, "bf16",
                                  512, "lsa", 256, 4, 512, 32),
    # batch 64, 6-token draft chunk, 16 / 8 heads, C = 16384
    "draft_chunk_16k": Workload("draft_chunk_16k", 64, 6, 16, 8, 128, 16384,
                                "bf16", 64, "mean", 16, 64, 256, 8),
    # column-sparse (bidirectional) attention over T = 65536 tokens, 32 / 8
    # heads, bf16: top_k = the columns listed per 64-token group (20% of T)
    "column_64k": Workload("column_64k", 1, 65536, 32, 8, 128, 0, "bf16",
                           64, "mean", 13120, 0, 0, 0, prefill=True),
}


def make_columns(w: Workload, seed: int, n_cols: Optional[int] = None, device="cpu") -> torch.Tensor:
    """Column lists [B, Hkv, ceil(T/64), n_cols] int32 for column-sparse
    attention over T = w.n_q tokens: per (sequence, KV head) one random set
    of n_cols - 64 key positions shared by all its 64-token groups (the
    important columns recur across rows), joined for each group with the
    group's own tokens; ascending, -1 padded.  n_cols defaults to w.top_k."""
    n_cols = w.top_k if n_cols is None else int(n_cols)
    T, B, Hkv = w.n_q, w.batch, w.num_kv_heads
    groups = (T + 63) // 64
    out = torch.full((B, Hkv, groups, n_cols), -1, dtype=torch.int32)
    n_shared = max(min(n_cols - 64, T), 0)
    for bi in range(B):
        for h in range(Hkv):
            g = _gen("cpu", seed * 1000003 + (bi * Hkv + h) * 4 + 5)
            shared = torch.randperm(T, generator=g)[:n_shared]
            mark = torch.zeros(T, dtype=torch.bool)
            mark[shared] = True
            for t in range(groups):
                m = mark.clone()
                lo, hi = t * 64, min(t * 64 + 64, T)
                if n_cols >= 64:
                    m[lo:hi] = True
                cols = torch.nonzero(m).flatten()[:n_cols].to(torch.int32)
                out[bi, h, t, :len(cols)] = cols
    return out.to(device)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def needle_block_range(w: Workload):
    """Block ids [lo, hi) a needle may occupy: after the sink, wholly before
    the window of the defining query's context."""
    b = w.block_size
    c_def = w.ctx_len
    if w.prefill:
        c_def = ((w.n_q - 1) // b) * b
    lo = -(-w.sink_keys // b)
    hi = max((c_def - w.window_keys) // b, lo)
    return lo, hi


def make_inputs(w: Workload, seed: int, device="cpu",
                kv_capacity: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw Q, K, V (and the needle block ids) for workload ``w``.

    Returns dict(Q [B,n_q,Hq,d], K/V [B,Hkv,cap,d] in the workload dtype,
    needles int64 [B,Hkv,n]).  ``kv_capacity`` >= C + n_q pads the token axis
    (the padding rows are zero).
    """
    B, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    T = w.kv_len
    cap = T if kv_capacity is None else int(kv_capacity)
    assert cap >= T
    out_dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    Q32 = torch.randn((B, w.n_q, Hq, d), generator=_gen(device, seed * 7919 + 1),
                      device=device, dtype=torch.float32)
    K = torch.zeros((B, Hkv, cap, d), device=device, dtype=out_dt)
    V = torch.zeros((B, Hkv, cap, d), device=device, dtype=out_dt)
    lo, hi = needle_block_range(w)
    n_nd = min(w.n_needles, max(hi - lo, 0))
    needles = torch.zeros((B, Hkv, n_nd), dtype=torch.int64)
    def_tok = (w.n_q - 1) if w.prefill else 0
    G = w.group
    b = w.block_size
    for bi in range(B):
        for h in range(Hkv):
            slab = (bi * Hkv + h) * 4
            k = torch.randn((T, d), generator=_gen(device, seed * 1000003 + slab + 2),
                            device=device, dtype=torch.float32)
            v = torch.randn((T, d), generator=_gen(device, seed * 1000003 + slab + 3),
                            device=device, dtype=torch.float32)
            if n_nd > 0:
                pick = torch.randperm(hi - lo, generator=_gen("cpu", seed * 1000003 + slab + 4))
                blocks = (pick[:n_nd] + lo).sort().values
                needles[bi, h] = blocks
                u = Q32[bi, def_tok, h * G:(h + 1) * G, :].mean(dim=0)
                for j in blocks.tolist():
                    k[j * b:(j + 1) * b] += 0.5 * u
            K[bi, h, :T] = k.to(out_dt)
            V[bi, h, :T] = v.to(out_dt)
    Q = Q32.to(out_dt)
    return dict(Q=Q, K=K, V=V, needles=needles)
