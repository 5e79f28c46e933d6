"""Float64 CPU oracle for indexer-driven top-k block-sparse attention.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously-correct
definition that the CUDA library is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  It shares no code with the CUDA path and
imports nothing from ``top_block_sparse_b200``.

Every step works on ONE (sequence, KV head) slab at a time, in float64
(bf16 and fp32 inputs convert exactly), with no tiling, no online softmax and
no fusion.  Library primitives used as steps: numpy matmul / dot, sort, exp,
log.

Sources (web pages on the method; each function cites the passage it restates):

* [S3R review]   "港科大(广州)S3R:稀疏起草+稠密验证,RL训练吞吐1.39倍"
                 (longzhangge.com PaperDaily), section "稀疏起草": the
                 sparse-attention formula over a retained index set T and the
                 KV-selection formula (recent window + top-K); the k=6 draft
                 chunk with the selection held fixed.
* [LSA review]   "精读:LSA——当稀疏注意力的账单从「算」搬到「找」"
                 (tuntang.top), §2.2 (L2-normalise, sum 4 keys into a pool key,
                 centroid = normalised sum), §2.3 (normalised query scores
                 centroids, top buckets + 4 sink keys + 512 window keys, one
                 index table shared by the heads), §2.4 (query heads summed
                 into one index query).
* [SparDA]       hyper.ai paper summary 2606.04511 (SparDA on InfLLM-V2),
                 section "方法": attention = initial tokens + local sliding
                 window + top-k selected blocks; keys mean-pooled into
                 compressed keys; one forecast (index) head per GQA group.
* [PulseCol]     "PulseCol:周期性刷新的列稀疏注意力机制..." (bittide), §3.1
                 eq. (1) Z = QK^T/sqrt(d_h) and eq. (2) masked softmax
                 softmax(Z + M(S)) V.

Readings taken where the pages leave a step open (each is also listed in the
design notes of the repository):

* R1  GQA aggregation: the index query is the plain SUM of the group's query
      vectors; block score s_j = qbar . Kc_j * scale  (LSA §2.4 sums heads).
* R2  Prefill tile aggregation: a 64-query tile scores block j with the MAX
      over its rows of the GQA-summed logit (the pages do not say; max keeps
      any block some row needs, cf. N-LSA's max aggregation in LSA §2.5).
* R3  Window = the last W keys of the context [C-W, C); the new tokens
      (decode token, draft chunk, prefill diagonal tile) are attended causally
      in addition.
* R4  Blocks lying wholly inside sink or window are not candidates; a block
      partly covered stays a candidate and its covered keys count once.
* R5  Only complete blocks (b keys inside the context) are candidates.
* R6  Ties: score descending, then lower block index first.  A pair whose
      k-th and (k+1)-th candidate scores differ by less than 1e-4*|s_k| is a
      near-tie; more than one selected set is then correct.
* R7  LSA pooling order: normalise each raw key, sum 4 consecutive unit keys
      into a pool key, centroid = normalise(sum of the block's pool keys);
      score = (qbar/|qbar|) . c_j (cosine).  normalise(0) = 0.  In a causal
      prefill each row's index query is normalised before the tile max (R2).
* R8  Softmax scale 1/sqrt(d) unless given (PulseCol eq. (1)).
* R9  Multi-token chunk: the selection is made once from the chunk's FIRST
      query and reused by every token of the chunk (S3R draft chunk); token j
      of the chunk also sees chunk keys C..C+j.
* R17 Column-sparse attention (PulseCol §3.1 eq. (2) with a column mask): the
      mask is token-granular and shared by a group of 64 consecutive query
      tokens and the KV head's query heads; each listed key is attended once
      (duplicates and -1 entries are ignored); no causal mask, no sink or
      window.  An empty list gives O = 0, lse = -inf.
* R15 Dense verify (S3R review, "稠密验证"): every token of the chunk attends
      causally to ALL keys 0..C+j.  The verifier's attention "mass" of a
      complete context block is the SUM over the chunk's tokens and the KV
      head's G query heads of the attention weights its keys receive (the
      pages do not say how tokens and heads combine; a sum matches the
      GQA-summed scoring of R1).  The refreshed selection is the top-k of the
      candidate blocks by mass, with the candidates and ties of R4-R6 (the
      KV-selection formula: recent window plus top-K by the previous verify's
      attention scores).
* R18 Overlapping compressed keys (SparDA, "方法": InfLLM-V2 mean-pools the
      keys into OVERLAPPING compressed representations, coarse to fine; the
      window length and stride are not given, so they are parameters):
      compressed key c is the mean of the l keys starting at c*s (complete
      windows only), and the score of selectable block j is the MAX of the
      scores of the compressed keys whose windows share a key with block j.
      In a causal prefill, query tile i (context C = i*b) sees the windows
      complete inside its context, and block j's tile score is the max over
      those windows of the max over the tile's rows (R2).
* R19 LSA flat bucket retrieval (LSA review §2.2-2.3).  Pool keys as in R7
      (each raw key L2-normalised, ``pool_stride`` = 4 consecutive unit keys
      summed).  A cluster block is ``block_size`` = 512 RAW keys (128 pool
      keys): the page's 512-key window is "exactly one cluster block", and 64
      buckets of 8 keys on average fill 512 raw keys.  Inside a complete
      cluster block every pool key starts as its own bucket; each round
      every bucket finds its cheapest partner by Ward's criterion (the rise
      of the within-bucket sum of squares, n_a n_b / (n_a + n_b) |mean_a -
      mean_b|^2 over the member pool keys) among the buckets it may join
      without passing 16 raw keys (lower bucket index first on equal cost),
      and all pairs that are each other's cheapest partner merge at once; if
      that would leave fewer than block_size / 8 buckets, only the cheapest
      such pairs merge (cost, then lower indices).  Buckets are indexed by
      their lowest member within the block, and globally block by block.
      Centroid = the normalised sum of the members' pool keys.  The index
      query (R1) is normalised and scores every centroid (cosine); the
      candidates are the buckets with a key outside sink and window (R4);
      the top ``top_k`` buckets (R6 ties) are expanded to their raw keys.
      With ``bucket_keys`` = N > 0 only the N / pool_stride best member pool
      keys by their own cosine with the query (lower position first on
      ties) are kept ("expanded by within-bucket merit to N long-range
      keys"); with 0 every member key is kept.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

NEAR_TIE_REL = 1e-4


@dataclass
class OracleParams:
    """Selection and attention parameters of one problem (sizes in keys)."""

    block_size: int            # b: raw keys per selectable block
    top_k: int                 # k: blocks chosen by score
    sink_keys: int             # S: keys [0, S) always attended
    window_keys: int           # W: keys [C-W, C) always attended
    pool: str = "mean"         # "mean" (SparDA), "lsa" (LSA §2.2) or
                               # "overlap" (SparDA / InfLLM-V2, reading R18)
    pool_stride: int = 4       # LSA: raw keys summed into one pool key;
                               # overlap: keys between window starts (s)
    pool_kernel: int = 0       # overlap: keys per compressed key (l)
    bucket_keys: int = 0       # LSA buckets: long-range key budget N (0 = all)
    scale: Optional[float] = None   # softmax scale; None -> 1/sqrt(d)


# --------------------------------------------------------------------------
# 1. Compression (one slab: K [T, d] float64)
# --------------------------------------------------------------------------

def pool_mean(K: np.ndarray, b: int) -> np.ndarray:
    """Compressed keys by mean pooling  [SparDA, "方法"].

    Kc[j] = (1/b) * sum_{t = j*b}^{j*b + b - 1} K[t]  for every COMPLETE block j
    of the rows given (reading R5: a partial trailing block has no compressed
    key).  Returns [nb, d] with nb = len(K) // b.
    """
    K = np.asarray(K, dtype=np.float64)
    nb = K.shape[0] // b
    out = np.zeros((nb, K.shape[1]), dtype=np.float64)
    for j in range(nb):
        out[j] = K[j * b:(j + 1) * b].sum(axis=0) / b
    return out


def _normalise(x: np.ndarray) -> np.ndarray:
    """x / ||x||_2 along the last axis, with normalise(0) = 0 (reading R7)."""
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def pool_lsa(K: np.ndarray, b: int, stride: int = 4) -> np.ndarray:
    """LSA centroids  [LSA review, §2.2].

    Steps in the page's order: (1) L2-normalise every raw key; (2) sum each
    ``stride`` consecutive unit keys into one pool key; (3) a block of b raw
    keys holds b/stride pool keys and its centroid is the normalised sum of
    them.  Returns [nb, d] unit vectors (or zero rows), nb = len(K) // b.
    """
    assert b % stride == 0
    K = np.asarray(K, dtype=np.float64)
    nb = K.shape[0] // b
    if nb == 0:
        return np.zeros((0, K.shape[1]))                            # no complete block (R5)
    khat = _normalise(K[:nb * b])                                   # (1)
    pool_keys = khat.reshape(nb * b // stride, stride, -1).sum(1)   # (2)
    per_block = b // stride
    cent = np.zeros((nb, K.shape[1]), dtype=np.float64)
    for j in range(nb):                                             # (3)
        cent[j] = pool_keys[j * per_block:(j + 1) * per_block].sum(axis=0)
    return _normalise(cent)


def pool_overlap(K: np.ndarray, kernel: int, stride: int) -> np.ndarray:
    """Overlapping mean-pooled compressed keys  [SparDA, "方法": the keys
    are average-pooled into overlapping compressed representations]
    (reading R18 for the window geometry):

        Kc[c] = (1/kernel) * sum_{t = c*stride}^{c*stride + kernel - 1} K[t]

    for every c whose window lies wholly inside the rows given.  Returns
    [n_c, d] with n_c = (T - kernel) // stride + 1 if T >= kernel, else 0.
    """
    K = np.asarray(K, dtype=np.float64)
    T = K.shape[0]
    n_c = (T - kernel) // stride + 1 if T >= kernel else 0
    out = np.zeros((n_c, K.shape[1]), dtype=np.float64)
    for c in range(n_c):
        out[c] = K[c * stride:c * stride + kernel].sum(axis=0) / kernel
    return out


def compress(K: np.ndarray, p: OracleParams) -> np.ndarray:
    if p.pool == "mean":
        return pool_mean(K, p.block_size)
    if p.pool == "lsa":
        return pool_lsa(K, p.block_size, p.pool_stride)
    if p.pool == "overlap":
        return pool_overlap(K, p.pool_kernel, p.pool_stride)
    raise ValueError(p.pool)


# --------------------------------------------------------------------------
# 2. Scoring
# --------------------------------------------------------------------------

def index_query(q_group: np.ndarray) -> np.ndarray:
    """One index query per GQA group: the sum of the group's query vectors.

    [LSA review, §2.4] (the query side sums the heads into one index query);
    [SparDA, "方法"] (one forecast head per GQA group).  q_group: [G, d].
    """
    return np.asarray(q_group, dtype=np.float64).sum(axis=0)


def softmax_scale(d: int, p: OracleParams) -> float:
    """1/sqrt(d_h)  [PulseCol, §3.1 eq. (1)] unless the caller fixes it."""
    return (1.0 / math.sqrt(d)) if p.scale is None else float(p.scale)


def block_scores(qbar: np.ndarray, Kc: np.ndarray, p: OracleParams) -> np.ndarray:
    """Score of every compressed key.

    mean pooling: s_j = qbar . Kc_j * scale   (reading R1)
    LSA pooling : s_j = (qbar / |qbar|) . c_j (LSA §2.3: the query is
                  normalised before it scores the centroids; reading R7)
    """
    qbar = np.asarray(qbar, dtype=np.float64)
    if p.pool == "lsa":
        return Kc @ _normalise(qbar)
    return (Kc @ qbar) * softmax_scale(Kc.shape[1], p)


def blocks_from_compressed(sigma: np.ndarray, C: int, p: OracleParams) -> np.ndarray:
    """Coarse-to-fine step of overlapping compression (reading R18; SparDA
    "方法"): the score of complete block j, keys [j*b, j*b + b), is the
    largest score among the compressed keys whose window
    [c*s, c*s + l) shares at least one key with the block.  Returns [nb]
    with nb = C // b (-inf for a block no window reaches)."""
    b, l, s = p.block_size, p.pool_kernel, p.pool_stride
    starts = np.arange(len(sigma)) * s
    out = np.full(C // b, -np.inf)
    for j in range(C // b):
        hit = (starts < (j + 1) * b) & (starts + l > j * b)
        if hit.any():
            out[j] = np.max(np.asarray(sigma)[hit])
    return out


# --------------------------------------------------------------------------
# 3. Candidates and top-k
# --------------------------------------------------------------------------

def sink_window(C: int, p: OracleParams):
    """Always-attended context keys: sink [0, S) and window [C-W, C), clipped
    to the context [0, C)  [SparDA, "方法" (initial tokens + local window);
    LSA review §2.3 (4 sink keys + 512 window keys); S3R review, KV-selection
    formula (recent window R)]."""
    s_end = min(p.sink_keys, C)
    w_begin = max(C - p.window_keys, 0)
    return s_end, w_begin


def candidate_blocks(C: int, p: OracleParams) -> List[int]:
    """Blocks that compete in top-k (readings R4, R5): complete blocks of the
    context whose keys are not ALL inside sink or window.

    Sink is the prefix [0, s_end) and window the suffix [w_begin, C), so the
    context keys outside both form the interval [s_end, w_begin); a complete
    block [j*b, j*b + b) competes iff it shares at least one key with it.
    """
    b = p.block_size
    s_end, w_begin = sink_window(C, p)
    out = []
    for j in range(C // b):
        lo, hi = j * b, (j + 1) * b
        if lo < w_begin and hi > s_end:
            out.append(j)
    return out


@dataclass
class Selection:
    selected: List[int]          # ascending block ids
    n_candidates: int
    kth_score: Optional[float]   # score of the k-th ranked candidate
    gap: Optional[float]         # s_(k) - s_(k+1); None when all are taken
    near_tie: bool               # gap < 1e-4 * |s_(k)|  (reading R6)


def select_topk(scores: np.ndarray, candidates: Sequence[int], k: int) -> Selection:
    """Top-k block selection [SparDA, "方法"; S3R review, KV-selection
    formula]: rank candidates by (score descending, block index ascending)
    and keep the first min(k, #candidates).  Returns them in ascending block
    order with the k-th/(k+1)-th gap used for near-tie accounting."""
    cand = list(candidates)
    ranked = sorted(cand, key=lambda j: (-float(scores[j]), j))
    take = ranked[:min(k, len(ranked))]
    kth = float(scores[take[-1]]) if take else None
    gap = None
    near = False
    if len(ranked) > k and k > 0:
        gap = float(scores[ranked[k - 1]]) - float(scores[ranked[k]])
        near = gap < NEAR_TIE_REL * abs(float(scores[ranked[k - 1]]))
    return Selection(sorted(take), len(cand), kth, gap, near)


# --------------------------------------------------------------------------
# 4. Attended set and masked softmax attention
# --------------------------------------------------------------------------

def attended_positions(C: int, p: OracleParams, selected: Sequence[int],
                       last_pos: int) -> np.ndarray:
    """Key positions one query at position ``last_pos`` (>= C) attends:

    {t < S} U {C-W <= t < C} U {t in a selected block} U {C <= t <= last_pos}

    [SparDA, "方法" (initial + local + top-k blocks); S3R review, the retained
    set T = recent window U top-K; reading R3 for the new tokens].  A key
    covered twice is listed once (reading R4).
    """
    b = p.block_size
    s_end, w_begin = sink_window(C, p)
    mask = np.zeros(last_pos + 1, dtype=bool)
    mask[0:s_end] = True
    mask[w_begin:C] = True
    for j in selected:
        mask[j * b:(j + 1) * b] = True
    mask[C:last_pos + 1] = True
    return np.flatnonzero(mask)


def masked_softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                             positions: np.ndarray, scale: float):
    """Attention over the retained set only.

    z_t = q . K_t * scale for t in the set; w = exp(z - max z) / sum exp;
    O = sum_t w_t V_t; lse = max z + log sum exp(z - max z).
    [S3R review, sparse-attention formula: softmax over K_T, weighted sum of
    V_T; PulseCol §3.1 eq. (1)-(2): keys outside the mask get -inf logits, so
    they receive zero weight.]
    Returns (O [d], lse, w [len(positions)]).
    """
    q = np.asarray(q, dtype=np.float64)
    Ks = np.asarray(K[positions], dtype=np.float64)
    Vs = np.asarray(V[positions], dtype=np.float64)
    z = (Ks @ q) * scale
    m = z.max()
    e = np.exp(z - m)
    den = e.sum()
    w = e / den
    O = w @ Vs
    lse = m + math.log(den)
    return O, lse, w


# --------------------------------------------------------------------------
# 5. One (sequence, KV head) pair: decode, draft chunk
# --------------------------------------------------------------------------

def decode_pair(q_tokens: np.ndarray, K: np.ndarray, V: np.ndarray, C: int,
                p: OracleParams, Kc: Optional[np.ndarray] = None) -> Dict:
    """Decode / multi-token chunk for one (sequence, KV head).

    q_tokens: [n_q, G, d] queries of the new tokens for the G query heads of
              this KV head (token j sits at position C + j).
    K, V:     [>= C + n_q, d] this pair's cache rows (new tokens' keys at C..).
    Steps: compress the context keys [0, C) -> index query of token 0 ->
    scores -> candidates -> top-k -> per token j and head g, attention over
    sink U window U selected U chunk keys C..C+j  (reading R9).
    """
    n_q, G, d = q_tokens.shape
    if Kc is None:
        Kc = compress(K[:C], p)
    qbar = index_query(q_tokens[0])
    s = block_scores(qbar, Kc, p)
    if p.pool == "overlap":
        s = blocks_from_compressed(s, C, p)
    cand = candidate_blocks(C, p)
    sel = select_topk(s, cand, p.top_k)
    scale = softmax_scale(d, p)
    O = np.zeros((n_q, G, d))
    lse = np.zeros((n_q, G))
    wsum = np.zeros((n_q, G))
    pos_list = []
    for j in range(n_q):
        pos = attended_positions(C, p, sel.selected, C + j)
        pos_list.append(pos)
        for g in range(G):
            O[j, g], lse[j, g], w = masked_softmax_attention(
                q_tokens[j, g], K, V, pos, scale)
            wsum[j, g] = w.sum()
    return dict(Kc=Kc, qbar=qbar, scores=s, candidates=cand, sel=sel,
                O=O, lse=lse, wsum=wsum, positions=pos_list)


def verify_pair(q_tokens: np.ndarray, K: np.ndarray, V: np.ndarray, C: int,
                p: OracleParams) -> Dict:
    """Dense verify of a draft chunk for one (sequence, KV head), and the
    block selection it refreshes (reading R15).

    [S3R review, "稠密验证": the chunk's candidate tokens go through one causal
    forward with full attention over the dense cache, and the verifier's
    attention weights refresh the subset the drafts use; "稀疏起草",
    KV-selection formula: recent window plus the top-K positions by the
    previous verify's attention scores.]

    q_tokens: [n_q, G, d]; token j sits at position C + j and attends to
    keys 0..C+j.  K, V: [>= C + n_q, d].  Returns O [n_q, G, d], lse
    [n_q, G], mass [nb] (nb = C // b complete blocks: mass_j = sum over
    tokens j' and heads g of the weights on keys [j*b, (j+1)*b)), wtail
    [n_q, G] (weight on the keys past the complete blocks), and the
    Selection of the top-k candidates by mass.
    """
    n_q, G, d = q_tokens.shape
    b = p.block_size
    nb = C // b
    scale = softmax_scale(d, p)
    O = np.zeros((n_q, G, d))
    lse = np.zeros((n_q, G))
    wtail = np.zeros((n_q, G))
    mass = np.zeros(nb)
    for j in range(n_q):
        pos = np.arange(C + j + 1)
        for g in range(G):
            O[j, g], lse[j, g], w = masked_softmax_attention(q_tokens[j, g], K, V, pos, scale)
            mass += w[:nb * b].reshape(nb, b).sum(axis=1)
            wtail[j, g] = w[nb * b:].sum()
    cand = candidate_blocks(C, p)
    sel = select_topk(mass, cand, p.top_k)
    return dict(O=O, lse=lse, mass=mass, wtail=wtail, candidates=cand, sel=sel)


def column_attention_group(q_rows: np.ndarray, K: np.ndarray, V: np.ndarray,
                           cols: Sequence[int], p: OracleParams) -> Dict:
    """Column-sparse attention of one group of query tokens of one (sequence,
    KV head) (reading R17) [PulseCol §3.1: eq. (1) logits Q K^T / sqrt(d_h);
    eq. (2) softmax(Z + M(S)) V with S(i, j) = 1 for the kept key columns j of
    row i: here the same columns for every row of the group, and every key
    position may be kept, before or after the query (bidirectional)].

    q_rows: [n, G, d] the group's tokens x the KV head's query heads; cols:
    key positions (duplicates and negative entries ignored).  Returns O
    [n, G, d], lse [n, G] (O = 0, lse = -inf when no column is kept).
    """
    n, G, d = q_rows.shape
    pos = np.array(sorted({int(c) for c in cols if int(c) >= 0}), dtype=np.int64)
    O = np.zeros((n, G, d))
    lse = np.full((n, G), -np.inf)
    if len(pos) == 0:
        return dict(O=O, lse=lse, positions=pos)
    scale = softmax_scale(d, p)
    for i in range(n):
        for g in range(G):
            O[i, g], lse[i, g], _ = masked_softmax_attention(q_rows[i, g], K, V, pos, scale)
    return dict(O=O, lse=lse, positions=pos)


# --------------------------------------------------------------------------
# 6. Prefill (one KV head): 64-query tiles, tile-max scoring
# --------------------------------------------------------------------------

def context_rows(C: int, p: OracleParams) -> int:
    """Compressed keys a context of C keys holds: its complete blocks (mean
    and LSA pooling, reading R5) or its complete windows (overlapping
    compression, reading R18)."""
    if p.pool == "overlap":
        return (C - p.pool_kernel) // p.pool_stride + 1 if C >= p.pool_kernel else 0
    return C // p.block_size


def prefill_tile_scores(q_rows: np.ndarray, Kc: np.ndarray, p: OracleParams,
                        C: Optional[int] = None) -> np.ndarray:
    """Tile score of each complete block of the context: max over the tile's
    rows of the row's GQA-summed block score (readings R1, R2).  q_rows:
    [rows, G, d]; Kc: the context's compressed keys (context_rows(C, p) of
    them).

    Overlapping compression (readings R2 and R18 together): every window
    takes the max over the rows, then block j the max over the complete
    windows touching it; both steps are maxima, so this is also the max over
    rows of each row's own block score.  C (the tile's context length) is
    needed in that mode only."""
    per_row = np.stack([block_scores(index_query(q_rows[r]), Kc, p)
                        for r in range(q_rows.shape[0])])
    tile = per_row.max(axis=0)
    if p.pool == "overlap":
        if C is None:
            raise ValueError("overlapping compression needs the context length C")
        return blocks_from_compressed(tile, C, p)
    return tile


def prefill_tile(q_tile: np.ndarray, K: np.ndarray, V: np.ndarray, i: int,
                 p: OracleParams, Kc_all: Optional[np.ndarray] = None) -> Dict:
    """Query tile i of a causal prefill (tile size = block size b).

    The tile's queries sit at positions [i*b, i*b + rows); the tile's context
    is C_i = i*b (blocks 0..i-1).  Its selection uses the tile-max score over
    the context's complete blocks; every query row then attends sink U window
    U selected blocks U the causal part of its own tile (readings R2, R3).
    q_tile: [rows, G, d];  K, V: this KV head's rows [T, d].
    """
    b = p.block_size
    C = i * b
    rows, G, d = q_tile.shape
    if Kc_all is None:
        Kc_all = compress(K, p)
    Kc = Kc_all[:context_rows(C, p)]
    s = prefill_tile_scores(q_tile, Kc, p, C) if C // b > 0 else np.zeros(0)
    cand = candidate_blocks(C, p)
    sel = select_topk(s, cand, p.top_k)
    scale = softmax_scale(d, p)
    O = np.zeros((rows, G, d))
    lse = np.zeros((rows, G))
    wsum = np.zeros((rows, G))
    for r in range(rows):
        pos = attended_positions(C, p, sel.selected, C + r)
        for g in range(G):
            O[r, g], lse[r, g], w = masked_softmax_attention(
                q_tile[r, g], K, V, pos, scale)
            wsum[r, g] = w.sum()
    return dict(scores=s, candidates=cand, sel=sel, O=O, lse=lse, wsum=wsum)


def prefill_head_selection(q_head_rows: np.ndarray, Kc_all: np.ndarray,
                           p: OracleParams, tiles: Sequence[int]) -> Dict[int, Selection]:
    """Selections only (no attention) for the given tiles of one KV head.
    q_head_rows: [T, G, d]."""
    b = p.block_size
    out = {}
    for i in tiles:
        q_tile = q_head_rows[i * b:(i + 1) * b]
        C = i * b
        Kc = Kc_all[:context_rows(C, p)]
        s = prefill_tile_scores(q_tile, Kc, p, C) if C // b > 0 else np.zeros(0)
        out[i] = select_topk(s, candidate_blocks(C, p), p.top_k)
    return out


# --------------------------------------------------------------------------
# 7. LSA flat bucket retrieval (reading R19)
# --------------------------------------------------------------------------

def lsa_pool_keys(K: np.ndarray, stride: int = 4) -> np.ndarray:
    """Pool keys [LSA review §2.2]: each raw key L2-normalised, then every
    ``stride`` consecutive unit keys summed.  Returns [len(K) // stride, d]."""
    K = np.asarray(K, dtype=np.float64)
    m = K.shape[0] // stride
    if m == 0:
        return np.zeros((0, K.shape[1]))
    return _normalise(K[:m * stride]).reshape(m, stride, -1).sum(axis=1)


def ward_cost(sum_a, n_a, sum_b, n_b):
    """Ward's merge cost of two buckets given their member sums (last axis)
    and sizes: the rise of the within-bucket sum of squares,
    n_a n_b / (n_a + n_b) * |mean_a - mean_b|^2.  Broadcasts over leading
    axes (all pairs of a round at once)."""
    diff = np.asarray(sum_a) / np.asarray(n_a)[..., None] - np.asarray(sum_b) / np.asarray(n_b)[..., None]
    return np.asarray(n_a) * n_b / (np.asarray(n_a) + n_b) * (diff * diff).sum(axis=-1)


def ward_buckets(P: np.ndarray, n_buckets: int, cap: int, history: Optional[list] = None) -> List[List[int]]:
    """Bottom-up Ward clustering of one cluster block's pool keys P [m, d]
    into n_buckets buckets of at most ``cap`` pool keys  [LSA review §2.2:
    every pool key its own bucket; each round, buckets that are each other's
    cheapest merge merge in parallel; 64 buckets per block, at most 16 keys
    each] (reading R19 for ties and the last round).  Returns the buckets
    as ascending member lists, ordered by their lowest member.  ``history``
    (optional) receives, per round, (bucket list, merged index pairs)."""
    P = np.asarray(P, dtype=np.float64)
    buckets = [[i] for i in range(P.shape[0])]
    while len(buckets) > n_buckets:
        nb = len(buckets)
        sums = np.stack([P[b].sum(axis=0) for b in buckets])
        size = np.array([len(b) for b in buckets], dtype=np.float64)
        # cost[a, b] for every pair; a pair may merge if b != a and it fits the cap
        cost = ward_cost(sums[:, None, :], size[:, None], sums[None, :, :], size[None, :])
        cost = np.where((size[:, None] + size[None, :] <= cap) & ~np.eye(nb, dtype=bool), cost, math.inf)
        best = []
        for a in range(nb):
            part_a = int(np.argmin(cost[a]))            # the first of equal costs: the lower index
            best.append((part_a, float(cost[a, part_a])) if math.isfinite(cost[a, part_a]) else (-1, math.inf))
        pairs = [(best[a][1], a, best[a][0]) for a in range(nb)
                 if best[a][0] > a and best[best[a][0]][0] == a]
        if not pairs:
            raise RuntimeError("no pair of buckets may merge under the size cap")
        pairs.sort()
        pairs = pairs[:nb - n_buckets]
        if history is not None:
            history.append(([list(b) for b in buckets], [(a, b) for _, a, b in pairs]))
        gone = set()
        merged = []
        for _, a, b in pairs:
            merged.append(sorted(buckets[a] + buckets[b]))
            gone.update((a, b))
        buckets = sorted([bk for i, bk in enumerate(buckets) if i not in gone] + merged, key=lambda x: x[0])
    return buckets


def lsa_bucket_index(K: np.ndarray, C: int, p: OracleParams):
    """The bucket cache of a context of C keys (reading R19): for every
    complete cluster block of ``block_size`` raw keys, its block_size / 8
    buckets.  Returns (members, centroids): members[g] = ascending global
    pool-key ids of bucket g, centroids [n, d] unit vectors."""
    b, stride = p.block_size, p.pool_stride
    per = b // stride
    P = lsa_pool_keys(K[:(C // b) * b], stride)
    members, cents = [], []
    for j in range(C // b):
        for bk in ward_buckets(P[j * per:(j + 1) * per], b // 8, 16 // stride):
            ids = [j * per + i for i in bk]
            members.append(ids)
            cents.append(P[ids].sum(axis=0))
    d = K.shape[1]
    cents = _normalise(np.array(cents)) if cents else np.zeros((0, d))
    return members, cents


def bucket_decode_pair(q_tokens: np.ndarray, K: np.ndarray, V: np.ndarray, C: int,
                       p: OracleParams, index=None) -> Dict:
    """Decode / draft chunk for one (sequence, KV head) with LSA's flat bucket
    retrieval [LSA review §2.2-2.3] (reading R19): normalised index query of
    the first new token scores every bucket centroid; the top-k candidate
    buckets are expanded to raw keys and joined with sink, window and the
    chunk (R3, R9); masked softmax attention as in decode_pair.  ``index``
    (optional) is this context's (members, centroids) as lsa_bucket_index
    returns them, when the caller has built it already."""
    n_q, G, d = q_tokens.shape
    stride = p.pool_stride
    members, cents = lsa_bucket_index(K, C, p) if index is None else index
    qhat = _normalise(index_query(q_tokens[0]))
    scores = cents @ qhat if len(members) else np.zeros(0)
    s_end, w_begin = sink_window(C, p)
    cand = [g for g, ids in enumerate(members)
            if any(s_end <= stride * m + r < w_begin for m in ids for r in range(stride))]
    sel = select_topk(scores, cand, p.top_k)
    kept = sorted(m for g in sel.selected for m in members[g])
    if p.bucket_keys > 0:
        P = lsa_pool_keys(K[:(C // p.block_size) * p.block_size], stride)
        own = {m: float(_normalise(P[m]) @ qhat) for m in kept}
        kept = sorted(sorted(kept, key=lambda m: (-own[m], m))[:p.bucket_keys // stride])
    scale = softmax_scale(d, p)
    O = np.zeros((n_q, G, d))
    lse = np.zeros((n_q, G))
    pos_list = []
    for j in range(n_q):
        mask = np.zeros(C + j + 1, dtype=bool)
        mask[0:s_end] = True
        mask[w_begin:C] = True
        for m in kept:
            mask[m * stride:(m + 1) * stride] = True
        mask[C:C + j + 1] = True
        pos = np.flatnonzero(mask)
        pos_list.append(pos)
        for g in range(G):
            O[j, g], lse[j, g], _ = masked_softmax_attention(q_tokens[j, g], K, V, pos, scale)
    return dict(members=members, centroids=cents, scores=scores, candidates=cand, sel=sel,
                kept=kept, O=O, lse=lse, positions=pos_list)

