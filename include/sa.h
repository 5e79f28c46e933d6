/*
 * sa.h - C ABI of the B200 (sm_100a) indexer-driven top-k block-sparse
 * attention library (libsa.so).
 *
 * The method (sources are web pages on it; each entry point cites the passage
 * that defines its operation):
 *   1. keys of every complete block of b keys are compressed: mean-pooled
 *      (SparDA summary on hyper.ai 2606.04511, section "方法": keys are
 *      average-pooled into compressed keys), or LSA-style: each key
 *      L2-normalised, 4 consecutive unit keys summed into a pool key, the
 *      block centroid = the normalised sum of its pool keys (LSA review,
 *      §2.2); or into OVERLAPPING windows (SparDA "方法": InfLLM-V2 pools
 *      keys into overlapping compressed representations, coarse to fine),
 *      a block then scoring as the best window that touches it;
 *   2. one index query per (sequence, KV head) = the SUM of the query vectors
 *      of the GQA group (LSA review §2.4; SparDA "方法": one forecast head per
 *      GQA group) scores every compressed key: s_j = qbar.Kc_j * scale, or the
 *      cosine (qbar/|qbar|).c_j for LSA centroids (LSA review §2.3);
 *   3. the top-k candidate blocks (score descending, lower block id on ties)
 *      are united with the sink keys [0, S) and the window keys [C-W, C)
 *      (SparDA "方法": initial tokens + local sliding window + top-k blocks;
 *      LSA review §2.3: 4 sink keys + 512 window keys; S3R review, section
 *      "稀疏起草", KV-selection formula: recent window + top-K).  Blocks lying
 *      wholly inside sink or window are not candidates; only complete blocks
 *      of the context are;
 *   4. softmax attention runs over the retained keys only (S3R review,
 *      "稀疏起草", sparse-attention formula; PulseCol §3.1 eq. (1)-(2): logits
 *      QK^T/sqrt(d_h), keys outside the mask get zero weight).  The n_q new
 *      tokens sit at positions C..C+n_q-1 and token j also sees the new keys
 *      C..C+j (a multi-token draft chunk keeps one selection, made from its
 *      first query, for all its tokens: S3R review, "稀疏起草").
 *
 * Layouts (all row-major, contiguous, element strides implied):
 *   K, V : [B, Hkv, kv_capacity, d]   dtype = params.dtype
 *   Q    : [B, n_q, Hq, d]            dtype = params.dtype
 *   O    : [B, n_q, Hq, d]            dtype = params.out_dtype
 *   lse  : [B, n_q, Hq] float32, natural log of the softmax denominator
 *   Kc   : [B, Hkv, nb, d] float32, nb = number of complete blocks
 *          (decode: floor(ctx_len / b); prefill: floor(n_q / b));
 *          SA_POOL_OVERLAP: [B, Hkv, n_c, d], n_c = the number of complete
 *          windows = floor((L - l) / s) + 1 if L >= l, else 0, with L =
 *          ctx_len (decode) or n_q (prefill)
 *   idx  : decode / chunk: [B, Hkv, top_k] int32; prefill: [B, Hkv,
 *          n_tiles, top_k] int32 with n_tiles = ceil(n_q / b).  Block ids in
 *          ascending order, unused entries -1 at the end.
 *   Query head h uses KV head h / (Hq / Hkv).
 *
 * Ownership: the caller allocates every buffer, including the workspace; the
 * library allocates no device or host memory and keeps no state besides a
 * per-thread error string and cached device attributes.  Every call is
 * asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream).
 * Pointers are device pointers unless stated; K, V, Q, O, Kc must be 16-byte
 * aligned.
 *
 * Errors: arguments are validated on the host before any launch
 * (SA_ERR_INVALID / SA_ERR_UNSUPPORTED / SA_ERR_WORKSPACE, with a message in
 * sa_last_error(); sizes are refused as SA_ERR_UNSUPPORTED when B x Hkv or
 * B x n_q x Hq reaches 2^31, kv_capacity passes 2^40 or B x Hkv x
 * kv_capacity passes 2^48); a failed launch returns SA_ERR_CUDA.  Conditions found on
 * the device (an out-of-range or repeated block id in a caller's index table,
 * a bounded wait that ran out) set bits of a status word kept in the
 * workspace; the affected block is skipped and sa_read_status() reports
 * them.  No kernel traps or asserts.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID = 1,      /* bad argument (null, shape, alignment, range) */
  SA_ERR_UNSUPPORTED = 2,  /* valid but not built (head_dim != 128, sizes above limits) */
  SA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than sa_workspace_size() */
  SA_ERR_INDEX = 4,        /* device: a caller's block id was out of range or repeated */
  SA_ERR_CUDA = 5,         /* a CUDA launch or runtime call failed */
  SA_ERR_TIMEOUT = 6       /* device: a bounded wait inside a kernel ran out */
} sa_status;

enum { SA_F32 = 0, SA_BF16 = 1 };                 /* element types */
enum { SA_POOL_MEAN = 0, SA_POOL_LSA = 1, SA_POOL_OVERLAP = 2 };  /* compression (step 1) */
enum { SA_SEL_QUERY0 = 0, SA_SEL_TILE_MAX = 1 };  /* how the index query is formed */
enum {                                            /* ops for sa_workspace_size */
  SA_OP_SCORE_TOPK = 0,
  SA_OP_GIVEN_IDX = 1,
  SA_OP_DECODE = 2,
  SA_OP_PREFILL = 3,
  SA_OP_VERIFY = 4,
  SA_OP_COLUMN = 5,
  SA_OP_BUCKET_DECODE = 6
};

/* Problem description shared by every entry point (96 bytes). */
typedef struct sa_params {
  int32_t batch;          /* B >= 1 */
  int32_t num_q_heads;    /* Hq, a multiple of Hkv */
  int32_t num_kv_heads;   /* Hkv >= 1 */
  int32_t head_dim;       /* d; only 128 is built */
  int64_t ctx_len;        /* C: keys cached before the new tokens (prefill: 0) */
  int64_t kv_capacity;    /* token stride of K and V, >= ctx_len + n_q */
  int32_t n_q;            /* new tokens per sequence (decode 1, draft chunk m, prefill T) */
  int32_t block_size;     /* b: keys per selectable block (a multiple of 16) */
  int32_t pool;           /* SA_POOL_MEAN, SA_POOL_LSA or SA_POOL_OVERLAP */
  int32_t pool_stride;    /* LSA: raw keys per pool key (divides b);
                             OVERLAP: s, keys between window starts (divides b);
                             ignored for mean */
  int32_t top_k;          /* k >= 0 blocks chosen by score */
  int32_t dtype;          /* SA_F32 or SA_BF16: element type of Q, K, V */
  int32_t out_dtype;      /* SA_F32 or SA_BF16: element type of O */
  int32_t select;         /* SA_SEL_QUERY0: decode / chunk (index query of the
                             chunk's first token); SA_SEL_TILE_MAX: causal
                             prefill (query tiles of b rows, ctx_len == 0) */
  int64_t sink_keys;      /* S >= 0 */
  int64_t window_keys;    /* W >= 0 */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim) */
  int32_t flags;          /* OR of SA_FLAG_* (other bits must be 0) */
  int32_t pool_kernel;    /* OVERLAP: l, keys per window, s <= l <= b; must be
                             0 for the other pool modes */
} sa_params;

/* sa_params.flags: the caller's index table is known to hold only
 * ascending in-range block ids and -1 (e.g. it came from sa_score_topk), so
 * sa_sparse_attn_given_idx[_noalloc] skips its checking pass. */
#define SA_FLAG_TRUSTED_IDX 1

/* Version of this ABI (major * 100 + minor). */
int32_t sa_version(void);

/* Bytes of workspace `op` needs for `p` (0 if p is invalid or refused).  The workspace
 * also carries the device status word and self-resetting counters, so it
 * must be zero-filled once before its first use (sa_workspace_init) and may
 * then be reused by later calls on the same stream.  Calls that share one
 * workspace must not overlap on the device. */
size_t sa_workspace_size(const sa_params* p, int32_t op);

/* Zero-fills `ws_bytes` bytes at device pointer `ws` on `stream`. */
sa_status sa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Step 1 (compression) for every complete block of the context:
 * SA_POOL_MEAN: Kc[j] = (1/b) sum_{t=jb}^{jb+b-1} K[t] (SparDA "方法");
 * SA_POOL_OVERLAP: Kc[c] = (1/l) sum_{t=cs}^{cs+l-1}
 *               K[t] for every complete window c (l = pool_kernel,
 *               s = pool_stride; SparDA "方法", overlapping compressed keys);
 * SA_POOL_LSA : Kc[j] = normalise(sum over the block's pool keys), a pool
 *               key being the sum of pool_stride consecutive L2-normalised
 *               keys (LSA review §2.2).
 * Blocks counted over ctx_len keys (prefill: over n_q keys).  Reads K,
 * writes Kc (fp32, see layouts).  No workspace. */
sa_status sa_pool_keys(const sa_params* p, const void* K, float* Kc, void* stream);

/* Cache append for decode / draft chunks (select == SA_SEL_QUERY0): the n_q
 * new tokens' keys and values go to rows ctx_len .. ctx_len + n_q - 1 of the
 * cache, K[b, h, ctx_len + t, :] = K_new[b, h, t, :] and the same for V.
 * K_new, V_new: [B, Hkv, n_q, d] in dtype, contiguous, 16-byte aligned; K, V
 * as in the layouts (ctx_len + n_q <= kv_capacity is checked).  Compressed
 * keys are not touched: call sa_pool_keys when a block fills.  Asynchronous
 * on `stream`; one kernel, no workspace. */
sa_status sa_append_kv(const sa_params* p, const void* K_new, const void* V_new,
                       void* K, void* V, void* stream);

/* Steps 2-3 (scoring and selection).  SA_SEL_QUERY0: one table row per
 * (sequence, KV head) from the first new token's GQA-summed query.
 * SA_SEL_TILE_MAX: one row per (sequence, KV head, query tile of b rows),
 * the tile score of block j being the max over the tile's rows (reading of
 * the pages, which do not fix the tile aggregation).  Writes idx (see
 * layouts).  scores (optional, may be NULL): fp32 block scores,
 * [B, Hkv, nb] for SA_SEL_QUERY0 or [B, Hkv, n_tiles, nb] for
 * SA_SEL_TILE_MAX.  Kc may be NULL when the context holds no complete
 * block.  SA_POOL_OVERLAP: every window is scored as above and block j
 * takes the largest score among the complete windows [cs, cs + l) that
 * share a key with [jb, jb + b) (the coarse-to-fine step; the pages do not
 * fix the rule, the max is this library's reading); with SA_SEL_TILE_MAX a
 * tile sees the windows complete inside its context (keys before the tile),
 * each window taking the max over the tile's rows first.  scores then holds
 * those block scores.  SA_POOL_LSA with SA_SEL_TILE_MAX: each row's index
 * query is normalised, so the tile score is the largest row cosine. */
sa_status sa_score_topk(const sa_params* p, const void* Q, const float* Kc,
                        int32_t* idx, float* scores, void* ws, size_t ws_bytes,
                        void* stream);

/* Step 4 alone with the CALLER's index table (a page table of selected
 * blocks, as LSA review §2.6 feeds its attention kernel).  idx holds
 * idx_len entries per row (layout as above with top_k replaced by idx_len);
 * entries are block ids in [0, nb) in strictly ascending order, -1 for none.
 * Attended set per token = sink U window U listed blocks U new keys up to the
 * token; keys of a listed block that lie in sink or window count once.  An
 * entry is used only if it is in [0, nb) and larger than every earlier
 * in-range entry of its row; any other entry except -1 sets SA_ERR_INDEX in
 * the status word and is skipped.  Writes O and (if non-NULL) lse.  The
 * workspace size reported for SA_OP_GIVEN_IDX assumes idx_len == top_k. */
sa_status sa_sparse_attn_given_idx(const sa_params* p, const void* Q,
                                   const void* K, const void* V,
                                   const int32_t* idx, int32_t idx_len,
                                   void* O, float* lse, void* ws,
                                   size_t ws_bytes, void* stream);

/* Steps 2-4 for decode and draft chunks (select == SA_SEL_QUERY0) with the
 * compressed keys Kc kept up to date by the caller (sa_pool_keys).  Writes
 * O, lse (optional) and the index table (optional idx_out, [B, Hkv, top_k]).
 * Runs as one cooperative launch where sa_decode_launches(p) == 1, else as
 * the scoring + top-k kernel followed by the attention kernel. */
sa_status sa_sparse_attn_decode(const sa_params* p, const void* Q,
                                const void* K, const void* V, const float* Kc,
                                void* O, float* lse, int32_t* idx_out,
                                void* ws, size_t ws_bytes, void* stream);

/* Dense verify of a draft chunk and the block selection it refreshes
 * (S3R review, section "稠密验证": the chunk's tokens go through one causal
 * forward with full attention over the dense cache, and the verifier's
 * attention weights refresh the subset the drafts read; section "稀疏起草",
 * KV-selection formula: recent window plus the top-K positions by the
 * previous verify's attention scores).
 *
 * The n_q tokens at positions C..C+n_q-1 (Q [B, n_q, Hq, d], their keys
 * already at rows C.. of K and V) attend causally to EVERY key 0..C+j: no
 * selection, sink_keys and window_keys do not restrict it.  Outputs:
 *   O       [B, n_q, Hq, d] in out_dtype, lse [B, n_q, Hq] fp32 (natural
 *           log; may be NULL);
 *   mass    [B, Hkv, nb] fp32, nb = C / block_size: for each complete context
 *           block, the attention weight its keys receive summed over the n_q
 *           tokens and the KV head's G query heads (so the masses of a pair
 *           plus the weight on the keys past the complete blocks total
 *           n_q * G);
 *   idx_out [B, Hkv, top_k] int32: the top_k candidate blocks by mass
 *           (candidates and ties as in sa_score_topk: blocks not wholly
 *           inside [0, sink_keys) or the last window_keys context keys;
 *           higher mass first, then the lower block id), ascending, -1
 *           padded; may be NULL when top_k == 0.
 * Built for dtype SA_BF16, block_size a multiple of 64, n_q * (Hq / Hkv)
 * <= 16 rows per KV head (else SA_ERR_UNSUPPORTED); pool fields are
 * ignored; select must be SA_SEL_QUERY0.  Device buffers, 16-byte aligned;
 * the caller owns all of them, the workspace (sa_workspace_size(p,
 * SA_OP_VERIFY)) included.  Asynchronous on `stream`: three launches (the
 * dense attention, which also keeps per-32-key row sums of the complete
 * blocks, the block masses, the top-k); K and V are read once. */
sa_status sa_verify_refresh(const sa_params* p, const void* Q, const void* K,
                            const void* V, void* O, float* lse, float* mass,
                            int32_t* idx_out, void* ws, size_t ws_bytes,
                            void* stream);

/* Column-sparse attention (PulseCol §3.1, eq. (1) logits QK^T/sqrt(d_h) and
 * eq. (2) softmax(Z + M(S)) V, with a token-granular column mask S): every
 * group of 64 consecutive query tokens of a (sequence, KV head) and the
 * KV head's 4 query heads attend to the key positions listed for the group,
 * before or after them alike (no causal mask, no sink or window).
 *
 * p describes a full sequence as in prefill: select = SA_SEL_TILE_MAX,
 * ctx_len = 0, n_q = T tokens, block_size = 64 (the group), Hq / Hkv a
 * multiple of 4, bf16;
 * top_k, sink_keys, window_keys and pool are ignored.  Q [B, T, Hq, d];
 * K, V [B, Hkv, kv_capacity, d] (rows 0..T-1 are the keys); cols [B, Hkv,
 * ceil(T/64), n_cols] int32: per group, key positions in [0, T), ascending,
 * -1 padded.  Unless p->flags has SA_FLAG_TRUSTED_IDX the table is checked
 * first: entries out of range or not above every earlier kept entry are
 * dropped and set SA_ERR_INDEX in the workspace status (the rest are used).
 * An empty list gives O = 0 and lse = -inf for its rows.  Outputs O
 * [B, T, Hq, d] in out_dtype, lse [B, T, Hq] fp32 (may be NULL).
 * Workspace: sa_workspace_size(p, SA_OP_COLUMN) sized for n_cols ==
 * p->top_k.  Asynchronous on `stream`: one tensor-core launch (the K and V
 * rows gathered by 16-byte copies), plus the table check. */
sa_status sa_column_attn(const sa_params* p, const void* Q, const void* K,
                         const void* V, const int32_t* cols, int32_t n_cols,
                         void* O, float* lse, void* ws, size_t ws_bytes,
                         void* stream);

/* Number of kernels one sa_sparse_attn_decode call with `p` launches on this
 * device: 1 when scoring, top-k and attention run as one cooperative launch
 * (bf16, SA_POOL_MEAN or SA_POOL_LSA, at most 512 complete blocks or, for
 * top_k <= 8, up to 16384 while each SM scores at most 4 x 128 of them and a
 * (sequence, KV head) pair's are scored on at most 31 SMs, at most 4 query rows (n_q x Hq /
 * Hkv) per KV head and at most two (sequence, KV head) pairs per SM), else
 * 2; 0 if p is
 * invalid.  A cooperative launch the device refuses at run time falls back
 * to the 2-kernel path.  Host only; launches nothing. */
int32_t sa_decode_launches(const sa_params* p);

/* Steps 1-4 for a causal prefill (select == SA_SEL_TILE_MAX, ctx_len == 0,
 * n_q = T): pools K into Kc (caller-provided, [B, Hkv, floor(T/b), d] fp32;
 * SA_POOL_OVERLAP: [B, Hkv, n_c, d] as in the layouts), scores every query
 * tile of b rows against the compressed keys before it (the tile max over
 * its rows; LSA centroids by each row's cosine; overlapping windows as in
 * sa_score_topk), selects per (tile, KV head) and runs causal sparse
 * attention: tile i attends sink U window U selected U its own keys
 * (causal).  Writes O, lse (optional), idx_out (optional).  Built for bf16,
 * b = 64, Hq / Hkv a multiple of 4, sink and window multiples of 64 (else
 * SA_ERR_UNSUPPORTED). */
sa_status sa_sparse_attn_prefill(const sa_params* p, const void* Q,
                                 const void* K, const void* V, float* Kc,
                                 void* O, float* lse, int32_t* idx_out,
                                 void* ws, size_t ws_bytes, void* stream);

/* LSA flat bucket retrieval, building the bucket cache (LSA review
 * "精读:LSA", §2.2 "语义聚类:流式 Ward 装桶").  Needs pool == SA_POOL_LSA,
 * pool_stride (raw keys per pool key) 1, 2 or 4, and block_size = b raw keys
 * per cluster block with b / pool_stride <= 128.  For every (sequence, KV
 * head) and every complete cluster block c in [first_block, ctx_len / b):
 * each raw key is L2-normalised (a zero key stays zero), pool_stride
 * consecutive unit keys are summed into a pool key, and the block's
 * b / pool_stride pool keys are clustered bottom-up by Ward's criterion (the
 * rise n_a n_b / (n_a + n_b) |mean_a - mean_b|^2 of the within-bucket sum of
 * squares): all start as singletons; every round each bucket takes the
 * cheapest partner it may join without passing 16 raw keys (lower index on
 * equal cost), and all pairs that chose each other merge, unless that would
 * leave fewer than b / 8 buckets, in which case only the cheapest such pairs
 * merge (cost, then lower index); rounds repeat until b / 8 buckets remain.
 * Buckets are ordered by their lowest pool key.  Blocks before first_block
 * are left as they are (a cluster block's buckets never change once built,
 * so a decode loop calls this with first_block = the blocks built so far).
 * Writes, per pair, rows [c * b / 8, (c + 1) * b / 8) of
 *   centroids [B, Hkv, R, d] fp32: the normalised sum of the bucket's pool keys;
 *   members   [B, Hkv, R, 16 / pool_stride] int32: the bucket's global pool-key
 *             ids ascending (pool key i = raw keys [i * pool_stride, (i + 1) *
 *             pool_stride)), -1 padded;
 * with R = floor(kv_capacity / b) * b / 8 rows per pair (room for every
 * cluster block the cache can hold).  Reads K only; no workspace.  One launch,
 * one CTA per (pair, cluster block). */
sa_status sa_bucket_build(const sa_params* p, const void* K, int64_t first_block,
                          float* centroids, int32_t* members, void* stream);

/* LSA flat bucket retrieval, a decode / draft-chunk step (LSA review §2.3
 * "检索:flat 打分与 tree 下降"; S3R review "稀疏起草" for the chunk), on the
 * bucket cache sa_bucket_build wrote for the ctx_len / b complete cluster
 * blocks.  The index query of (sequence, KV head) is the sum of its query
 * heads of the chunk's FIRST token, normalised; it scores every bucket's
 * centroid (cosine).  A bucket is a candidate if one of its raw keys lies
 * outside sink [0, S) and window [C - W, C); the top_k candidates by score
 * (lower bucket first on ties) are selected.  Their member pool keys are
 * expanded: with bucket_keys = N > 0 (a multiple of pool_stride) only the
 * N / pool_stride members of best own cosine with the index query are kept
 * (lower position first on ties), with 0 every member is kept.  Every token j
 * of the chunk then attends sink U window U the kept pool keys' raw keys U
 * chunk keys C..C+j (a key counted once), softmax scale as in decode.
 * Writes O [B, n_q, Hq, d], lse (optional) [B, n_q, Hq], sel_out (optional)
 * [B, Hkv, top_k] selected buckets ascending, -1 padded, kept_out (optional)
 * [B, Hkv, K'] kept pool keys ascending, -1 padded, K' = min(N / pool_stride,
 * top_k * 16 / pool_stride) if N > 0, else top_k * 16 / pool_stride.
 * top_k * 16 / pool_stride <= 4096, and ceil(buckets / 8192) * min(top_k,
 * 8192) <= 28672 (the selection keeps each 8192 buckets' top-k, then the
 * top-k of those in shared memory; with top_k = 256, contexts up to 7.3M
 * keys at b = 512).  Workspace: sa_workspace_size(p,
 * SA_OP_BUCKET_DECODE) (enough for any bucket_keys), zero-filled once.
 * Kernels: centroid scores, top-k, (own cosines,) expansion, attention. */
sa_status sa_bucket_decode(const sa_params* p, const void* Q, const void* K,
                           const void* V, const float* centroids,
                           const int32_t* members, int32_t bucket_keys, void* O,
                           float* lse, int32_t* sel_out, int32_t* kept_out,
                           void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of sa_sparse_attn_given_idx (the paper has no
 * counterpart; it exists for callers that cannot allocate device memory,
 * e.g. code inside a framework whose allocator must not be re-entered or
 * plug-ins that are handed only their input and output buffers).  Same
 * arguments, layouts and results as sa_sparse_attn_given_idx without the
 * workspace: the kernel's scratch lives in a 16 MiB static device array that
 * every device loading the library holds until exit.  Problems needing more
 * scratch are rejected with SA_ERR_WORKSPACE before any launch.  The first
 * call on a device looks up the array's device address (with that device
 * current); make that first call before any stream capture.  All calls share
 * the one array, so calls that overlap on the device race: issue them on one
 * stream or otherwise order them.  Each call clears the array's status word
 * and tickets first; bad index entries are skipped exactly as in
 * sa_sparse_attn_given_idx but cannot be read back (there is no workspace to
 * pass to sa_read_status).  Only decode and draft-chunk tables
 * (select == SA_SEL_QUERY0) are taken: prefill tables (SA_SEL_TILE_MAX)
 * return SA_ERR_UNSUPPORTED; pass those to sa_sparse_attn_given_idx.  The
 * array's address is looked up once per device ordinal and kept: after a
 * cudaDeviceReset of that device the kept address is stale, so reload the
 * library before calling this entry point again.  Calls no allocating
 * routine. */
sa_status sa_sparse_attn_given_idx_noalloc(const sa_params* p, const void* Q,
                                           const void* K, const void* V,
                                           const int32_t* idx, int32_t idx_len,
                                           void* O, float* lse, void* stream);

/* Synchronises `stream`, returns the worst device condition recorded in the
 * workspace status word since the last call (SA_OK, SA_ERR_INDEX or
 * SA_ERR_TIMEOUT) and clears it. */
sa_status sa_read_status(void* ws, void* stream);

/* Static name of a status code. */
const char* sa_status_string(sa_status s);

/* Message of the last error returned on the calling thread ("" if none). */
const char* sa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
