// C ABI of libsa.so: argument validation, workspace layout, launch planning.
// Every entry point validates on the host before launching anything and
// never allocates memory; see include/sa.h for the contract.
#include <algorithm>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "cache_ops.h"
#include "internal.h"
#include "sa.h"

namespace sa {
namespace {

thread_local char g_err[512] = "";

sa_status fail(sa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

sa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared validation of sa_params.  `prefill` selects the SA_SEL_TILE_MAX rules.
sa_status check_params(const sa_params* p, bool prefill) {
  if (!p) return fail(SA_ERR_INVALID, "params is NULL");
  if ((p->flags & ~SA_FLAG_TRUSTED_IDX) != 0) return fail(SA_ERR_INVALID, "params.flags has unknown bits");
  if (p->batch < 1 || p->num_kv_heads < 1 || p->num_q_heads < 1)
    return fail(SA_ERR_INVALID, "batch, num_q_heads and num_kv_heads must be >= 1");
  if (p->num_q_heads % p->num_kv_heads != 0)
    return fail(SA_ERR_INVALID, "num_q_heads (%d) must be a multiple of num_kv_heads (%d)", p->num_q_heads,
                p->num_kv_heads);
  if (p->head_dim != kHeadDim) return fail(SA_ERR_UNSUPPORTED, "head_dim %d: only 128 is built", p->head_dim);
  if (p->dtype != SA_F32 && p->dtype != SA_BF16) return fail(SA_ERR_INVALID, "dtype %d", p->dtype);
  if (p->out_dtype != SA_F32 && p->out_dtype != SA_BF16) return fail(SA_ERR_INVALID, "out_dtype %d", p->out_dtype);
  if (p->n_q < 1) return fail(SA_ERR_INVALID, "n_q must be >= 1");
  if (p->ctx_len < 0) return fail(SA_ERR_INVALID, "ctx_len must be >= 0");
  if (p->kv_capacity < p->ctx_len + p->n_q)
    return fail(SA_ERR_INVALID, "kv_capacity (%lld) < ctx_len + n_q (%lld)", (long long)p->kv_capacity,
                (long long)(p->ctx_len + p->n_q));
  // index arithmetic: (sequence, KV head) pairs and query rows are counted in
  // 32-bit integers, cache rows in 64-bit ones
  {
    const int64_t pairs = static_cast<int64_t>(p->batch) * p->num_kv_heads;
    const int64_t q_rows = static_cast<int64_t>(p->batch) * p->n_q * p->num_q_heads;
    if (pairs > INT32_MAX || q_rows > INT32_MAX)
      return fail(SA_ERR_UNSUPPORTED, "batch x heads x n_q too large (%lld query rows, %lld pairs)",
                  (long long)q_rows, (long long)pairs);
    if (p->kv_capacity > (int64_t(1) << 40) || pairs * p->kv_capacity > (int64_t(1) << 48))
      return fail(SA_ERR_UNSUPPORTED, "cache of %lld pairs x %lld rows too large", (long long)pairs,
                  (long long)p->kv_capacity);
  }
  if (p->block_size < 16 || p->block_size % 16 != 0 || p->block_size > 65536)
    return fail(SA_ERR_INVALID, "block_size %d must be a multiple of 16 in [16, 65536]", p->block_size);
  if (p->pool != SA_POOL_MEAN && p->pool != SA_POOL_LSA && p->pool != SA_POOL_OVERLAP)
    return fail(SA_ERR_INVALID, "pool %d", p->pool);
  if ((p->pool == SA_POOL_LSA || p->pool == SA_POOL_OVERLAP) &&
      (p->pool_stride < 1 || p->block_size % p->pool_stride != 0))
    return fail(SA_ERR_INVALID, "pool_stride %d must divide block_size %d", p->pool_stride, p->block_size);
  if (p->pool == SA_POOL_OVERLAP && (p->pool_kernel < p->pool_stride || p->pool_kernel > p->block_size))
    return fail(SA_ERR_INVALID, "pool_kernel %d must lie in [pool_stride %d, block_size %d]", p->pool_kernel,
                p->pool_stride, p->block_size);
  if (p->pool != SA_POOL_OVERLAP && p->pool_kernel != 0)
    return fail(SA_ERR_INVALID, "pool_kernel must be 0 unless pool = SA_POOL_OVERLAP");
  if (p->top_k < 0 || p->top_k > 4096) return fail(SA_ERR_INVALID, "top_k %d must be in [0, 4096]", p->top_k);
  if (p->sink_keys < 0 || p->window_keys < 0) return fail(SA_ERR_INVALID, "sink_keys and window_keys must be >= 0");
  if (p->select != SA_SEL_QUERY0 && p->select != SA_SEL_TILE_MAX) return fail(SA_ERR_INVALID, "select %d", p->select);
  if (prefill) {
    if (p->select != SA_SEL_TILE_MAX) return fail(SA_ERR_INVALID, "prefill needs select = SA_SEL_TILE_MAX");
    if (p->ctx_len != 0) return fail(SA_ERR_INVALID, "prefill needs ctx_len = 0 (n_q is the sequence length)");
  } else if (p->select != SA_SEL_QUERY0) {
    return fail(SA_ERR_INVALID, "decode / chunk calls need select = SA_SEL_QUERY0");
  }
  return SA_OK;
}

DecodeGeom decode_geom(const sa_params* p) {
  DecodeGeom g;
  g.B = p->batch;
  g.Hq = p->num_q_heads;
  g.Hkv = p->num_kv_heads;
  g.G = p->num_q_heads / p->num_kv_heads;
  g.n_q = p->n_q;
  g.R = g.n_q * g.G;
  g.C = p->ctx_len;
  g.cap = p->kv_capacity;
  g.kv_end = p->ctx_len + p->n_q;
  g.b = p->block_size;
  g.nb = p->ctx_len / p->block_size;
  g.kc_rows = g.nb;
  g.n_rows = g.nb;
  g.ov_s = g.ov_l = 0;
  if (p->pool == SA_POOL_OVERLAP) {
    g.ov_s = p->pool_stride;
    g.ov_l = p->pool_kernel;
    g.kc_rows = g.C >= g.ov_l ? (g.C - g.ov_l) / g.ov_s + 1 : 0;
    // windows starting at or past the last complete block's end touch no
    // complete block (s divides b, so block j's windows start below (j+1)b)
    g.n_rows = std::min<int64_t>(g.kc_rows, g.nb * (g.b / g.ov_s));
  }
  g.s_end = p->sink_keys < g.C ? p->sink_keys : g.C;
  const int64_t wb = g.C - p->window_keys;
  g.w_begin = wb > g.s_end ? wb : g.s_end;
  g.pairs = g.B * g.Hkv;
  return g;
}

float scale_of(const sa_params* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->head_dim));
}

// Workspace layout of the decode-type ops.
struct DecodeWs {
  size_t score_cnt, attn_cnt, scores, idx, clean_idx, part_O, part_ml, ready, exit_cnt, cand, total;
};

// idx_len: entries per row of a caller's index table (SA_OP_GIVEN_IDX).
DecodeWs decode_ws(const DecodeGeom& g, const DecodePlan& plan, int top_k, int op, int idx_len = 0) {
  DecodeWs w = {};
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t pairs = static_cast<size_t>(g.pairs);
  w.score_cnt = take(pairs * 4);
  w.attn_cnt = take(pairs * 4);
  if (op == SA_OP_SCORE_TOPK || op == SA_OP_DECODE) {
    w.scores = take(pairs * static_cast<size_t>(std::max(g.nb, g.n_rows)) * 4);
  }
  if (op == SA_OP_DECODE) {
    w.idx = take(pairs * static_cast<size_t>(top_k) * 4);
    w.ready = take(pairs * 4);       // fused decode: per-pair table flags
    w.exit_cnt = take(4);
    w.cand = take(pairs * kFusedCandSlots * kFusedSmallK * 8);   // fused decode past 512 blocks
  }
  if (op == SA_OP_GIVEN_IDX) w.clean_idx = take(pairs * static_cast<size_t>(idx_len) * 4);
  if (op == SA_OP_DECODE || op == SA_OP_GIVEN_IDX) {
    const size_t slots = pairs * static_cast<size_t>(plan.n_slots) * plan.R4;
    w.part_O = take(slots * kHeadDim * 4);
    w.part_ml = take(slots * 2 * 4);
  }
  w.total = off;
  return w;
}

sa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(SA_ERR_WORKSPACE, "workspace is NULL (needs %zu bytes)", need);
  if (!aligned16(ws)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  if (ws_bytes < need) return fail(SA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return SA_OK;
}

sa_status plan_for(const sa_params* p, int idx_slots, DecodeGeom* g, DecodePlan* plan) {
  *g = decode_geom(p);
  const char* why = "";
  if (!plan_decode(*g, idx_slots, p->dtype == SA_BF16, device_sms(), plan, &why))
    return fail(SA_ERR_UNSUPPORTED, "%s", why);
  return SA_OK;
}

// caller_scores may be null; the workspace receives the scores when a pair
// is split over several CTAs.
ScoreArgs score_args(const sa_params* p, const DecodeGeom& g, const void* Q, const float* Kc,
                     float* caller_scores, int32_t* idx, unsigned char* ws, const DecodeWs& L) {
  float* ws_scores = reinterpret_cast<float*>(ws + L.scores);
  unsigned* counters = reinterpret_cast<unsigned*>(ws + L.score_cnt);
  ScoreArgs a = {};
  a.Q = Q;
  a.Kc = Kc;
  a.idx = idx;
  a.counters = counters;
  a.status = reinterpret_cast<unsigned*>(ws);
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.G;
  a.n_q = g.n_q;
  a.nb = g.nb;
  a.kc_rows = g.kc_rows;
  a.n_rows = g.n_rows;
  a.ov_s = g.ov_s;
  a.ov_l = g.ov_l;
  a.b = g.b;
  a.s_end = g.s_end;
  a.w_begin = g.w_begin;
  a.top_k = p->top_k;
  a.scale = scale_of(p);
  a.lsa = p->pool == SA_POOL_LSA;
  // as many chunks per pair as keep every CTA resident (two per SM)
  const int64_t pairs = std::max<int64_t>(1, g.pairs);
  const int64_t passes = std::max<int64_t>(1, (g.n_rows + kScoreRowsPerPass - 1) / kScoreRowsPerPass);
  const int64_t want = std::min<int64_t>(passes, std::max<int64_t>(1, 2 * device_sms() / pairs));
  const int64_t per = (passes + want - 1) / want;
  a.rows_per_chunk = per * kScoreRowsPerPass;
  a.chunks = static_cast<int>((passes + per - 1) / per);
  if (g.ov_s > 0) {
    a.scores = caller_scores;
    a.cscores = a.chunks > 1 ? ws_scores : nullptr;
  } else {
    a.scores = caller_scores ? caller_scores : (a.chunks > 1 ? ws_scores : nullptr);
  }
  return a;
}

DecodeAttnArgs attn_args(const sa_params* p, const DecodeGeom& g, const DecodePlan& plan, const void* Q,
                         const void* K, const void* V, const int32_t* idx, int idx_stride, void* O, float* lse,
                         unsigned char* ws, const DecodeWs& L) {
  DecodeAttnArgs a = {};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.idx = idx;
  a.idx_stride = idx_stride;
  a.top_k = p->top_k;
  a.O = O;
  a.lse = lse;
  a.part_O = reinterpret_cast<float*>(ws + L.part_O);
  a.part_ml = reinterpret_cast<float*>(ws + L.part_ml);
  a.counters = reinterpret_cast<unsigned*>(ws + L.attn_cnt);
  a.status = reinterpret_cast<unsigned*>(ws);
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.G;
  a.n_q = g.n_q;
  a.R = g.R;
  a.R4 = plan.R4;
  a.C = g.C;
  a.cap = g.cap;
  a.kv_end = g.kv_end;
  a.b = g.b;
  a.nb = g.nb;
  a.s_end = g.s_end;
  a.w_begin = g.w_begin;
  a.tile = plan.tile;
  a.n_tiles = plan.n_tiles;
  a.n_sink_tiles = plan.n_sink_tiles;
  a.tpb = plan.tpb;
  a.n_wc_tiles = plan.n_wc_tiles;
  a.MT = plan.MT;
  a.total_tiles = plan.total_tiles;
  a.tpc = plan.tpc;
  a.n_slots = plan.n_slots;
  a.n_stages = plan.n_stages;
  a.qscale = scale_of(p) * 1.4426950408889634f;
  return a;
}

// ---- prefill -------------------------------------------------------------------
struct PrefillGeom {
  int B, Hq, Hkv, G, T, nb, n_tiles, P;
  int nc;          // compressed rows scored per pair (blocks, or windows touching a complete block)
  int kc_rows;     // rows per pair of the caller's Kc
  int ov_s, ov_l;  // overlapping windows, 0 otherwise
  int64_t cap;
};

// Shape limits of the tensor-core prefill path (besides check_params).
sa_status check_prefill(const sa_params* p, PrefillGeom* g) {
  if (p->dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "prefill runs on bf16 tensor cores: dtype must be SA_BF16");
  if ((p->num_q_heads / p->num_kv_heads) % 4 != 0)
    return fail(SA_ERR_UNSUPPORTED, "prefill is built for GQA groups of a multiple of 4 query heads per KV head");
  if (p->block_size != 64) return fail(SA_ERR_UNSUPPORTED, "prefill is built for block_size 64 (= query tile)");
  if (p->sink_keys % 64 != 0 || p->window_keys % 64 != 0)
    return fail(SA_ERR_UNSUPPORTED, "prefill needs sink_keys and window_keys to be multiples of 64");
  g->B = p->batch;
  g->Hq = p->num_q_heads;
  g->Hkv = p->num_kv_heads;
  g->G = p->num_q_heads / p->num_kv_heads;
  g->T = p->n_q;
  g->nb = p->n_q / 64;
  g->n_tiles = (p->n_q + 63) / 64;
  g->P = p->batch * p->num_kv_heads;
  g->cap = p->kv_capacity;
  g->nc = g->kc_rows = g->nb;
  g->ov_s = g->ov_l = 0;
  if (p->pool == SA_POOL_OVERLAP) {
    // windows starting at or past the last complete block's end touch no
    // complete block (s divides b)
    g->ov_s = p->pool_stride;
    g->ov_l = p->pool_kernel;
    g->kc_rows = g->T >= g->ov_l ? (g->T - g->ov_l) / g->ov_s + 1 : 0;
    g->nc = std::min(g->kc_rows, g->nb * (64 / g->ov_s));
  }
  if (g->nb > 6144) return fail(SA_ERR_UNSUPPORTED, "prefill is built for sequences up to 393216 tokens");
  if (static_cast<int64_t>(g->B) * g->T > 0x7fffffff) return fail(SA_ERR_UNSUPPORTED, "too many tokens");
  return SA_OK;
}

struct PrefillWs {
  size_t kc2, scores, idx, clean, total;
};

PrefillWs prefill_ws(const PrefillGeom& g, int top_k, int op, int idx_len) {
  PrefillWs w = {};
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  const size_t rows = static_cast<size_t>(g.P) * g.n_tiles;
  if (op == SA_OP_PREFILL || op == SA_OP_SCORE_TOPK) {
    w.kc2 = take(static_cast<size_t>(g.P) * g.nc * 512);
    w.scores = take(rows * g.nc * 4);
  }
  if (op == SA_OP_PREFILL) w.idx = take(rows * static_cast<size_t>(top_k) * 4);
  if (op == SA_OP_GIVEN_IDX) w.clean = take(rows * static_cast<size_t>(idx_len) * 4);
  w.total = off;
  return w;
}

PrefillArgs prefill_args(const sa_params* p, const PrefillGeom& g) {
  PrefillArgs a = {};
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.T = g.T;
  a.nb = g.nb;
  a.nc = g.nc;
  a.kc_rows = g.kc_rows;
  a.lsa = p->pool == SA_POOL_LSA;
  a.ov_s = g.ov_s;
  a.ov_l = g.ov_l;
  a.n_tiles = g.n_tiles;
  a.top_k = p->top_k;
  a.out_bf16 = p->out_dtype == SA_BF16;
  a.num_sms = device_sms();
  a.cap = g.cap;
  a.S = p->sink_keys;
  a.W = p->window_keys;
  a.scale = scale_of(p);
  return a;
}

// ---- LSA flat bucket retrieval ------------------------------------------------
struct BucketGeom {
  int stride, m, nbk, mcap;
  int64_t nblk;            // complete cluster blocks of the context
  int64_t rows_per_pair;   // bucket rows per pair: every cluster block the cache can hold
  int64_t n_bkt;           // buckets of the context's complete cluster blocks
};

// First-level winners of the bucket selection per pair.
int64_t bucket_cands(const sa_params* p, const BucketGeom& g) {
  const int64_t chunks = (g.n_bkt + kBucketChunk - 1) / kBucketChunk;
  return chunks * std::min(p->top_k, kBucketChunk);
}

sa_status check_bucket(const sa_params* p, BucketGeom* g) {
  sa_status st = check_params(p, false);
  if (st != SA_OK) return st;
  if (p->pool != SA_POOL_LSA) return fail(SA_ERR_INVALID, "bucket retrieval needs pool = SA_POOL_LSA");
  if (p->pool_stride != 1 && p->pool_stride != 2 && p->pool_stride != 4)
    return fail(SA_ERR_UNSUPPORTED, "pool_stride %d: bucket retrieval is built for pool keys of 1, 2 or 4 raw keys",
                p->pool_stride);
  g->stride = p->pool_stride;
  g->m = p->block_size / p->pool_stride;
  if (g->m > 128)
    return fail(SA_ERR_UNSUPPORTED, "a cluster block holds at most 128 pool keys (block_size / pool_stride = %d)",
                g->m);
  g->nbk = p->block_size / 8;
  g->mcap = 16 / p->pool_stride;
  g->nblk = p->ctx_len / p->block_size;
  g->rows_per_pair = (p->kv_capacity / p->block_size) * g->nbk;
  g->n_bkt = g->nblk * g->nbk;
  if (p->kv_capacity / p->pool_stride >= (int64_t(1) << 31))
    return fail(SA_ERR_UNSUPPORTED, "pool-key ids of a %lld-row cache do not fit 32 bits", (long long)p->kv_capacity);
  if (g->rows_per_pair > (int64_t(1) << 26))
    return fail(SA_ERR_UNSUPPORTED, "%lld buckets per sequence exceed the 2^26 built", (long long)g->rows_per_pair);
  if (static_cast<int64_t>(p->top_k) * g->mcap > 4096)
    return fail(SA_ERR_UNSUPPORTED, "top_k x %d members = %d entries exceed the 4096 the expansion sorts", g->mcap,
                p->top_k * g->mcap);
  if (static_cast<int64_t>(p->batch) * p->num_kv_heads > 65535)
    return fail(SA_ERR_UNSUPPORTED, "more than 65535 (sequence, KV head) pairs");
  if (bucket_cands(p, *g) > kBucketMaxCand)
    return fail(SA_ERR_UNSUPPORTED,
                "%lld buckets with top_k %d: the selection's %lld first-level winners per sequence exceed %d",
                (long long)g->n_bkt, p->top_k, (long long)bucket_cands(p, *g), kBucketMaxCand);
  return SA_OK;
}

struct BucketWs {
  DecodeWs attn;
  size_t keys, cand_key, cand_id, sel, own, kept, total;
};

// Attention plan of the run mode: the selected section holds kept_cap runs,
// tile / stride of them per tile.
sa_status bucket_plan(const sa_params* p, const BucketGeom& bg, int kept_cap, DecodeGeom* g, DecodePlan* plan) {
  *g = decode_geom(p);
  const int T = p->dtype == SA_BF16 ? 64 : 32;
  g->b = T;
  const int rpt = T / bg.stride;
  const int n_sel = (kept_cap + rpt - 1) / rpt;
  const char* why = "";
  if (!plan_decode(*g, n_sel, p->dtype == SA_BF16, device_sms(), plan, &why))
    return fail(SA_ERR_UNSUPPORTED, "%s", why);
  return SA_OK;
}

BucketWs bucket_ws(const sa_params* p, const BucketGeom& bg, const DecodeGeom& g, const DecodePlan& plan) {
  BucketWs w;
  w.attn = decode_ws(g, plan, 0, SA_OP_GIVEN_IDX, 0);
  const size_t pairs = static_cast<size_t>(g.pairs);
  const size_t n_ent = static_cast<size_t>(p->top_k) * bg.mcap;
  const size_t nc = static_cast<size_t>(bucket_cands(p, bg));
  w.keys = align_up(w.attn.total, 256);
  w.cand_key = align_up(w.keys + pairs * static_cast<size_t>(bg.n_bkt) * 4, 256);
  w.cand_id = align_up(w.cand_key + pairs * nc * 4, 256);
  w.sel = align_up(w.cand_id + pairs * nc * 4, 256);
  w.own = align_up(w.sel + pairs * static_cast<size_t>(p->top_k) * 4, 256);
  w.kept = align_up(w.own + pairs * n_ent * 8, 256);
  w.total = align_up(w.kept + pairs * n_ent * 4, 256);
  return w;
}

// Workspace for any bucket_keys: the largest over the run counts the kept
// table can have.
size_t bucket_ws_bytes(const sa_params* p, const BucketGeom& bg) {
  const int n_ent = p->top_k * bg.mcap;
  const int rpt = (p->dtype == SA_BF16 ? 64 : 32) / bg.stride;
  size_t best = 0;
  for (int kc = 0;; kc += rpt) {
    const int cap = kc < n_ent ? kc : n_ent;
    DecodeGeom g;
    DecodePlan plan;
    if (bucket_plan(p, bg, cap, &g, &plan) != SA_OK) return 0;
    best = std::max(best, bucket_ws(p, bg, g, plan).total);
    if (cap >= n_ent) break;
  }
  return best;
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" {

int32_t sa_version(void) { return 103; }

const char* sa_last_error(void) { return g_err; }

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID: return "SA_ERR_INVALID";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_INDEX: return "SA_ERR_INDEX";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
  }
  return "SA_ERR_UNKNOWN";
}

// ---- dense verify -----------------------------------------------------------
// The dense pass is the decode attention with the whole context as its window
// and no table: every token sees keys 0..C+j.
sa_params verify_dense_params(const sa_params* p) {
  sa_params d = *p;
  d.sink_keys = 0;
  d.window_keys = p->ctx_len;
  d.top_k = 0;
  d.flags = SA_FLAG_TRUSTED_IDX;
  return d;
}

struct VerifyWs {
  DecodeWs attn;          // the dense attention's workspace (status, tickets, partials)
  size_t lse;             // lse of the rows when the caller passes none
  size_t part;            // [pairs, nb * b / 32, 16] float2 half-tile row sums
  size_t total;
};

// nb: complete blocks of the caller's context
VerifyWs verify_ws(const DecodeGeom& g, const DecodePlan& plan, int64_t nb) {
  VerifyWs w;
  w.attn = decode_ws(g, plan, 0, SA_OP_GIVEN_IDX, 0);
  w.lse = align_up(w.attn.total, 256);
  w.part = align_up(w.lse + static_cast<size_t>(g.B) * g.n_q * g.Hq * 4, 256);
  w.total = w.part + static_cast<size_t>(g.pairs) * static_cast<size_t>(nb * g.b / 32) * 16 * 8;
  return w;
}

// ---- column-sparse attention ------------------------------------------------
sa_status check_column(const sa_params* p, PrefillGeom* g) {
  if (p->dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "column attention runs on bf16 tensor cores");
  if ((p->num_q_heads / p->num_kv_heads) % 4 != 0)
    return fail(SA_ERR_UNSUPPORTED, "column attention is built for GQA groups of a multiple of 4 query heads per KV head");
  if (p->block_size != 64) return fail(SA_ERR_UNSUPPORTED, "column attention groups 64 query tokens: block_size 64");
  g->B = p->batch;
  g->Hq = p->num_q_heads;
  g->Hkv = p->num_kv_heads;
  g->G = p->num_q_heads / p->num_kv_heads;
  g->T = p->n_q;
  g->nb = p->n_q / 64;
  g->n_tiles = (p->n_q + 63) / 64;
  g->P = p->batch * p->num_kv_heads;
  g->cap = p->kv_capacity;
  if (static_cast<int64_t>(g->B) * g->T > 0x7fffffff) return fail(SA_ERR_UNSUPPORTED, "too many tokens");
  return SA_OK;
}

size_t column_ws(const PrefillGeom& g, int n_cols) {
  return align_up(kWsHeader, 1024) + static_cast<size_t>(g.P) * g.n_tiles * static_cast<size_t>(n_cols) * 4;
}

size_t sa_workspace_size(const sa_params* p, int32_t op) {
  if (op == SA_OP_COLUMN) {
    // top_k is the column count here (checked against its own limit)
    if (!p || p->top_k < 0 || p->top_k > (1 << 20)) return 0;
    sa_params q = *p;
    q.top_k = 0;
    if (check_params(&q, true) != SA_OK) return 0;
    PrefillGeom g;
    if (check_column(&q, &g) != SA_OK) return 0;
    return column_ws(g, p->top_k);
  }
  if (op == SA_OP_VERIFY) {
    if (check_params(p, false) != SA_OK) return 0;
    const sa_params d = verify_dense_params(p);
    DecodeGeom g;
    DecodePlan plan;
    if (plan_for(&d, 0, &g, &plan) != SA_OK) return 0;
    return verify_ws(g, plan, decode_geom(p).nb).total;
  }
  if (op == SA_OP_BUCKET_DECODE) {
    BucketGeom bg;
    if (check_bucket(p, &bg) != SA_OK) return 0;
    return bucket_ws_bytes(p, bg);
  }
  const bool prefill = (op == SA_OP_PREFILL) || (p && p->select == SA_SEL_TILE_MAX);
  if (check_params(p, prefill) != SA_OK) return 0;
  if (prefill) {
    PrefillGeom g;
    if (check_prefill(p, &g) != SA_OK) return 0;
    return prefill_ws(g, p->top_k, op, p->top_k).total;
  }
  DecodeGeom g;
  DecodePlan plan;
  int slots = (op == SA_OP_DECODE) ? p->top_k : 0;
  if (op == SA_OP_GIVEN_IDX) slots = p->top_k;   // sized for idx_len == top_k
  if (op == SA_OP_SCORE_TOPK) slots = 0;
  if (plan_for(p, slots, &g, &plan) != SA_OK) return 0;
  return decode_ws(g, plan, p->top_k, op, p->top_k).total;
}

sa_status sa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return fail(SA_ERR_INVALID, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return SA_OK;
}

sa_status sa_append_kv(const sa_params* p, const void* K_new, const void* V_new, void* K, void* V, void* stream) {
  sa_status st = check_params(p, false);
  if (st != SA_OK) return st;
  if (!K_new || !V_new || !K || !V) return fail(SA_ERR_INVALID, "K_new, V_new, K and V must be non-NULL");
  if (!aligned16(K_new) || !aligned16(V_new) || !aligned16(K) || !aligned16(V))
    return fail(SA_ERR_INVALID, "K_new, V_new, K and V must be 16-byte aligned");
  const int row_bytes = p->head_dim * (p->dtype == SA_BF16 ? 2 : 4);
  cudaError_t e = launch_append_kv(K_new, V_new, K, V, p->batch * p->num_kv_heads, p->n_q, p->kv_capacity,
                                   p->ctx_len, row_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  return SA_OK;
}

sa_status sa_pool_keys(const sa_params* p, const void* K, float* Kc, void* stream) {
  const bool prefill = p && p->select == SA_SEL_TILE_MAX;
  sa_status st = check_params(p, prefill);
  if (st != SA_OK) return st;
  const int64_t keys = prefill ? static_cast<int64_t>(p->n_q) : p->ctx_len;
  const bool ovl = p->pool == SA_POOL_OVERLAP;
  const int64_t rows = ovl ? (keys >= p->pool_kernel ? (keys - p->pool_kernel) / p->pool_stride + 1 : 0)
                           : keys / p->block_size;
  if (rows == 0) return SA_OK;   // no complete block / window: nothing to write
  if (!K || !Kc) return fail(SA_ERR_INVALID, "K and Kc must be non-NULL");
  if (!aligned16(K) || !aligned16(Kc)) return fail(SA_ERR_INVALID, "K and Kc must be 16-byte aligned");
  PoolArgs a = {};
  a.K = K;
  a.Kc = Kc;
  a.pairs = p->batch * p->num_kv_heads;
  a.cap = p->kv_capacity;
  a.nb = rows;
  a.stride = ovl ? p->pool_stride : p->block_size;
  a.len = ovl ? p->pool_kernel : p->block_size;
  a.lsa = p->pool == SA_POOL_LSA;
  cudaError_t e = launch_pool(a, p->dtype == SA_BF16, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pool kernel launch");
  return SA_OK;
}

sa_status sa_score_topk(const sa_params* p, const void* Q, const float* Kc, int32_t* idx, float* scores, void* ws,
                        size_t ws_bytes, void* stream) {
  const bool prefill = p && p->select == SA_SEL_TILE_MAX;
  sa_status st = check_params(p, prefill);
  if (st != SA_OK) return st;
  if (prefill) {
    PrefillGeom g;
    if ((st = check_prefill(p, &g)) != SA_OK) return st;
    if (!Q || (!Kc && g.nb > 0) || (!idx && p->top_k > 0)) return fail(SA_ERR_INVALID, "Q, Kc and idx must be non-NULL");
    if (!aligned16(Q) || !aligned16(Kc)) return fail(SA_ERR_INVALID, "Q and Kc must be 16-byte aligned");
    const PrefillWs L = prefill_ws(g, p->top_k, SA_OP_SCORE_TOPK, 0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
    unsigned char* w = static_cast<unsigned char*>(ws);
    PrefillArgs a = prefill_args(p, g);
    a.Q = Q;
    a.Kc = Kc;
    a.kc2 = reinterpret_cast<uint16_t*>(w + L.kc2);
    // per-block scores go straight to the caller's buffer; window scores
    // stay in the workspace and the caller gets the block scores
    if (g.ov_s > 0) {
      a.scores = reinterpret_cast<float*>(w + L.scores);
      a.bscores = scores;
    } else {
      a.scores = scores ? scores : reinterpret_cast<float*>(w + L.scores);
    }
    a.idx = idx;
    a.status = reinterpret_cast<unsigned*>(w);
    cudaError_t e = launch_prefill_score(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "prefill scoring launch");
    return SA_OK;
  }
  if (!Q || (!Kc && p->ctx_len >= p->block_size) || (!idx && p->top_k > 0))
    return fail(SA_ERR_INVALID, "Q, Kc and idx must be non-NULL (Kc may be NULL without a complete block)");
  if (!aligned16(Q) || !aligned16(Kc)) return fail(SA_ERR_INVALID, "Q and Kc must be 16-byte aligned");
  DecodeGeom g;
  DecodePlan plan;
  if ((st = plan_for(p, 0, &g, &plan)) != SA_OK) return st;
  if (g.nb > kMaxSelectBlocks)
    return fail(SA_ERR_UNSUPPORTED, "%lld blocks per sequence exceed the %lld the selector handles",
                (long long)g.nb, (long long)kMaxSelectBlocks);
  const DecodeWs L = decode_ws(g, plan, p->top_k, SA_OP_SCORE_TOPK);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  ScoreArgs a = score_args(p, g, Q, Kc, scores, idx, w, L);
  cudaError_t e = launch_score_topk_query0(a, p->dtype == SA_BF16, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "score/top-k kernel launch");
  return SA_OK;
}

sa_status sa_sparse_attn_given_idx(const sa_params* p, const void* Q, const void* K, const void* V,
                                   const int32_t* idx, int32_t idx_len, void* O, float* lse, void* ws,
                                   size_t ws_bytes, void* stream) {
  const bool prefill = p && p->select == SA_SEL_TILE_MAX;
  sa_status st = check_params(p, prefill);
  if (st != SA_OK) return st;
  if (!Q || !K || !V || !O) return fail(SA_ERR_INVALID, "Q, K, V and O must be non-NULL");
  if (idx_len < 0 || idx_len > 4096) return fail(SA_ERR_INVALID, "idx_len %d must be in [0, 4096]", idx_len);
  if (idx_len > 0 && !idx) return fail(SA_ERR_INVALID, "idx is NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(SA_ERR_INVALID, "Q, K, V and O must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (prefill) {
    PrefillGeom g;
    if ((st = check_prefill(p, &g)) != SA_OK) return st;
    const PrefillWs L = prefill_ws(g, p->top_k, SA_OP_GIVEN_IDX, idx_len);
    if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
    unsigned char* w = static_cast<unsigned char*>(ws);
    const int32_t* table = idx;
    if (!(p->flags & SA_FLAG_TRUSTED_IDX)) {
      int32_t* clean = reinterpret_cast<int32_t*>(w + L.clean);
      cudaError_t e = launch_sanitize_prefill_idx(idx, clean, g.P, g.n_tiles, idx_len, p->sink_keys, p->window_keys,
                                                  reinterpret_cast<unsigned*>(w), s);
      if (e != cudaSuccess) return cuda_fail(e, "index-table check launch");
      table = clean;
    }
    PrefillArgs a = prefill_args(p, g);
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.idx = const_cast<int32_t*>(table);
    a.top_k = idx_len;
    a.O = O;
    a.lse = lse;
    a.status = reinterpret_cast<unsigned*>(w);
    cudaError_t e = launch_prefill_attn(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
    return SA_OK;
  }
  DecodeGeom g;
  DecodePlan plan;
  if ((st = plan_for(p, idx_len, &g, &plan)) != SA_OK) return st;
  const DecodeWs L = decode_ws(g, plan, p->top_k, SA_OP_GIVEN_IDX, idx_len);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  const int32_t* table = idx;
  cudaError_t e = cudaSuccess;
  if (!(p->flags & SA_FLAG_TRUSTED_IDX)) {
    int32_t* clean = reinterpret_cast<int32_t*>(w + L.clean_idx);
    e = launch_sanitize_idx(idx, clean, g.pairs, idx_len, g.nb, reinterpret_cast<unsigned*>(w), s);
    if (e != cudaSuccess) return cuda_fail(e, "index-table check launch");
    table = clean;
  }
  DecodeAttnArgs a = attn_args(p, g, plan, Q, K, V, table, idx_len, O, lse, w, L);
  a.pdl = 0;
  e = launch_decode_attn(a, plan, p->dtype == SA_BF16, p->out_dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SA_OK;
}

sa_status sa_sparse_attn_decode(const sa_params* p, const void* Q, const void* K, const void* V, const float* Kc,
                                void* O, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  sa_status st = check_params(p, false);
  if (st != SA_OK) return st;
  if (!Q || !K || !V || !O || (!Kc && p->ctx_len >= p->block_size))
    return fail(SA_ERR_INVALID, "Q, K, V, Kc and O must be non-NULL (Kc may be NULL without a complete block)");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(Kc))
    return fail(SA_ERR_INVALID, "Q, K, V, Kc and O must be 16-byte aligned");
  DecodeGeom g;
  DecodePlan plan;
  if ((st = plan_for(p, p->top_k, &g, &plan)) != SA_OK) return st;
  if (g.nb > kMaxSelectBlocks)
    return fail(SA_ERR_UNSUPPORTED, "%lld blocks per sequence exceed the %lld the selector handles",
                (long long)g.nb, (long long)kMaxSelectBlocks);
  const DecodeWs L = decode_ws(g, plan, p->top_k, SA_OP_DECODE);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + L.idx);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->dtype == SA_BF16 && g.nb >= 1) {
    // one cooperative launch: scores, top-k and attention
    DecodeAttnArgs a = attn_args(p, g, plan, Q, K, V, idx, p->top_k, O, lse, w, L);
    if (p->pool != SA_POOL_OVERLAP && decode_fused_supported(a, plan, g.nb)) {
      a.Kc = Kc;
      a.scores = reinterpret_cast<float*>(w + L.scores);
      a.score_cnt = reinterpret_cast<unsigned*>(w + L.score_cnt);
      a.ready = reinterpret_cast<unsigned*>(w + L.ready);
      a.exit_cnt = reinterpret_cast<unsigned*>(w + L.exit_cnt);
      a.cand = reinterpret_cast<uint2*>(w + L.cand);
      a.idx_w = idx;
      a.top_k = p->top_k;
      a.sscale = scale_of(p);
      a.lsa = p->pool == SA_POOL_LSA;
      cudaError_t e = launch_decode_fused(a, plan, p->out_dtype == SA_BF16, s);
      if (e == cudaSuccess) return SA_OK;
      // a cooperative grid that cannot be resident at once (e.g. SMs taken by
      // other work) is refused at launch: take the two-kernel path
      if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail(e, "fused decode launch");
      (void)cudaGetLastError();
    }
  }
  ScoreArgs sa_ = score_args(p, g, Q, Kc, nullptr, idx, w, L);
  cudaError_t e = launch_score_topk_query0(sa_, p->dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "score/top-k kernel launch");
  DecodeAttnArgs a = attn_args(p, g, plan, Q, K, V, idx, p->top_k, O, lse, w, L);
  a.pdl = 1;
  e = launch_decode_attn(a, plan, p->dtype == SA_BF16, p->out_dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SA_OK;
}

sa_status sa_verify_refresh(const sa_params* p, const void* Q, const void* K, const void* V, void* O, float* lse,
                            float* mass, int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  sa_status st = check_params(p, false);
  if (st != SA_OK) return st;
  if (!Q || !K || !V || !O || !mass) return fail(SA_ERR_INVALID, "Q, K, V, O and mass must be non-NULL");
  if (p->top_k > 0 && !idx_out) return fail(SA_ERR_INVALID, "idx_out is NULL with top_k > 0");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(SA_ERR_INVALID, "Q, K, V and O must be 16-byte aligned");
  if (p->dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "verify runs on bf16 tensor cores: dtype must be SA_BF16");
  if (p->block_size % 64 != 0) return fail(SA_ERR_UNSUPPORTED, "verify block mass needs block_size a multiple of 64");
  const sa_params d = verify_dense_params(p);
  DecodeGeom g;
  DecodePlan plan;
  if ((st = plan_for(&d, 0, &g, &plan)) != SA_OK) return st;
  const DecodeGeom gs = decode_geom(p);          // the caller's sink and window: the candidates
  if (gs.nb > kMaxSelectBlocks)
    return fail(SA_ERR_UNSUPPORTED, "%lld blocks per sequence exceed the %lld the selector handles",
                (long long)gs.nb, (long long)kMaxSelectBlocks);
  if (g.R > 16) return fail(SA_ERR_UNSUPPORTED, "verify needs n_q * G <= 16 rows per KV head");
  const VerifyWs L = verify_ws(g, plan, gs.nb);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* lse_rows = lse ? lse : reinterpret_cast<float*>(w + L.lse);
  float2* part = reinterpret_cast<float2*>(w + L.part);

  // 1. dense attention (O, lse) with the half-tile row sums of the complete
  //    blocks (tensor-core kernel only)
  DecodeAttnArgs a = attn_args(&d, g, plan, Q, K, V, nullptr, 0, O, lse_rows, w, L.attn);
  a.pdl = 0;
  a.mass_part = part;
  a.mass_keys = gs.nb * g.b;
  a.mass_hts = static_cast<int>(a.mass_keys / 32);
  if (!decode_tc_supported(a)) return fail(SA_ERR_UNSUPPORTED, "verify needs the tensor-core attention kernel");
  cudaError_t e = launch_decode_tc(a, plan, p->out_dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "dense attention launch");
  // 2. block masses
  e = launch_mass_finalize(part, lse_rows, mass, g.B, g.Hkv, g.G, g.n_q, static_cast<int>(gs.nb), g.b, s);
  if (e != cudaSuccess) return cuda_fail(e, "block mass launch");
  // 3. the refreshed selection: top-k candidates by mass
  if (p->top_k > 0) {
    e = launch_mass_topk(mass, g.pairs, static_cast<int>(gs.nb), g.b, gs.s_end, gs.w_begin, p->top_k, idx_out, s);
    if (e != cudaSuccess) return cuda_fail(e, "mass top-k launch");
  }
  return SA_OK;
}

sa_status sa_column_attn(const sa_params* p0, const void* Q, const void* K, const void* V, const int32_t* cols,
                         int32_t n_cols, void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!p0) return fail(SA_ERR_INVALID, "params is NULL");
  sa_params pc = *p0;
  pc.top_k = 0;                               // not used by this call
  const sa_params* p = &pc;
  sa_status st = check_params(p, true);
  if (st != SA_OK) return st;
  if (!Q || !K || !V || !O) return fail(SA_ERR_INVALID, "Q, K, V and O must be non-NULL");
  if (n_cols < 0 || n_cols > (1 << 20)) return fail(SA_ERR_INVALID, "n_cols %d must be in [0, 2^20]", n_cols);
  if (n_cols > 0 && !cols) return fail(SA_ERR_INVALID, "cols is NULL with n_cols > 0");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(SA_ERR_INVALID, "Q, K, V and O must be 16-byte aligned");
  PrefillGeom g;
  if ((st = check_column(p, &g)) != SA_OK) return st;
  const size_t need = column_ws(g, n_cols);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t* table = cols;
  if (n_cols > 0 && !(p->flags & SA_FLAG_TRUSTED_IDX)) {
    int32_t* clean = reinterpret_cast<int32_t*>(w + align_up(kWsHeader, 1024));
    cudaError_t e = launch_sanitize_cols(cols, clean, static_cast<int64_t>(g.P) * g.n_tiles, n_cols, g.T,
                                         reinterpret_cast<unsigned*>(w), s);
    if (e != cudaSuccess) return cuda_fail(e, "column-table check launch");
    table = clean;
  }
  PrefillArgs a = prefill_args(p, g);
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.idx = const_cast<int32_t*>(table);
  a.top_k = n_cols;
  a.O = O;
  a.lse = lse;
  a.status = reinterpret_cast<unsigned*>(w);
  cudaError_t e = launch_column_attn(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "column attention launch");
  return SA_OK;
}

int32_t sa_decode_launches(const sa_params* p) {
  if (check_params(p, false) != SA_OK) return 0;
  DecodeGeom g;
  DecodePlan plan;
  if (plan_for(p, p->top_k, &g, &plan) != SA_OK) return 0;
  if (p->dtype == SA_BF16 && g.nb >= 1) {
    const DecodeWs L = decode_ws(g, plan, p->top_k, SA_OP_DECODE);
    DecodeAttnArgs a = attn_args(p, g, plan, nullptr, nullptr, nullptr, nullptr, p->top_k, nullptr, nullptr,
                                 nullptr, L);
    if (p->pool != SA_POOL_OVERLAP && decode_fused_supported(a, plan, g.nb)) return 1;
  }
  return 2;
}

sa_status sa_sparse_attn_prefill(const sa_params* p, const void* Q, const void* K, const void* V, float* Kc,
                                 void* O, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  sa_status st = check_params(p, true);
  if (st != SA_OK) return st;
  PrefillGeom g;
  if ((st = check_prefill(p, &g)) != SA_OK) return st;
  if (!Q || !K || !V || !O || (!Kc && g.nb > 0)) return fail(SA_ERR_INVALID, "Q, K, V, Kc and O must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(Kc))
    return fail(SA_ERR_INVALID, "Q, K, V, Kc and O must be 16-byte aligned");
  const PrefillWs L = prefill_ws(g, p->top_k, SA_OP_PREFILL, 0);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = sa_pool_keys(p, K, Kc, stream)) != SA_OK) return st;
  PrefillArgs a = prefill_args(p, g);
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.Kc = Kc;
  a.kc2 = reinterpret_cast<uint16_t*>(w + L.kc2);
  a.scores = reinterpret_cast<float*>(w + L.scores);
  a.idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + L.idx);
  a.O = O;
  a.lse = lse;
  a.status = reinterpret_cast<unsigned*>(w);
  cudaError_t e = launch_prefill_score(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill scoring launch");
  e = launch_prefill_attn(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
  return SA_OK;

}

sa_status sa_read_status(void* ws, void* stream) {
  if (!ws) return fail(SA_ERR_INVALID, "workspace is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (status word)");
  if (word) {
    e = cudaMemset(ws, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset (status word)");
  }
  if (word & kStatusTimeout) return fail(SA_ERR_TIMEOUT, "a bounded wait inside a kernel ran out");
  if (word & kStatusIndex) return fail(SA_ERR_INDEX, "an index-table entry was out of range or repeated");
  return SA_OK;
}

}  // extern "C"

// ---- LSA flat bucket retrieval (LSA review §2.2-2.3) --------------------------
extern "C" sa_status sa_bucket_build(const sa_params* p, const void* K, int64_t first_block, float* centroids,
                                     int32_t* members, void* stream) {
  BucketGeom bg;
  sa_status st = check_bucket(p, &bg);
  if (st != SA_OK) return st;
  if (first_block < 0 || first_block > bg.nblk)
    return fail(SA_ERR_INVALID, "first_block %lld must be in [0, %lld]", (long long)first_block, (long long)bg.nblk);
  if (first_block == bg.nblk) return SA_OK;
  if (!K || !centroids || !members) return fail(SA_ERR_INVALID, "K, centroids and members must be non-NULL");
  if (!aligned16(K) || !aligned16(centroids) || !aligned16(members))
    return fail(SA_ERR_INVALID, "K, centroids and members must be 16-byte aligned");
  WardArgs a = {};
  a.K = K;
  a.cents = centroids;
  a.members = members;
  a.cap = p->kv_capacity;
  a.rows_per_pair = bg.rows_per_pair;
  a.first_block = first_block;
  a.b = p->block_size;
  a.stride = bg.stride;
  a.m = bg.m;
  a.nbk = bg.nbk;
  a.mcap = bg.mcap;
  cudaError_t e = launch_ward(a, p->batch * p->num_kv_heads, bg.nblk - first_block, p->dtype == SA_BF16,
                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bucket clustering launch");
  return SA_OK;
}

extern "C" sa_status sa_bucket_decode(const sa_params* p, const void* Q, const void* K, const void* V,
                                      const float* centroids, const int32_t* members, int32_t bucket_keys, void* O,
                                      float* lse, int32_t* sel_out, int32_t* kept_out, void* ws, size_t ws_bytes,
                                      void* stream) {
  BucketGeom bg;
  sa_status st = check_bucket(p, &bg);
  if (st != SA_OK) return st;
  if (bucket_keys < 0 || bucket_keys % bg.stride != 0)
    return fail(SA_ERR_INVALID, "bucket_keys %d must be >= 0 and a multiple of pool_stride %d", bucket_keys,
                bg.stride);
  const bool retrieve = p->top_k > 0 && bg.n_bkt > 0;
  if (!Q || !K || !V || !O || (retrieve && (!centroids || !members)))
    return fail(SA_ERR_INVALID, "Q, K, V, O (and centroids, members with buckets to score) must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(centroids) ||
      !aligned16(members))
    return fail(SA_ERR_INVALID, "Q, K, V, O, centroids and members must be 16-byte aligned");
  const int n_ent = p->top_k * bg.mcap;
  const int keep_pool = bucket_keys / bg.stride;
  const int kept_cap = keep_pool > 0 ? std::min(keep_pool, n_ent) : n_ent;
  DecodeGeom g;
  DecodePlan plan;
  if ((st = bucket_plan(p, bg, kept_cap, &g, &plan)) != SA_OK) return st;
  const BucketWs L = bucket_ws(p, bg, g, plan);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SA_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = p->dtype == SA_BF16;
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w + L.sel);
  int32_t* kept = kept_out ? kept_out : reinterpret_cast<int32_t*>(w + L.kept);
  BucketScoreArgs sc = {};
  sc.Q = Q;
  sc.cents = centroids;
  sc.members = members;
  sc.keys = reinterpret_cast<uint32_t*>(w + L.keys);
  sc.cand_key = reinterpret_cast<uint32_t*>(w + L.cand_key);
  sc.cand_id = reinterpret_cast<int32_t*>(w + L.cand_id);
  sc.Hq = p->num_q_heads;
  sc.Hkv = p->num_kv_heads;
  sc.G = p->num_q_heads / p->num_kv_heads;
  sc.n_q = p->n_q;
  sc.rows_per_pair = bg.rows_per_pair;
  sc.n_bkt = retrieve ? bg.n_bkt : 0;
  sc.nbk = bg.nbk;
  sc.b = p->block_size;
  sc.stride = bg.stride;
  sc.mcap = bg.mcap;
  sc.s_end = g.s_end;
  sc.w_begin = g.w_begin;
  sc.rows_per_cta = 2048;
  BucketExpandArgs ex = {};
  ex.Q = Q;
  ex.K = K;
  ex.members = members;
  ex.sel = sel;
  ex.own = reinterpret_cast<unsigned long long*>(w + L.own);
  ex.kept = kept;
  ex.Hq = sc.Hq;
  ex.Hkv = sc.Hkv;
  ex.G = sc.G;
  ex.n_q = sc.n_q;
  ex.cap = p->kv_capacity;
  ex.rows_per_pair = bg.rows_per_pair;
  ex.top_k = retrieve ? p->top_k : 0;
  ex.mcap = bg.mcap;
  ex.stride = bg.stride;
  ex.keep_pool = keep_pool;
  ex.kept_cap = kept_cap;
  const int pairs = g.pairs;
  cudaError_t e = cudaSuccess;
  if (retrieve) {
    e = launch_bucket_select(sc, ex, pairs, bf16, s);
    if (e != cudaSuccess) return cuda_fail(e, "bucket scoring launch");
  } else if (sel_out && p->top_k > 0) {
    e = cudaMemsetAsync(sel_out, 0xff, static_cast<size_t>(pairs) * p->top_k * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  }
  if (kept_cap > 0) {
    if (retrieve) {
      e = launch_bucket_expand(ex, pairs, bf16, s);
      if (e != cudaSuccess) return cuda_fail(e, "bucket expansion launch");
    } else {
      e = cudaMemsetAsync(kept, 0xff, static_cast<size_t>(pairs) * kept_cap * 4, s);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    }
  }
  const int rpt = (bf16 ? 64 : 32) / bg.stride;
  DecodeAttnArgs a = attn_args(p, g, plan, Q, K, V, kept, (kept_cap + rpt - 1) / rpt, O, lse, w, L.attn);
  a.pdl = 0;
  a.runs = kept;
  a.runs_stride = kept_cap;
  a.run_len = bg.stride;
  e = launch_decode_attn(a, plan, bf16, p->out_dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SA_OK;
}

// ---- allocation-free variant of sa_sparse_attn_given_idx --------------------
// For callers that cannot call cudaMalloc themselves: code running inside a
// host framework whose allocator must not be re-entered, plug-ins handed only
// input and output buffers, or callers whose memory budget was fixed before
// they run.  The attention kernel's scratch (status word, per-pair tickets,
// split partials) lives in one file-scope device array instead of a
// caller-provided workspace.
#include <mutex>

namespace sa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB per device, held until exit

// In host code this name is only a host-side stand-in for the device array,
// not a device address: the address is obtained once per device with
// cudaGetSymbolAddress and passed to the kernel.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[64] = {nullptr};

// Device address of g_static_scratch on the current device (set-up on the
// first call per device, with that device current).
sa_status static_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device ordinal %d: at most 64 devices", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_static_ptr[dev]);
  return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_sparse_attn_given_idx_noalloc(const sa_params* p, const void* Q, const void* K,
                                                      const void* V, const int32_t* idx, int32_t idx_len,
                                                      void* O, float* lse, void* stream) {
  const bool prefill = p && p->select == SA_SEL_TILE_MAX;
  sa_status st = check_params(p, prefill);
  if (st != SA_OK) return st;
  if (prefill)
    return fail(SA_ERR_UNSUPPORTED,
                "the allocation-free entry point takes decode and draft-chunk index tables (SA_SEL_QUERY0) only; "
                "pass prefill tables (SA_SEL_TILE_MAX) to sa_sparse_attn_given_idx with a workspace");
  if (!Q || !K || !V || !O) return fail(SA_ERR_INVALID, "Q, K, V and O must be non-NULL");
  if (idx_len < 0 || idx_len > 4096) return fail(SA_ERR_INVALID, "idx_len %d must be in [0, 4096]", idx_len);
  if (idx_len > 0 && !idx) return fail(SA_ERR_INVALID, "idx is NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(SA_ERR_INVALID, "Q, K, V and O must be 16-byte aligned");
  DecodeGeom g;
  DecodePlan plan;
  if ((st = plan_for(p, idx_len, &g, &plan)) != SA_OK) return st;
  const DecodeWs L = decode_ws(g, plan, p->top_k, SA_OP_GIVEN_IDX, idx_len);
  if (L.total > kStaticScratchBytes)
    return fail(SA_ERR_WORKSPACE,
                "this problem needs %zu bytes of scratch; the allocation-free entry point has a static "
                "array of %zu bytes (use sa_sparse_attn_given_idx with a workspace)",
                L.total, kStaticScratchBytes);
  unsigned char* w = nullptr;
  if ((st = static_scratch(&w)) != SA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the status word and the
  // tickets must start at zero.
  cudaError_t e = cudaMemsetAsync(w, 0, L.clean_idx, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (static scratch)");
  const int32_t* table = idx;
  if (!(p->flags & SA_FLAG_TRUSTED_IDX)) {
    int32_t* clean = reinterpret_cast<int32_t*>(w + L.clean_idx);
    e = launch_sanitize_idx(idx, clean, g.pairs, idx_len, g.nb, reinterpret_cast<unsigned*>(w), s);
    if (e != cudaSuccess) return cuda_fail(e, "index-table check launch");
    table = clean;
  }
  DecodeAttnArgs a = attn_args(p, g, plan, Q, K, V, table, idx_len, O, lse, w, L);
  a.pdl = 0;
  e = launch_decode_attn(a, plan, p->dtype == SA_BF16, p->out_dtype == SA_BF16, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SA_OK;
}
