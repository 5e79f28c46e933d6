// Host-side interface between the C ABI layer (sa_api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

// Geometry of one decode / chunk problem, derived from sa_params on the host.
struct DecodeGeom {
  int B, Hq, Hkv, G, n_q, R;       // R = n_q * G query rows per (sequence, KV head)
  int64_t C, cap, kv_end;          // context length, token stride, C + n_q
  int b;                           // block size
  int64_t nb;                      // complete blocks of the context
  int64_t kc_rows;                 // rows of Kc per pair (nb, or the windows of SA_POOL_OVERLAP)
  int64_t n_rows;                  // rows of Kc that scoring reads (the windows touching a complete block)
  int ov_s, ov_l;                  // SA_POOL_OVERLAP window stride and length (0 otherwise)
  int64_t s_end, w_begin;          // sink [0, s_end), window [w_begin, C)
  int pairs;                       // B * Hkv
};

// ---- pooling ----------------------------------------------------------------
// Row j of a pair's Kc compresses keys [j * stride, j * stride + len).
struct PoolArgs {
  const void* K;
  float* Kc;
  int pairs;
  int64_t cap;      // token stride of K
  int64_t nb;       // rows of Kc per pair
  int64_t stride;   // keys between row starts (b, or s of SA_POOL_OVERLAP)
  int len;          // keys per row (b, or l of SA_POOL_OVERLAP)
  int lsa;          // 0 mean, 1 LSA centroid (len == stride)
};
cudaError_t launch_pool(const PoolArgs& a, bool bf16, cudaStream_t s);

// ---- decode scoring + top-k --------------------------------------------------
// SA_POOL_OVERLAP (ov_s > 0): the rows are windows of ov_l keys every ov_s
// keys; block j's score is the max over the windows touching it.
struct ScoreArgs {
  const void* Q;
  const float* Kc;        // [pairs, kc_rows, d]
  float* scores;          // [pairs, nb] block scores; may be null when chunks == 1
                          // (or, with ov_s > 0, when the caller wants none)
  float* cscores;         // ov_s > 0 and chunks > 1: [pairs, n_rows] window scores
  int32_t* idx;           // [pairs, top_k]
  unsigned* counters;     // [pairs], zero between calls
  unsigned* status;       // workspace status word
  int B, Hq, Hkv, G, n_q;
  int64_t nb;
  int64_t kc_rows;        // Kc rows per pair
  int64_t n_rows;         // rows scored per pair (a prefix of the kc_rows)
  int ov_s, ov_l;         // window stride and length; 0 = one row per block
  int b;
  int64_t s_end, w_begin;
  int top_k;
  float scale;            // softmax scale (mean pooling)
  int lsa;                // cosine scores
  int chunks;             // CTAs per pair
  int64_t rows_per_chunk; // a multiple of kScoreRowsPerPass
};
constexpr int kScoreRowsPerPass = 64;
constexpr int64_t kMaxSelectBlocks = 16384;
cudaError_t launch_score_topk_query0(const ScoreArgs& a, bool bf16, cudaStream_t s);

// ---- decode / chunk sparse attention ---------------------------------------
// Work order of the tensor-core decode kernel: two pair-major lists of units
// (two tiles each), each split evenly over its first g CTAs (CTA c takes
// units [c*tot/g, (c+1)*tot/g)) and run list I first.  With `split`, list I
// holds the tiles that need no index table (sink, window and new keys) and
// list D the selected-block tiles of every pair, so a CTA can attend while
// the tables are still being selected.  Without it both lists hold whole
// per-pair tile lists: list I the first floor(pairs / SMs) * SMs pairs, so
// that every CTA attends the same number of pairs alone and writes their
// outputs directly, list D the remaining pairs, split evenly over the CTAs.
// List I covers pairs [0, pI), list D pairs [pD0, pD0 + totD / mD).  Tile t
// of a list is tile t + off of the per-pair order sink | selected | window
// (I: off = dI for t >= n_sink_tiles, else 0; D: off = dD).  A pair's
// partial results take slots [0, nI) for its list-I CTAs and [nI, nI + nD)
// for its list-D CTAs.
struct TcOrder {
  int mI, mD;             // units per pair
  int ntI, ntD;           // tiles per pair
  int dI, dD;             // tile offsets into the per-pair order
  int gI, gD;             // CTAs sharing each list
  int64_t totI, totD;     // units over all pairs
  int64_t pI, pD0;        // pairs [0, pI) are in list I; list D starts at pair pD0
  int grid;               // max(gI, gD)
  int slots;              // partial slots a pair may need
};
TcOrder tc_order(int64_t pairs, int n_sink_tiles, int n_sel_tiles, int n_wc_tiles, bool split, int num_sms);

struct DecodeAttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;     // [pairs, idx_stride]
  int idx_stride;         // entries per pair
  void* O;
  float* lse;             // may be null
  float* part_O;          // [pairs, n_slots, R4, 128]
  float* part_ml;         // [pairs, n_slots, R4, 2]
  unsigned* counters;     // [pairs], zero between calls
  unsigned* status;
  int B, Hq, Hkv, G, n_q, R, R4;
  int64_t C, cap, kv_end;
  int b;
  int64_t nb;
  int64_t s_end, w_begin;
  int tile;               // keys per tile (64 bf16, 32 fp32); a ring stage holds two
  int n_sink_tiles, tpb, n_wc_tiles, n_tiles;
  int MT;                 // work units (tile pairs) per (sequence, KV head)
  int64_t total_tiles;    // work units over all pairs
  int tpc;                // work units per CTA
  int n_slots;            // partial slots per pair
  int n_stages;
  float qscale;           // softmax scale * log2(e)
  int pdl;                // launched as a programmatic dependent of the scorer
  // fused decode (scoring, selection and attention in one cooperative launch)
  const float* Kc;        // [pairs, nb, 128] compressed keys
  float* scores;          // [pairs, nb] workspace
  unsigned* score_cnt;    // [pairs] score chunks done, zero between calls
  unsigned* ready;        // [pairs] index table published, zero between calls
  unsigned* exit_cnt;     // CTAs finished, zero between calls
  int32_t* idx_w;         // [pairs, top_k] index table written by the fused kernel
  uint2* cand;            // [pairs, kFusedCandSlots, kFusedSmallK] (key, block id) per run of score chunks
  int top_k;
  int cpp;                // score chunks (128 compressed keys) per pair
  int cpc;                // score chunks per CTA
  float sscale;           // scoring scale (the softmax scale)
  int lsa;                // LSA centroids: the index query is normalised instead of scaled
  TcOrder ord;            // tensor-core kernel work order
  // dense verify: per 32-key half-tile of the complete blocks and query row,
  // (sum of the row's probabilities, the running max they are taken against)
  float2* mass_part;      // [pairs, mass_hts, 16], or null
  int64_t mass_keys;      // keys of the complete blocks, nb * b
  int mass_hts;           // mass_keys / 32
  // run mode (CUDA-core kernel only): the selected section is a list of
  // key runs instead of blocks.  Entry e of a pair's row names the run of
  // keys [e_id * run_len, e_id * run_len + run_len), clipped to [s_end,
  // w_begin); -1 entries are empty.  Tile t of the section packs the runs of
  // entries [t * tile / run_len, (t + 1) * tile / run_len) back to back
  // (idx_stride = tiles of the section, tpb = 1).
  const int32_t* runs;    // [pairs, runs_stride], or null
  int runs_stride;
  int run_len;
};

struct DecodePlan {
  int R, R4, RG, KG;
  int tile, n_sink_tiles, tpb, n_wc_tiles, n_tiles, MT;
  int64_t total_tiles;
  int grid, tpc, n_slots, n_stages;
  size_t smem;
  int threads;
  TcOrder tc_plain, tc_split;   // tensor-core orders (two-kernel / fused)
};
// Fills `plan`; returns false (with a reason) if the shape is not built.
bool plan_decode(const DecodeGeom& g, int idx_slots, bool bf16, int num_sms, DecodePlan* plan,
                 const char** why);
cudaError_t launch_decode_attn(const DecodeAttnArgs& a, const DecodePlan& p, bool bf16,
                               bool out_bf16, cudaStream_t s);
// Tensor-core variant for bf16 inputs (decode_tc.cu); launch_decode_attn
// picks it whenever decode_tc_supported() holds.
bool decode_tc_supported(const DecodeAttnArgs& a);
size_t decode_tc_smem_bytes();
cudaError_t launch_decode_tc(const DecodeAttnArgs& a, const DecodePlan& p, bool out_bf16, cudaStream_t s);
// The whole decode step (scores, top-k, attention) in one cooperative launch
// of the tensor-core kernel; for mean pooling or LSA centroids and nb <=
// kFusedMaxBlocks, or past it for k <= kFusedSmallK when every CTA scores at
// most kFusedRunChunks chunks and a pair's chunks span at most
// kFusedCandSlots CTAs.
constexpr int kFusedMaxBlocks = 512;
constexpr int kFusedSmallK = 8;
constexpr int kFusedRunChunks = 4;
constexpr int kFusedCandSlots = 32;
bool decode_fused_supported(const DecodeAttnArgs& a, const DecodePlan& p, int64_t nb);
cudaError_t launch_decode_fused(DecodeAttnArgs a, const DecodePlan& p, bool out_bf16, cudaStream_t s);
// Copies a caller's [rows, len] index table to `out`, keeping only entries
// that are in [0, nb) and above every earlier in-range entry of the row.
cudaError_t launch_sanitize_idx(const int32_t* idx, int32_t* out, int rows, int len, int64_t nb,
                                unsigned* status, cudaStream_t s);

// ---- LSA flat bucket retrieval (bucket.cu) ----------------------------------
// Bucket cache of a pair: rows_per_pair rows, nbk per cluster block of b raw
// keys (block c's buckets are rows [c * nbk, (c + 1) * nbk)), ordered by their
// lowest member; centroids [rows, 128] fp32 unit vectors, members [rows,
// mcap] int32 global pool-key ids (pool key i = raw keys [i * stride, (i + 1)
// * stride)), ascending, -1 padded.
struct WardArgs {
  const void* K;          // [pairs, cap, 128]
  float* cents;
  int32_t* members;
  int64_t cap;            // token stride of K
  int64_t rows_per_pair;
  int64_t first_block;    // cluster blocks [first_block, first_block + gridDim.x) are built
  int b, stride, m, nbk, mcap;   // raw keys per block, per pool key; pool keys per block; buckets; cap
};
cudaError_t launch_ward(const WardArgs& a, int pairs, int64_t n_blocks, bool bf16, cudaStream_t s);
size_t ward_smem_bytes();

struct BucketScoreArgs {
  const void* Q;
  const float* cents;
  const int32_t* members;
  uint32_t* keys;         // [pairs, n_bkt] order-preserving cosine keys, 0 = not a candidate
  uint32_t* cand_key;     // [pairs, chunks * min(top_k, kBucketChunk)] first-level winners (workspace)
  int32_t* cand_id;       // their bucket ids
  int Hq, Hkv, G, n_q;
  int64_t rows_per_pair;
  int64_t n_bkt;          // buckets of the context's complete cluster blocks
  int nbk, b, stride, mcap;
  int64_t s_end, w_begin;
  int64_t rows_per_cta;
};
struct BucketExpandArgs {
  const void* Q;
  const void* K;
  const int32_t* members;
  int32_t* sel;           // [pairs, top_k] selected buckets, ascending, -1 padded
  unsigned long long* own;  // [pairs, top_k * mcap] expansion keys (workspace)
  int32_t* kept;          // [pairs, kept_cap] kept pool keys, ascending, -1 padded
  int Hq, Hkv, G, n_q;
  int64_t cap, rows_per_pair;
  int top_k, mcap, stride;
  int keep_pool;          // pool keys kept (0: every member of the selected buckets)
  int kept_cap;
};
// Scores of every bucket and the top-k selection into ea.sel (two levels:
// the top-k of every kBucketChunk buckets, then of those winners, at most
// kBucketMaxCand per pair, in shared memory).
constexpr int kBucketChunk = 8192;
constexpr int kBucketMaxCand = 28672;
cudaError_t launch_bucket_select(const BucketScoreArgs& sa_, const BucketExpandArgs& ea, int pairs, bool bf16,
                                 cudaStream_t s);
// Expansion of the selected buckets into ea.kept.
cudaError_t launch_bucket_expand(const BucketExpandArgs& a, int pairs, bool bf16, cudaStream_t s);

// ---- dense verify: block attention mass and the refreshed selection --------
// mass[pair][j] = sum over j's half-tiles h and rows r < R of
// part[pair][h][r].x * 2^(part[pair][h][r].y - lse_r * log2 e).
cudaError_t launch_mass_finalize(const float2* part, const float* lse, float* mass, int B, int Hkv, int G, int n_q,
                                 int nb, int b, cudaStream_t s);
cudaError_t launch_mass_topk(const float* mass, int pairs, int nb, int b, int64_t s_end, int64_t w_begin, int k,
                             int32_t* idx, cudaStream_t s);

// ---- prefill (tensor cores) -------------------------------------------------
struct PrefillArgs {
  const void* Q;          // [B, T, Hq, 128] bf16
  const void* K;          // [B, Hkv, cap, 128] bf16
  const void* V;
  const float* Kc;        // [B, Hkv, kc_rows, 128] fp32 (blocks, or windows when ov_s > 0)
  uint16_t* kc2;          // workspace: [B*Hkv, nc, 256] bf16 (hi | lo)
  float* scores;          // scorer output [B*Hkv, n_tiles, nc]: workspace, or the caller's when nc is per block
  float* bscores;         // overlapping windows: the caller's block scores [B*Hkv, n_tiles, nb] or null
  int32_t* idx;           // [B*Hkv, n_tiles, top_k]
  void* O;                // [B, T, Hq, 128]
  float* lse;             // [B, T, Hq] or null
  unsigned* status;
  int B, Hq, Hkv, T, nb, n_tiles, top_k, out_bf16, num_sms;
  int nc;                 // compressed rows scored per pair: nb, or the windows that touch a complete block
  int kc_rows;            // rows per pair of the caller's Kc
  int lsa;                // LSA centroids: each query row normalised instead of scaled
  int ov_s, ov_l;         // overlapping windows (stride, length), 0 otherwise
  int64_t cap, S, W;
  float scale;
};
// Kc split, tile scoring (tcgen05) and per-tile top-k into pa.idx.
cudaError_t launch_prefill_score(const PrefillArgs& pa, cudaStream_t s);
// Causal sparse attention of every tile over pa.idx (tcgen05).
cudaError_t launch_prefill_attn(const PrefillArgs& pa, cudaStream_t s);
size_t prefill_score_smem();
size_t prefill_attn_smem();
// Column-sparse attention (PulseCol eq. (2) with a column mask): every
// 64-token group attends to the columns pa.idx lists for it ([P, n_tiles,
// pa.top_k], ascending from the front, -1 padded), no causal mask.
cudaError_t launch_column_attn(const PrefillArgs& pa, cudaStream_t s);
// Caller column tables: kept entries in [0, T), ascending, packed, -1 padded.
cudaError_t launch_sanitize_cols(const int32_t* in, int32_t* out, int64_t rows, int len, int T, unsigned* status,
                                 cudaStream_t s);
// Caller prefill tables [P, n_tiles, len]: keeps ids j < tile that are above
// every earlier such id of the row and outside sink / window of the tile.
cudaError_t launch_sanitize_prefill_idx(const int32_t* idx, int32_t* out, int P, int n_tiles, int len,
                                        int64_t S, int64_t W, unsigned* status, cudaStream_t s);

}  // namespace sa
