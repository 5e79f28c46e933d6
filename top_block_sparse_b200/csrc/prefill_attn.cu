// Prefill step 4 on tensor cores: causal sparse attention of every 64-query
// tile over the keys its selection retains (S3R review, section "稀疏起草":
// softmax over the retained set only; PulseCol §3.1 eq. (1)-(2): logits
// q.k/sqrt(d_h), other keys weight zero).  Tile t (context C = 64 t) attends
//   sink [0, min(S, C)) U selected blocks U window [max(C - W, sink end), C)
//   U its own block, causally (query row r sees keys 64 t .. 64 t + r).
//
// One work item = (sequence x KV head, tile, group of 4 of the KV head's G
// query heads): 64 tokens x 4 heads = 256 query rows = two M = 128 halves
// (row m = 4 * token + head, the order a 3-D TMA box of Q lands in); G a
// multiple of 4, the G / 4 items of a tile sharing its block list.  Per 64-key block:
//   S   = Q K^T          tcgen05.mma, M 128, N 64, K 128 per half, fp32 in TMEM
//   P   = softmax(S)     8 warps, one query row per thread (online, lazy
//                        rescale when the row max grows by more than 2^8),
//                        bf16 into 128-byte-swizzled shared memory
//   O  += P V            tcgen05.mma, M 128, N 128, K 64 per half; V is the
//                        MN-major operand straight from its TMA tile
// CTA roles: warps 0-7 softmax / epilogue, warp 8 TMA producer (Q once per
// item, then K and V blocks through a 4-stage ring), warp 9 TMEM owner and
// MMA issuer.  S(b + 1) is issued as soon as the softmax has read S(b), so
// the tensor cores overlap the softmax.
//
// Column mode (PulseCol §3.1 eq. (2) with a token-granular column mask): the
// item's 64 tokens x 4 heads attend to the key columns listed for the group
// (ascending, -1 padded), before or after them alike.  Four producer warps
// gather each chunk of 64 listed K and V rows with 16-byte cp.async copies
// into the same 128-byte-swizzled stage layout the tensor maps produce,
// keeps up to three chunks in flight (cp.async groups), and, once a chunk
// has landed, fences it for the tensor cores and arrives on the stage's
// barrier (one arrival per lane).  The last chunk's unused columns are
// masked; an empty list is one fully masked chunk (O = 0, lse = -inf).
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace sa {
namespace {

constexpr int kT = 64;                         // tile = block = 64
constexpr int kG = 4;                          // query heads of one work item
constexpr int kRows = kT * kG;                 // 256 query rows per item
constexpr int kNKV = 4;                        // K/V ring stages
constexpr int kQBytes = kRows * 256;           // 64 KB (two 32 KB boxes: d 0-63, d 64-127)
constexpr int kKVStage = 32768;                // K 16 KB (two 8 KB boxes) + V 16 KB
constexpr int kPBytes = 2 * 16384;             // P: two halves of 128 rows x 64 keys
constexpr int kThreads = 320;
constexpr int kGatherWarps = 4;                // column mode: warps 8, 10, 11 and 12 gather K and V rows
constexpr int kGatherRows = kT / kGatherWarps;  // rows of a chunk per gathering warp
constexpr int kLanesPerRow = 32 / kGatherRows;
constexpr int kThreadsCol = kThreads + (kGatherWarps - 1) * 32;
constexpr uint32_t kIdescS = tc::idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescO = tc::idesc_bf16(128, 128, false, true);
constexpr float kLazy = 8.f;                   // rescale when the max grows by > 2^8

// 2^x by the hardware approximation (ex2.approx, relative error ~2^-22);
// 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 -> packed bf16 pair (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

struct PAArgs {
  const int32_t* idx;       // [P, n_tiles, k] (column mode: the column lists, k = n_cols)
  const void* K;            // column mode: [P, cap, 128] bf16 (gathered by cp.async)
  const void* V;
  int64_t cap;
  void* O;                  // [B, T, Hq, 128]
  float* lse;               // [B, T, Hq] or null
  unsigned* status;
  int B, Hq, Hkv, T, n_tiles, P, top_k, out_bf16;
  int HG;                   // groups of kG query heads per KV head (G / 4)
  int64_t S, W;
  float scale_log2;         // softmax scale * log2(e)
};

struct Blocks {
  int n_sink, n_sel, w_first, n_blk;   // sink blocks, selected, first window block, total
};

// Block list of tile t: sink blocks, the selected blocks (ascending, -1
// entries skipped; they lie between sink and window), window blocks, the
// tile's own block.  n_sel is counted by the calling warp.
__device__ __forceinline__ Blocks blocks_of(const PAArgs& a, int p, int t, int lane) {
  Blocks bl;
  const int64_t C = static_cast<int64_t>(t) * kT;
  const int64_t s_end = a.S < C ? a.S : C;
  const int64_t w_begin = (C - a.W) > s_end ? (C - a.W) : s_end;
  bl.n_sink = static_cast<int>(s_end / kT);
  bl.w_first = static_cast<int>(w_begin / kT);
  const int32_t* row = a.idx + (static_cast<int64_t>(p) * a.n_tiles + t) * a.top_k;
  int cnt = 0;
  for (int s = lane; s < a.top_k; s += 32) cnt += __ldg(row + s) >= 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  bl.n_sel = cnt;
  bl.n_blk = bl.n_sink + cnt + (t - bl.w_first) + 1;
  return bl;
}

// Column mode: n_sel = the group's listed columns (entries >= 0, which lead
// the row), n_blk = chunks of 64 of them, at least one.
__device__ __forceinline__ Blocks col_blocks_of(const PAArgs& a, int p, int t, int lane) {
  Blocks bl;
  const int32_t* row = a.idx + (static_cast<int64_t>(p) * a.n_tiles + t) * a.top_k;
  int cnt = 0;
  for (int s = lane; s < a.top_k; s += 32) cnt += __ldg(row + s) >= 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  bl.n_sink = 0;
  bl.n_sel = cnt;
  bl.w_first = 0;
  bl.n_blk = cnt > 0 ? (cnt + kT - 1) / kT : 1;
  return bl;
}

template <bool COL>
__device__ __forceinline__ Blocks item_blocks(const PAArgs& a, int p, int t, int lane) {
  if constexpr (COL) return col_blocks_of(a, p, t, lane);
  else return blocks_of(a, p, t, lane);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Item k -> (pair p, tile t, head group hg), most expensive tiles first, a
// tile's head groups next to each other (they read the same K and V blocks).
__device__ __forceinline__ void item_of(const PAArgs& a, int k, int* p, int* t, int* hg) {
  const int per_tile = a.P * a.HG;
  *t = a.n_tiles - 1 - k / per_tile;
  const int q = k - (k / per_tile) * per_tile;
  *p = q / a.HG;
  *hg = q - *p * a.HG;
}

template <bool COL>
__global__ void __launch_bounds__(COL ? kThreadsCol : kThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                        const __grid_constant__ CUtensorMap v_map, PAArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* Qs = smem;                                   // 64 KB
  unsigned char* KV = Qs + kQBytes;                           // kNKV x 32 KB
  unsigned char* Ps = KV + kNKV * kKVStage;                   // 32 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(Ps + kPBytes);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kNKV;
  uint64_t* q_full = kv_empty + kNKV;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_empty + 1;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* pv_done = p_full + 1;
  uint64_t* o_free = pv_done + 1;
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.n_tiles * a.P * a.HG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNKV; ++s) {
      mbar_init(&kv_full[s], COL ? 32 * kGatherWarps : 1);   // column mode: one arrival per gathering lane
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_full, 8);
    mbar_init(pv_done, 1);
    mbar_init(o_free, 8);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;      // S halves at columns 0 / 64, O halves at 128 / 256

  auto fail = [&]() {
    report(a.status, kStatusTimeout);
    *abort_flag = 1;
  };

  if (warp == 8 || (COL && warp >= 10)) {
    // -------------------------------------------------------- TMA producer
    // column mode: warps 8, 10, 11 and 12 gather kGatherRows of every
    // chunk's rows each, two lanes a row; warp 8 also loads Q
    const int gw = warp == 8 ? 0 : warp - 9;
    int use = 0, it = 0;
    bool ok = true;
    for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x, ++it) {
      int p, t, hg;
      item_of(a, k, &p, &t, &hg);
      const Blocks bl = item_blocks<COL>(a, p, t, lane);
      const int32_t* row = a.idx + (static_cast<int64_t>(p) * a.n_tiles + t) * a.top_k;
      const int bi = p / a.Hkv, h = p % a.Hkv;
      const int h0 = (h * a.HG + hg) * kG;           // the item's first query head
      if constexpr (COL) {
        if (warp == 8 && lane == 0) {
          if (it > 0 && !mbar_wait_bounded(q_empty, (it - 1) & 1, abort_flag)) { fail(); ok = false; }
          if (ok) {
            mbar_arrive_expect_tx(q_full, kQBytes);
            const int tok = bi * a.T + t * kT;
            tc::tma_load_3d(Qs, &q_map, 0, h0, tok, q_full);
            tc::tma_load_3d(Qs + kQBytes / 2, &q_map, 64, h0, tok, q_full);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        const unsigned char* kb = static_cast<const unsigned char*>(a.K) + static_cast<int64_t>(p) * a.cap * 256;
        const unsigned char* vb = static_cast<const unsigned char*>(a.V) + static_cast<int64_t>(p) * a.cap * 256;
        int pend = 0;                               // chunks copied but not yet signalled
        // slot r of chunk b <- listed column b * 64 + r (past the list:
        // column 0, masked; clamped into the sequence either way); this
        // warp copies slots kGatherRows gw .. + kGatherRows - 1, kLanesPerRow
        // lanes a slot, its column id loaded one chunk ahead of the copies
        const int r = gw * kGatherRows + lane % kGatherRows;
        auto load_col = [&](int b) -> int {
          const int e = b * kT + r;
          return e < bl.n_sel ? __ldg(row + e) : 0;
        };
        int nxt = load_col(0);
        for (int b = 0; b < bl.n_blk && ok; ++b, ++use) {
          const int cur = nxt;
          if (b + 1 < bl.n_blk) nxt = load_col(b + 1);
          const int s = use % kNKV;
          int fine = 1;
          if (lane == 0 && use >= kNKV && !mbar_wait_bounded(&kv_empty[s], ((use / kNKV) & 1) ^ 1, abort_flag)) {
            fail();
            fine = 0;
          }
          if (!__shfl_sync(0xffffffffu, fine, 0)) {
            ok = false;
            break;
          }
          unsigned char* st = KV + s * kKVStage;
          {
            const int col = min(max(cur, 0), a.T - 1);
            const unsigned char* ks = kb + static_cast<int64_t>(col) * 256;
            const unsigned char* vs = vb + static_cast<int64_t>(col) * 256;
            constexpr int kPer = 16 / kLanesPerRow;   // this lane's share of the row's 16 chunks of 16 bytes
            const int hb = (lane / kGatherRows) * kPer;
#pragma unroll
            for (int c = 0; c < kPer; ++c) {
              const int c16 = hb + c;
              const uint32_t off = (c16 >> 3) * 8192 + tc::sw128_off(r, c16 & 7);
              cp_async16(st + off, ks + c16 * 16);
              cp_async16(st + 16384 + off, vs + c16 * 16);
            }
          }
          cp_async_commit();
          if (++pend == 3) {
            // chunk use - 2 has landed: make it visible to the tensor cores
            cp_async_wait<2>();
            tc::fence_proxy_async_smem();
            mbar_arrive(&kv_full[(use - 2) % kNKV]);
            --pend;
          }
        }
        // the item's last chunks (also after an error: every copy must land)
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        for (int q = pend; q > 0; --q) mbar_arrive(&kv_full[(use - q) % kNKV]);
        continue;
      }
      if (lane == 0) {
        if (it > 0 && !mbar_wait_bounded(q_empty, (it - 1) & 1, abort_flag)) { fail(); ok = false; }
        if (ok) {
          mbar_arrive_expect_tx(q_full, kQBytes);
          const int tok = bi * a.T + t * kT;
          tc::tma_load_3d(Qs, &q_map, 0, h0, tok, q_full);
          tc::tma_load_3d(Qs + kQBytes / 2, &q_map, 64, h0, tok, q_full);
        }
        int sel = 0;   // position in the index row
        for (int b = 0; b < bl.n_blk && ok; ++b, ++use) {
          int j;
          if (b < bl.n_sink) {
            j = b;
          } else if (b < bl.n_sink + bl.n_sel) {
            j = -1;
            while (j < 0) j = __ldg(row + sel++);
          } else {
            j = bl.w_first + (b - bl.n_sink - bl.n_sel);     // window blocks, then the tile itself
          }
          const int s = use % kNKV;
          if (use >= kNKV && !mbar_wait_bounded(&kv_empty[s], ((use / kNKV) & 1) ^ 1, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          unsigned char* st = KV + s * kKVStage;
          mbar_arrive_expect_tx(&kv_full[s], kKVStage);
          tc::tma_load_3d(st, &k_map, 0, j * kT, p, &kv_full[s]);
          tc::tma_load_3d(st + 8192, &k_map, 64, j * kT, p, &kv_full[s]);
          tc::tma_load_3d(st + 16384, &v_map, 0, j * kT, p, &kv_full[s]);
          tc::tma_load_3d(st + 24576, &v_map, 64, j * kT, p, &kv_full[s]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0)
      for (int u = max(0, use - kNKV); u < use; ++u) mbar_wait_bounded(&kv_full[u % kNKV], (u / kNKV) & 1, nullptr);
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    int use = 0, it = 0, nb_all = 0;
    bool ok = true;
    const uint32_t qa = smem_u32(Qs), kva = smem_u32(KV), pa = smem_u32(Ps);
    for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x, ++it) {
      int p, t, hg;
      item_of(a, k, &p, &t, &hg);
      const Blocks bl = item_blocks<COL>(a, p, t, lane);
      // the whole warp runs the issue loop in lock step (descriptors stay
      // warp-uniform); one elected lane issues each MMA and commit
      {
        if (!mbar_wait_warp(q_full, it & 1, abort_flag)) { if (lane == 0) fail(); ok = false; }
        tc::fence_after_sync();
        // S(b) for both halves
        auto issue_s = [&](int b_use) {
          const int s = b_use % kNKV;
          const uint32_t kst = kva + s * kKVStage;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t qoff = (kk >> 2) * (kQBytes / 2) + hf * 16384 + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
              tc::mma_bf16_elect(tbase + hf * 64, tc::smem_desc(qa + qoff, 16, 1024), tc::smem_desc(kst + koff, 16, 1024),
                           kIdescS, kk > 0);
            }
          }
          tc::mma_commit_elect(s_full);
        };
        if (ok) {
          // S(0) needs the S columns free: the previous item's last S was read
          if (nb_all > 0 && !mbar_wait_warp(s_free, (nb_all - 1) & 1, abort_flag)) { if (lane == 0) fail(); ok = false; }
          if (ok && !mbar_wait_warp(&kv_full[use % kNKV], (use / kNKV) & 1, abort_flag)) { if (lane == 0) fail(); ok = false; }
          if (ok) {
            tc::fence_after_sync();
            issue_s(use);
          }
        }
        for (int b = 0; b < bl.n_blk && ok; ++b, ++use, ++nb_all) {
          if (b + 1 < bl.n_blk) {
            // S(b+1) as soon as the softmax has read S(b) and K(b+1) has landed
            if (!mbar_wait_warp(s_free, nb_all & 1, abort_flag) ||
                !mbar_wait_warp(&kv_full[(use + 1) % kNKV], ((use + 1) / kNKV) & 1, abort_flag)) {
              if (lane == 0) fail();
              ok = false;
              break;
            }
            tc::fence_after_sync();
            issue_s(use + 1);
          } else {
            tc::mma_commit_elect(q_empty);            // Q is read by no later MMA of this item
          }
          if (!mbar_wait_warp(p_full, nb_all & 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          if (b == 0 && it > 0 && !mbar_wait_warp(o_free, (it - 1) & 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          tc::fence_after_sync();
          const uint32_t vst = kva + (use % kNKV) * kKVStage + 16384;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              tc::mma_bf16_elect(tbase + 128 + hf * 128, tc::smem_desc(pa + hf * 16384 + kk * 32, 16, 1024),
                           tc::smem_desc(vst + kk * 2048, 8192, 1024), kIdescO, b > 0 || kk > 0);
            }
          }
          tc::mma_commit_elect(&kv_empty[use % kNKV]);
          tc::mma_commit_elect(pv_done);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      use = __shfl_sync(0xffffffffu, use, 0);
      nb_all = __shfl_sync(0xffffffffu, nb_all, 0);
    }
    tc::mma_commit_elect(mma_done);
    mbar_wait_warp(mma_done, 0, nullptr);
  } else {
    // ------------------------------------------------- softmax and epilogue
    const int hf = warp >> 2, q = warp & 3;
    const int m = hf * 128 + q * 32 + lane;       // query row of this thread
    const int r = m / kG, g = m % kG;             // token in tile, head in group
    const uint32_t t_s = tbase + (static_cast<uint32_t>(q * 32) << 16) + hf * 64;
    const uint32_t t_o = tbase + (static_cast<uint32_t>(q * 32) << 16) + 128 + hf * 128;
    unsigned char* prow = Ps + hf * 16384;
    int it = 0, nb_all = 0;
    bool ok = true;
    for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x, ++it) {
      int p, t, hg;
      item_of(a, k, &p, &t, &hg);
      const Blocks bl = item_blocks<COL>(a, p, t, lane);
      float m_ref = -CUDART_INF_F, l = 0.f;
      for (int b = 0; b < bl.n_blk; ++b, ++nb_all) {
        if (!mbar_wait_bounded(s_full, nb_all & 1, abort_flag)) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc::fence_after_sync();
        float s[64];
        tc::tmem_ld64(t_s, s);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        if constexpr (COL) {
          // the last chunk's slots past the list are masked
          const int nlast = bl.n_sel - b * kT;
          if (nlast < kT) {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = (c < nlast) ? s[c] : -CUDART_INF_F;
          }
        } else {
          const bool diag = b == bl.n_blk - 1;        // the tile's own block: causal
          if (diag) {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = (c <= r) ? s[c] : -CUDART_INF_F;
          }
        }
        // row max of the raw logits (8 independent chains; the scale is > 0)
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
        for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * a.scale_log2;
        float factor = 1.f;
        bool rescale = false;
        if (mx > m_ref + kLazy) {
          const float m_new = mx;
          if (m_ref != -CUDART_INF_F) {
            factor = ex2(m_ref - m_new);
            rescale = true;
          }
          l *= factor;
          m_ref = m_new;
        }
        // P(b) may be written once PV(b-1) has read P(b-1); O may be rescaled then too
        if (nb_all > 0 && (b > 0) && !mbar_wait_bounded(pv_done, (nb_all - 1) & 1, abort_flag)) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            float o[32];
            tc::tmem_ld32(t_o + c0, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= factor;
            tc::tmem_st32(t_o + c0, o);
          }
          tc::tmem_wait_st();
        }
        // p = 2^(s * scale_log2 - m_ref): one FFMA and one ex2 per element; the
        // row sum uses the fp32 values, P goes to the tensor cores in bf16
        float ls0 = 0.f, ls1 = 0.f;
        // (column mode: a row may have no key yet; 2^-inf = 0 then)
        const float neg_m = (COL && m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2(fmaf(s[8 * c8 + 2 * e], a.scale_log2, neg_m));
            const float p1 = ex2(fmaf(s[8 * c8 + 2 * e + 1], a.scale_log2, neg_m));
            ls0 += p0;
            ls1 += p1;
            w[e] = cvt_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + tc::sw128_off(q * 32 + lane, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        const float ls = ls0 + ls1;
        l += ls;
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      // epilogue: O / l once the item's last PV has completed
      if (!mbar_wait_bounded(pv_done, (nb_all - 1) & 1, abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      tc::fence_after_sync();
      const int bi = p / a.Hkv, h = p % a.Hkv;
      const int tok = t * kT + r;
      const bool valid = tok < a.T;
      const int64_t orow = (static_cast<int64_t>(bi) * a.T + tok) * a.Hq + (h * a.HG + hg) * kG + g;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float o[32];
        tc::tmem_ld32(t_o + c0, o);
        tc::tmem_wait_ld();
        if (valid) {
          if (a.out_bf16) {
            uint16_t* dst = static_cast<uint16_t*>(a.O) + orow * kHeadDim + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 8)
              *reinterpret_cast<uint4*>(dst + c) =
                  make_uint4(pack_bf16x2(o[c] * inv, o[c + 1] * inv), pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv),
                             pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv), pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv));
          } else {
            float* dst = static_cast<float*>(a.O) + orow * kHeadDim + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + c) = make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
          }
        }
      }
      if (valid && a.lse) a.lse[orow] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }
  // every warp reaches the final barrier converged (lane-0 drains above)
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 512);
  }
}

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

}  // namespace

size_t prefill_attn_smem() { return 1024 + kQBytes + kNKV * kKVStage + kPBytes + 16 * 8 + 64; }

cudaError_t launch_prefill_attn(const PrefillArgs& pa, cudaStream_t s) {
  EncodeFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  PAArgs a = {};
  a.idx = pa.idx;
  a.O = pa.O;
  a.lse = pa.lse;
  a.status = pa.status;
  a.B = pa.B;
  a.Hq = pa.Hq;
  a.Hkv = pa.Hkv;
  a.HG = pa.Hq / pa.Hkv / kG;
  a.T = pa.T;
  a.n_tiles = pa.n_tiles;
  a.P = pa.B * pa.Hkv;
  a.top_k = pa.top_k;
  a.out_bf16 = pa.out_bf16;
  a.S = pa.S;
  a.W = pa.W;
  a.scale_log2 = pa.scale * 1.4426950408889634f;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap qm, km, vm;
  {
    // Q [B*T tokens][Hq heads][128]: box 64 columns x 4 heads x 64 tokens
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(pa.Hq), static_cast<cuuint64_t>(pa.B) * pa.T};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(pa.Hq) * 256};
    cuuint32_t box[3] = {64, kG, kT};
    if (enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pa.Q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // K, V [P pairs][cap keys][128]: box 64 columns x 64 keys
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(pa.cap), static_cast<cuuint64_t>(a.P)};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(pa.cap) * 256};
    cuuint32_t box[3] = {64, kT, 1};
    if (enc(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pa.K), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (enc(&vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pa.V), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = prefill_attn_smem();
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int items = pa.n_tiles * a.P * a.HG;
  const int grid = items < pa.num_sms ? items : pa.num_sms;
  prefill_attn_kernel<false><<<grid, kThreads, smem, s>>>(qm, km, vm, a);
  return cudaGetLastError();
}

cudaError_t launch_column_attn(const PrefillArgs& pa, cudaStream_t s) {
  EncodeFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  PAArgs a = {};
  a.idx = pa.idx;
  a.K = pa.K;
  a.V = pa.V;
  a.cap = pa.cap;
  a.O = pa.O;
  a.lse = pa.lse;
  a.status = pa.status;
  a.B = pa.B;
  a.Hq = pa.Hq;
  a.Hkv = pa.Hkv;
  a.HG = pa.Hq / pa.Hkv / kG;
  a.T = pa.T;
  a.n_tiles = pa.n_tiles;
  a.P = pa.B * pa.Hkv;
  a.top_k = pa.top_k;
  a.out_bf16 = pa.out_bf16;
  a.scale_log2 = pa.scale * 1.4426950408889634f;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap qm;
  {
    // Q [B*T tokens][Hq heads][128]: box 64 columns x 4 heads x 64 tokens
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(pa.Hq), static_cast<cuuint64_t>(pa.B) * pa.T};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(pa.Hq) * 256};
    cuuint32_t box[3] = {64, kG, kT};
    if (enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pa.Q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = prefill_attn_smem();
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int items = pa.n_tiles * a.P * a.HG;
  const int grid = items < pa.num_sms ? items : pa.num_sms;
  // K and V are gathered by cp.async: their tensor-map slots are unused
  prefill_attn_kernel<true><<<grid, kThreadsCol, smem, s>>>(qm, qm, qm, a);
  return cudaGetLastError();
}

namespace {

// One warp per row of a caller's column table: keeps the entries in [0, T)
// that are above every earlier kept entry (ascending, no repeats), packed
// to the front and -1 padded; any other entry except -1 reports the index
// status bit.
__global__ void __launch_bounds__(256) sanitize_cols_kernel(const int32_t* __restrict__ in, int32_t* __restrict__ out,
                                                            int64_t rows, int len, int T, unsigned* status) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * 8) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int32_t* src = in + row * len;
  int32_t* dst = out + row * len;
  int last = -1, n = 0;
  bool bad = false;
  for (int base = 0; base < len; base += 32) {
    const int e = base + lane;
    const int v = e < len ? __ldg(src + e) : -1;
    const bool in_range = v >= 0 && v < T;
    bad |= e < len && v != -1 && !in_range;
    // largest in-range entry strictly before this lane (carried across chunks)
    int m = in_range ? v : -1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, m, o);
      if (lane >= o) m = max(m, y);
    }
    int before = __shfl_up_sync(0xffffffffu, m, 1);
    before = lane == 0 ? last : max(before, last);
    const bool keep = in_range && v > before;
    bad |= in_range && !keep;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) dst[n + __popc(bal & ((1u << lane) - 1u))] = v;
    n += __popc(bal);
    last = max(last, __shfl_sync(0xffffffffu, m, 31));
  }
  for (int e = n + lane; e < len; e += 32) dst[e] = -1;
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, kStatusIndex);
}

}  // namespace

cudaError_t launch_sanitize_cols(const int32_t* in, int32_t* out, int64_t rows, int len, int T, unsigned* status,
                                 cudaStream_t s) {
  if (rows == 0 || len == 0) return cudaSuccess;
  sanitize_cols_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(in, out, rows, len, T, status);
  return cudaGetLastError();
}

}  // namespace sa
