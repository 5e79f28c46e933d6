// Prefill steps 2-3 on tensor cores: tile scoring and per-tile top-k.
//
// Scoring (LSA review §2.4 and SparDA "方法": one index query per GQA group =
// the sum of the group's query vectors; the pages do not say how the rows of
// a 64-query tile are combined -- the reading taken is the max over rows):
//   s[t][j] = max_{r in tile t} ( sum_g q_{r,g} ) . Kc_j * scale
// for every candidate block j of tile t (complete, before the tile, not
// wholly inside sink / window).  LSA centroids (LSA review §2.3): each row's
// index query is normalised instead of scaled, so s is a cosine.
// Overlapping windows (SparDA "方法", overlapping compressed keys): the rows
// of Kc are windows of l keys every s keys; the scorer takes the tile max of
// every window complete inside the tile's context that touches a candidate
// block, and the top-k kernel gives block j the max over the windows that
// share a key with it.
//
// This is a dense contraction, so it runs on tcgen05 tensor cores.  The GEMM
// is transposed -- M = 128 compressed keys (TMEM lanes), N = 128 query rows
// (two tiles, TMEM columns), K = 128 -- so that a TMEM lane holds one block's
// scores against all query rows and the tile max is a per-thread reduction.
// Both operands are split into bf16 hi + lo parts (x = hi + lo exactly up to
// 2^-16 relative) and three products hi*hi + lo*hi + hi*lo are accumulated in
// fp32: single-pass bf16 scores would be ~1e-3 off and flip top-k choices.
//
// CTA roles (persistent, one CTA per SM, work items = (sequence x KV head,
// pair of query tiles) in decreasing-cost order):
//   warp 0      TMA producer: Kc hi / lo chunks of 128 blocks (128-byte swizzle)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 2-9   build the B operand: GQA sum (G a multiple of 4) x scale of
//               128 query rows, split into hi / lo, written to swizzled shared
//               memory (16 rows per warp, 4 rows x 4 heads of loads in flight
//               per round: Q is the kernel's HBM stream)
//   warps 10-13 epilogue: TMEM -> registers, max over each 64-row tile,
//               candidate mask, fp32 scores to global
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace sa {
namespace {

constexpr int kTile = 64;                      // query rows per tile = block size
constexpr int kNSA = 3;                        // A stages (32 KB: hi or lo of a 128-block chunk)
constexpr int kAStage = 32768;
constexpr int kBBuf = 65536;                   // B operand: hi atoms 0,1 then lo atoms 0,1
constexpr int kScoreThreadsTC = 448;
constexpr int kBuilders = 8;                   // warps 2..9 build the B operand, 16 rows each
constexpr uint32_t kIdesc = tc::idesc_bf16(128, 128, false, false);
constexpr int kND = 4;                         // TMEM accumulators of 128 columns (all 512)

struct PSArgs {
  const uint16_t* Q;        // [B, T, Hq, 128] bf16
  float* scores;            // [P, n_tiles, nc]: per compressed row
  float* bscores;           // overlapping windows: block scores [P, n_tiles, nb] or null
  unsigned* status;
  int B, Hq, Hkv, G, T, nb, n_tiles, n_tpairs, P;
  int nc;                   // compressed rows per pair (blocks, or windows)
  int lsa;                  // normalise each row's index query
  int ov_s, ov_l;           // overlapping windows: stride and length (0: blocks)
  int64_t S, W;
  float scale;
};

// Candidate blocks of query tile t (context C = 64 t): [*j_lo, *j_hi), the
// complete blocks that reach past the sink and start before the window
// (none when *j_hi <= *j_lo).
__device__ __forceinline__ void cand_range(const PSArgs& a, int t, int* j_lo, int* j_hi) {
  const int64_t C = static_cast<int64_t>(t) * kTile;
  const int64_t s_end = a.S < C ? a.S : C;
  const int64_t w_begin = (C - a.W) > s_end ? (C - a.W) : s_end;
  const int64_t jh = (w_begin + kTile - 1) / kTile;
  *j_lo = static_cast<int>(s_end / kTile);
  *j_hi = static_cast<int>(jh < a.nb ? jh : a.nb);
}

// Windows complete inside the context of tile t.
__device__ __forceinline__ int windows_in(const PSArgs& a, int t) {
  const int C = t * kTile;
  return C >= a.ov_l ? (C - a.ov_l) / a.ov_s + 1 : 0;
}

// Whether tile t needs the score of compressed row c: a candidate block, or
// a window complete inside the tile's context that shares a key with one.
__device__ __forceinline__ bool row_needed(const PSArgs& a, int t, int c) {
  int j_lo, j_hi;
  cand_range(a, t, &j_lo, &j_hi);
  if (a.ov_s == 0) return c >= j_lo && c < j_hi;
  const int64_t k0 = static_cast<int64_t>(c) * a.ov_s;
  return j_hi > j_lo && c < windows_in(a, t) && k0 < static_cast<int64_t>(j_hi) * kTile &&
         k0 + a.ov_l > static_cast<int64_t>(j_lo) * kTile;
}

// Rows [0, lim) hold every row tiles 2n and 2n+1 need; chunks of 128 of them.
__device__ __forceinline__ int chunk_count(const PSArgs& a, int n) {
  const int t = min(2 * n + 1, a.n_tiles - 1);
  int j_lo, j_hi;
  cand_range(a, t, &j_lo, &j_hi);
  if (j_hi <= j_lo) return 0;                // no block reaches past the sink
  int lim = j_hi;
  if (a.ov_s > 0) {
    // windows starting before the last candidate block's end (s divides 64)
    lim = min(windows_in(a, t), j_hi * (kTile / a.ov_s));
  }
  lim = min(lim, a.nc);
  return (lim + 127) / 128;
}

// Work item k -> (tile pair n, pair p), most expensive first.
__device__ __forceinline__ void item_of(const PSArgs& a, int k, int* n, int* p) {
  *n = a.n_tpairs - 1 - k / a.P;
  *p = k % a.P;
}

__global__ void __launch_bounds__(kScoreThreadsTC, 1)
    prefill_score_kernel(const __grid_constant__ CUtensorMap kc_map, PSArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled operand atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* A = smem;                                     // kNSA x 32 KB
  unsigned char* Bop = A + kNSA * kAStage;                     // 2 x 64 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(Bop + 2 * kBBuf);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + kNSA;
  uint64_t* b_full = a_empty + kNSA;
  uint64_t* b_empty = b_full + 2;
  uint64_t* d_full = b_empty + 2;
  uint64_t* d_empty = d_full + kND;
  uint64_t* mma_done = d_empty + kND;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.n_tpairs * a.P;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNSA; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&b_full[b], kBuilders);
      mbar_init(&b_empty[b], 1);
    }
    for (int d = 0; d < kND; ++d) {
      mbar_init(&d_full[d], 1);
      mbar_init(&d_empty[d], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_base_slot, 128 * kND);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_base_slot;

  auto fail = [&]() {
    report(a.status, kStatusTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- A producer
    if (lane == 0) {
      int use = 0;
      bool ok = true;
      for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x) {
        int n, p;
        item_of(a, k, &n, &p);
        const int mc = chunk_count(a, n);
        for (int m = 0; m < mc && ok; ++m) {
          for (int part = 0; part < 2 && ok; ++part, ++use) {
            const int s = use % kNSA;
            if (use >= kNSA && !mbar_wait_bounded(&a_empty[s], ((use / kNSA) & 1) ^ 1, abort_flag)) {
              fail();
              ok = false;
              break;
            }
            unsigned char* dst = A + s * kAStage;
            mbar_arrive_expect_tx(&a_full[s], kAStage);
            tc::tma_load_3d(dst, &kc_map, part * 128, 128 * m, p, &a_full[s]);
            tc::tma_load_3d(dst + 16384, &kc_map, part * 128 + 64, 128 * m, p, &a_full[s]);
          }
        }
      }
      // drain copies still in flight before the CTA may exit
      for (int u = max(0, use - kNSA); u < use; ++u) mbar_wait_bounded(&a_full[u % kNSA], (u / kNSA) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs the loop in lock step so that the descriptors stay
    // warp-uniform; one elected lane issues each MMA and commit.
    {
      int use = 0, mc_all = 0, it = 0;
      bool ok = true;
      const uint32_t bbase = smem_u32(Bop);
      const uint32_t abase = smem_u32(A);
      for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x) {
        int n, p;
        item_of(a, k, &n, &p);
        const int mc = chunk_count(a, n);
        if (mc == 0) continue;
        const int b = it & 1;
        if (!mbar_wait_warp(&b_full[b], (it >> 1) & 1, abort_flag)) { if (lane == 0) fail(); break; }
        tc::fence_after_sync();
        const uint32_t bhi = bbase + b * kBBuf, blo = bhi + 32768;
        for (int m = 0; m < mc; ++m, ++mc_all) {
          const int d = mc_all % kND;
          if (mc_all >= kND && !mbar_wait_warp(&d_empty[d], ((mc_all / kND) & 1) ^ 1, abort_flag)) {
            if (lane == 0) fail();
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t dt = tbase + d * 128;
          // hi part of Kc: hi*hi then hi*lo
          int s = use % kNSA;
          if (!mbar_wait_warp(&a_full[s], (use / kNSA) & 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          tc::fence_after_sync();
          const uint32_t ahi = abase + s * kAStage;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_elect(dt, tc::smem_desc(ahi + off, 16, 1024), tc::smem_desc(bhi + off, 16, 1024), kIdesc, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_elect(dt, tc::smem_desc(ahi + off, 16, 1024), tc::smem_desc(blo + off, 16, 1024), kIdesc, true);
          }
          tc::mma_commit_elect(&a_empty[s]);
          ++use;
          // lo part of Kc: lo*hi
          s = use % kNSA;
          if (!mbar_wait_warp(&a_full[s], (use / kNSA) & 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          tc::fence_after_sync();
          const uint32_t alo = abase + s * kAStage;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_elect(dt, tc::smem_desc(alo + off, 16, 1024), tc::smem_desc(bhi + off, 16, 1024), kIdesc, true);
          }
          tc::mma_commit_elect(&a_empty[s]);
          ++use;
          tc::mma_commit_elect(&d_full[d]);
        }
        tc::mma_commit_elect(&b_empty[b]);
        ++it;
      }
      // every MMA issued has completed before the CTA tears TMEM down
      tc::mma_commit_elect(mma_done);
      mbar_wait_warp(mma_done, 0, nullptr);
      __syncwarp();
    }
  } else if (warp < 2 + kBuilders) {
    // ---------------------------------------------------- B operand builders
    // Lane l owns the 16-byte column chunk cc = l % 16 (8 columns) of the
    // warp's rows of parity l / 16: it loads the chunk of all G = 4 query
    // heads (a half-warp reads 256 contiguous bytes per head), sums them in
    // fp32, scales, and writes both the bf16 hi part and the bf16 remainder.
    const int wq = warp - 2;                       // rows wq*16 .. wq*16+15 of the item
    const int cc = lane & 15;                      // 16-byte column chunk (8 columns)
    const int rp = lane >> 4;                      // row parity
    // This warp's 16 rows of item kk are prefetched into L2 two items ahead
    // of their use, so the loads below hit L2 and the HBM stream of Q runs
    // on the TMA engine rather than on the builders' registers.
    auto prefetch_item = [&](int kk) {
      if (kk >= n_items || lane >= 16) return;
      int n2, p2;
      item_of(a, kk, &n2, &p2);
      const int row = 128 * n2 + wq * 16 + lane;
      if (chunk_count(a, n2) == 0 || row >= a.T) return;
      const int bi2 = p2 / a.Hkv, h2 = p2 % a.Hkv;
      prefetch_l2_bulk(a.Q + ((static_cast<int64_t>(bi2) * a.T + row) * a.Hq + h2 * a.G) * kHeadDim,
                       static_cast<uint32_t>(a.G) * kHeadDim * 2);
    };
    prefetch_item(blockIdx.x);
    prefetch_item(blockIdx.x + gridDim.x);
    int it = 0;
    for (int k = blockIdx.x; k < n_items; k += gridDim.x) {
      int n, p;
      item_of(a, k, &n, &p);
      prefetch_item(k + 2 * gridDim.x);
      if (chunk_count(a, n) == 0) continue;
      const int b = it & 1;
      if (it >= 2 && !mbar_wait_bounded(&b_empty[b], ((it >> 1) & 1) ^ 1, abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      const int bi = p / a.Hkv, h = p % a.Hkv;
      unsigned char* dst_hi = Bop + b * kBBuf + (cc >> 3) * 16384;
      unsigned char* dst_lo = dst_hi + 32768;
#pragma unroll 1
      for (int rb = 0; rb < 8; rb += 4) {
        // the GQA sum over the group's G heads, four heads of four rows per round
        float vs[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < 8; ++e) vs[u][e] = 0.f;
#pragma unroll 1
        for (int hb = 0; hb < a.G; hb += 4) {
          uint4 x[4][4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int row = 128 * n + wq * 16 + 2 * (rb + u) + rp;
            const uint4* src = reinterpret_cast<const uint4*>(
                a.Q + ((static_cast<int64_t>(bi) * a.T + (row < a.T ? row : 0)) * a.Hq + h * a.G + hb) * kHeadDim);
#pragma unroll
            for (int g = 0; g < 4; ++g)
              x[u][g] = row < a.T ? __ldg(src + g * 16 + cc) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float f[8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              unpack8(x[u][g], f);
#pragma unroll
              for (int e = 0; e < 8; ++e) vs[u][e] += f[e];
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = wq * 16 + 2 * (rb + u) + rp;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = vs[u][e];
          float mul = a.scale;
          if (a.lsa) {
            // the row's 128 columns sit on the 16 lanes of this half-warp
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += v[e] * v[e];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            mul = ss > 0.f ? rsqrtf(ss) : 0.f;
          }
          uint32_t whi[4], wlo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float v0 = v[2 * e] * mul, v1 = v[2 * e + 1] * mul;
            whi[e] = pack_bf16x2(v0, v1);
            wlo[e] = pack_bf16x2(v0 - bf16lo(whi[e]), v1 - bf16hi(whi[e]));
          }
          *reinterpret_cast<uint4*>(dst_hi + tc::sw128_off(r, cc & 7)) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
          *reinterpret_cast<uint4*>(dst_lo + tc::sw128_off(r, cc & 7)) = make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_full[b]);
      ++it;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quadrant of this warp
    int mc_all = 0;
    bool ok = true;
    for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x) {
      int n, p;
      item_of(a, k, &n, &p);
      const int mc = chunk_count(a, n);
      for (int m = 0; m < mc; ++m, ++mc_all) {
        const int d = mc_all % kND;
        if (!mbar_wait_bounded(&d_full[d], (mc_all / kND) & 1, abort_flag)) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const int j = 128 * m + 32 * q + lane;      // this thread's compressed row
        float best[2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float v[64];
          tc::tmem_ld64(tbase + (static_cast<uint32_t>(32 * q) << 16) + d * 128 + half * 64, v);
          tc::tmem_wait_ld();
          const int t = 2 * n + half;
          const int rows = min(kTile, a.T - t * kTile);    // ragged last tile
          float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
          if (rows == kTile) {
#pragma unroll
            for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], v[c]);
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) m4[c & 3] = (c < rows) ? fmaxf(m4[c & 3], v[c]) : m4[c & 3];
          }
          best[half] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[d]);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int t = 2 * n + half;
          if (t < a.n_tiles && row_needed(a, t, j))
            a.scores[(static_cast<int64_t>(p) * a.n_tiles + t) * a.nc + j] = best[half];
        }
      }
    }
  }
  // every warp reaches the final barrier converged (lane-0 drains above)
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 128 * kND);
  }
}

// Kc (fp32, kc_rows rows per pair) -> [hi | lo] bf16 rows of 256 elements,
// the first nc rows of every pair, for the TMA loads.
__global__ void kc_split_kernel(const float* Kc, uint16_t* out, int64_t rows, int nc, int kc_rows) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;   // one float4 each
  if (i >= rows * 32) return;
  const int64_t r = i / 32, c = i % 32;
  const int64_t pr = r / nc, row = r - pr * nc;
  const float4 x = reinterpret_cast<const float4*>(Kc + (pr * kc_rows + row) * kHeadDim)[c];
  const float v[4] = {x.x, x.y, x.z, x.w};
  uint16_t hi[4], lo[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v[e]);
    hi[e] = __bfloat16_as_ushort(h);
    lo[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v[e] - __bfloat162float(h)));
  }
  uint16_t* o = out + r * 256 + c * 4;
  *reinterpret_cast<uint2*>(o) = make_uint2(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16));
  *reinterpret_cast<uint2*>(o + 128) = make_uint2(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16));
}

// Per (pair, tile) top-k over the candidate scores, one warp each.
__global__ void __launch_bounds__(256, 2) prefill_topk_kernel(PSArgs a, int top_k, int32_t* idx) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (row >= static_cast<int64_t>(a.P) * a.n_tiles) return;
  const int t = static_cast<int>(row % a.n_tiles);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw) + warp * a.nb;
  const float* sc = a.scores + row * a.nc;
  // blocks at or after the tile are never candidates
  const int nb_t = min(a.nb, t);
  int j_lo, j_hi;
  cand_range(a, t, &j_lo, &j_hi);
  j_hi = min(j_hi, nb_t);
  if (a.ov_s > 0) {
    // block j: the max over the windows complete inside the context that
    // share a key with it, c s + l > 64 j and c s < 64 (j + 1); every
    // candidate has one (the window starting at its first key)
    const int s = a.ov_s, l = a.ov_l, last = windows_in(a, t) - 1;
    for (int j = lane; j < nb_t; j += 32) {
      uint32_t key = 0u;
      if (j >= j_lo && j < j_hi) {
        const int ca = j * kTile - l >= 0 ? (j * kTile - l) / s + 1 : 0;
        const int cb = min(last, ((j + 1) * kTile - 1) / s);
        float m = -CUDART_INF_F;
        for (int c = ca; c <= cb; ++c) m = fmaxf(m, __ldcg(sc + c));
        if (a.bscores) a.bscores[row * a.nb + j] = m;
        key = float_key(m);
        key = key == 0u ? 1u : key;
      }
      keys[j] = key;
    }
  }
  for (int j0 = 0; a.ov_s == 0 && j0 < nb_t; j0 += 32 * 32) {
    float v[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int j = j0 + u * 32 + lane;
      v[u] = (j >= j_lo && j < j_hi) ? __ldcg(sc + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < nb_t) {
        const uint32_t key = float_key(v[u]);
        keys[j] = (j >= j_lo && j < j_hi) ? (key == 0u ? 1u : key) : 0u;
      }
    }
  }
  __syncwarp();
  warp_topk(keys, nb_t, top_k, idx + row * top_k);
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

size_t prefill_score_smem() {
  return 1024 + kNSA * kAStage + 2 * kBBuf + (2 * kNSA + 4 + 2 * kND + 1) * 8 + 64;
}

cudaError_t launch_prefill_score(const PrefillArgs& pa, cudaStream_t s) {
  EncodeFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  PSArgs a = {};
  a.Q = static_cast<const uint16_t*>(pa.Q);
  a.scores = pa.scores;
  a.bscores = pa.bscores;
  a.status = pa.status;
  a.B = pa.B;
  a.Hq = pa.Hq;
  a.Hkv = pa.Hkv;
  a.G = pa.Hq / pa.Hkv;
  a.T = pa.T;
  a.nb = pa.nb;
  a.nc = pa.nc;
  a.lsa = pa.lsa;
  a.ov_s = pa.ov_s;
  a.ov_l = pa.ov_l;
  a.n_tiles = pa.n_tiles;
  a.n_tpairs = (pa.n_tiles + 1) / 2;
  a.P = pa.B * pa.Hkv;
  a.S = pa.S;
  a.W = pa.W;
  a.scale = pa.scale;
  if (a.nc > 0) {
    // Kc -> hi / lo bf16
    const int64_t rows = static_cast<int64_t>(a.P) * a.nc;
    kc_split_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, s>>>(pa.Kc, pa.kc2, rows, a.nc,
                                                                                    pa.kc_rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap map;
    cuuint64_t dims[3] = {256, static_cast<cuuint64_t>(a.nc), static_cast<cuuint64_t>(a.P)};
    cuuint64_t strides[2] = {256 * 2, static_cast<cuuint64_t>(a.nc) * 256 * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pa.kc2, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const size_t smem = prefill_score_smem();
    e = cudaFuncSetAttribute(prefill_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int items = a.n_tpairs * a.P;
    const int grid = items < pa.num_sms ? items : pa.num_sms;
    prefill_score_kernel<<<grid, kScoreThreadsTC, smem, s>>>(map, a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = static_cast<int64_t>(a.P) * a.n_tiles;
  const size_t smem_k = 8 * static_cast<size_t>(a.nb) * 4;
  cudaError_t e = cudaFuncSetAttribute(prefill_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_k));
  if (e != cudaSuccess) return e;
  prefill_topk_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, smem_k, s>>>(a, pa.top_k, pa.idx);
  return cudaGetLastError();
}

}  // namespace sa
