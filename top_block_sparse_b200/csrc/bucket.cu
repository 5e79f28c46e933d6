// LSA flat bucket retrieval (LSA review "精读:LSA", §2.2 and §2.3).
//
// §2.2, building the bucket cache of a cluster block (ward_kernel, one CTA
// per (sequence, KV head, cluster block)): every raw key is L2-normalised,
// `stride` consecutive unit keys are summed into a pool key, and the block's
// pool keys are clustered bottom-up by Ward's criterion: each starts as its
// own bucket, and every round all pairs of buckets that are each other's
// cheapest merge merge at once, until b / 8 buckets remain, none holding more
// than 16 raw keys.  A bucket's centroid is the normalised sum of its pool
// keys; the cache keeps centroids and member lists.
//
// §2.3, retrieval for a decode step: the normalised index query (the sum of
// the KV head's query heads, first new token) scores every centroid
// (bucket_score_kernel, an HBM stream), the top-k candidate buckets are kept
// (bucket_select_kernel, one CTA per pair), their member pool keys are ranked
// by their own cosine with the query and the best N / stride kept
// (bucket_own_kernel + bucket_keep_kernel); the attention over sink, window,
// the kept 4-key runs and the new tokens is the decode attention kernel in
// run mode.
//
// Readings where the page is open (ties, the last round, the expansion rule)
// are those of the float64 oracle: lower bucket index first on equal cost;
// when merging every mutual pair would leave fewer than b / 8 buckets only
// the cheapest pairs (cost, then indices) merge; buckets are numbered by
// their lowest member; a bucket is a candidate if one of its raw keys lies
// outside sink and window.
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kWardMaxPool = 128;              // pool keys per cluster block (one CTA holds them)
constexpr int kWardRow = 132;                  // floats per coordinate row of the bucket sums
constexpr int kWardCost = kWardMaxPool + 1;    // floats per row of the cost matrix
constexpr int kWardThreads = 512;
constexpr int kWardWarps = kWardThreads / 32;
constexpr int kWardMaxMembers = 16;            // pool keys per bucket at most (16 raw keys, stride 1)
constexpr int kOwnPerCta = 64;                 // expansion entries per CTA of bucket_own_kernel
constexpr int kStageBytes = 131072;            // raw keys staged per bulk copy (inside M and the costs)

typedef unsigned long long u64;

__device__ __forceinline__ u64 pk2(float x, float y) {
  u64 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float lo2(u64 v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(u64 v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Coordinate d of key row `row` (element offset) as fp32.
template <bool BF16>
__device__ __forceinline__ float key_elem(const void* K, int64_t row, int d) {
  if constexpr (BF16) {
    const uint16_t u = __ldg(static_cast<const uint16_t*>(K) + row + d);
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
  } else {
    return __ldg(static_cast<const float*>(K) + row + d);
  }
}

// Sum of `stride` L2-normalised raw keys starting at element offset `row0`
// (rows of 128): this lane's coordinates lane + 32 e, e < 4.
template <bool BF16>
__device__ __forceinline__ void pool_key(const void* K, int64_t row0, int stride, int lane, float (&acc)[4]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int r = 0; r < stride; ++r) {
    const int64_t row = row0 + static_cast<int64_t>(r) * kHeadDim;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = key_elem<BF16>(K, row, lane + 32 * e);
    const float s2 = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float sc = s2 > 0.f ? 1.f / sqrtf(s2) : 0.f;      // normalise(0) = 0
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += x[e] * sc;
  }
}

// The same from raw key rows staged in shared memory (row bytes 128 x el).
template <bool BF16>
__device__ __forceinline__ void pool_key_smem(const unsigned char* row0, int stride, int lane, float (&acc)[4]) {
  constexpr int kRowBytes = kHeadDim * (BF16 ? 2 : 4);
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int r = 0; r < stride; ++r) {
    const unsigned char* row = row0 + r * kRowBytes;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (BF16) {
        x[e] = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(row)[lane + 32 * e]) << 16);
      } else {
        x[e] = reinterpret_cast<const float*>(row)[lane + 32 * e];
      }
    }
    const float s2 = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float sc = s2 > 0.f ? 1.f / sqrtf(s2) : 0.f;      // normalise(0) = 0
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += x[e] * sc;
  }
}

// The normalised index query of `pair`: the sum of its G query heads of the
// first new token, divided by its norm (0 stays 0); coordinates lane + 32 e.
template <bool BF16>
__device__ __forceinline__ void index_query_hat(const void* Q, int64_t pair, int Hkv, int Hq, int G, int n_q,
                                                int lane, float (&qh)[4]) {
  const int64_t bi = pair / Hkv, h = pair % Hkv;
#pragma unroll
  for (int e = 0; e < 4; ++e) qh[e] = 0.f;
  for (int g = 0; g < G; ++g) {
    const int64_t row = ((bi * n_q) * Hq + h * G + g) * kHeadDim;
#pragma unroll
    for (int e = 0; e < 4; ++e) qh[e] += key_elem<BF16>(Q, row, lane + 32 * e);
  }
  const float s2 = warp_sum(qh[0] * qh[0] + qh[1] * qh[1] + qh[2] * qh[2] + qh[3] * qh[3]);
  const float sc = s2 > 0.f ? 1.f / sqrtf(s2) : 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) qh[e] *= sc;
}

// ---- §2.2: Ward clustering of one cluster block --------------------------------
// Shared memory: bucket sums column-major (S[d * kWardRow + i], bucket i's
// coordinate d: a warp reading buckets i..i+127 at one d is conflict-free),
// the full symmetric cost matrix (row stride kWardCost), sizes, reciprocals,
// best partners, the round's pairs and the member lists (local pool-key ids,
// ascending).
template <bool BF16>
__global__ void __launch_bounds__(kWardThreads, 1) ward_kernel(WardArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  float* S = reinterpret_cast<float*>(smem);
  float* M = S + kHeadDim * kWardRow;                      // bucket means, same layout as S
  float* cost = M + kHeadDim * kWardRow;
  float* inv = cost + kWardMaxPool * kWardCost;
  float* bestc = inv + kWardMaxPool;
  float* pc = bestc + kWardMaxPool;                        // [64] pair costs
  int* n = reinterpret_cast<int*>(pc + kWardMaxPool / 2);
  int* best = n + kWardMaxPool;
  int* pa = best + kWardMaxPool;                           // [64]
  int* pb = pa + kWardMaxPool / 2;                         // [64]
  int* keep = pb + kWardMaxPool / 2;                       // [64]
  int* rank = keep + kWardMaxPool / 2;                     // [128]
  int* misc = rank + kWardMaxPool;                         // [8]
  uint8_t* mem = reinterpret_cast<uint8_t*>(misc + 8);     // [128][16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(mem + kWardMaxPool * kWardMaxMembers);
  // the block's raw keys are staged (one or two bulk copies of up to 128 KB)
  // in the space of M and the cost matrix, which are filled only afterwards
  unsigned char* stage = reinterpret_cast<unsigned char*>(M);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pair = blockIdx.y;
  const int64_t blk = a.first_block + blockIdx.x;
  const int m = a.m;

  if (threadIdx.x < kWardMaxPool) {
    const int t = threadIdx.x;
    n[t] = t < m ? 1 : 0;
    inv[t] = 1.f;
    mem[t * kWardMaxMembers] = static_cast<uint8_t>(t);
  }
  // pool keys (§2.2: normalise, sum `stride` consecutive keys) from the
  // staged raw keys
  {
    constexpr int kRowBytes = kHeadDim * (BF16 ? 2 : 4);
    constexpr int kChunkRows = kStageBytes / kRowBytes;              // a multiple of every stride
    if (threadIdx.x == 0) {
      mbar_init(bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    const unsigned char* src = static_cast<const unsigned char*>(a.K) + (pair * a.cap + blk * a.b) * kRowBytes;
    for (int r0 = 0, c = 0; r0 < a.b; r0 += kChunkRows, ++c) {
      const int rows = min(kChunkRows, a.b - r0);
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * kRowBytes);
        bulk_g2s(stage, src + static_cast<int64_t>(r0) * kRowBytes, static_cast<uint32_t>(rows) * kRowBytes, bar);
      }
      const bool ok = mbar_wait_bounded(bar, c & 1, nullptr);
      if (__syncthreads_or(!ok)) {
        // the copy did not land in time: leave this block's buckets empty
        // (members -1) after a last bounded wait for the copy in flight
        if (threadIdx.x == 0) mbar_wait_bounded(bar, c & 1, nullptr);
        int32_t* out = a.members + (pair * a.rows_per_pair + blk * a.nbk) * a.mcap;
        for (int t = threadIdx.x; t < a.nbk * a.mcap; t += kWardThreads) out[t] = -1;
        __syncthreads();
        return;
      }
      for (int i = r0 / a.stride + warp; i < (r0 + rows) / a.stride; i += kWardWarps) {
        float acc[4];
        pool_key_smem<BF16>(stage + (i * a.stride - r0) * kRowBytes, a.stride, lane, acc);
#pragma unroll
        for (int e = 0; e < 4; ++e) S[(lane + 32 * e) * kWardRow + i] = acc[e];
      }
      __syncthreads();                   // the stage is free for the next copy
    }
    for (int item = threadIdx.x; item < kHeadDim * kWardMaxPool; item += kWardThreads) {
      const int d = item >> 7, i = item & (kWardMaxPool - 1);
      M[d * kWardRow + i] = S[d * kWardRow + i];
    }
    __syncthreads();
  }

  // initial costs of singletons (n_a n_b / (n_a + n_b) = 1/2), upper
  // triangle of 4 x 4 bucket tiles, both halves of the matrix written.  Warp w
  // takes the column blocks w (rows 0..w) and 31 - w (rows 0..30 - w), one
  // tile per lane; the 16 diagonal tiles of blocks 16..31 left over are 96
  // single pairs done after.
  {
    const u64 neg1 = pk2(-1.f, -1.f);
    const int ib = lane <= warp ? lane : lane - warp - 1;          // row block
    const int jb = lane <= warp ? warp : 31 - warp;                // column block
    u64 acc[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = 0ull;
#pragma unroll 4
    for (int d = 0; d < kHeadDim; ++d) {
      const float* row = S + d * kWardRow;
      const float4 av = *reinterpret_cast<const float4*>(row + 4 * ib);
      const float4 bv = *reinterpret_cast<const float4*>(row + 4 * jb);
      const u64 b0 = pk2(bv.x, bv.y), b1 = pk2(bv.z, bv.w);
      const float ar[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const u64 a2 = pk2(ar[u], ar[u]);
        const u64 d0 = fma2(b0, neg1, a2), d1 = fma2(b1, neg1, a2);   // a - b, rounded once
        acc[u][0] = fma2(d0, d0, acc[u][0]);
        acc[u][1] = fma2(d1, d1, acc[u][1]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int ra = 4 * ib + u, cb = 4 * jb + v;
        if (ra < cb && cb < m) {
          const float c = 0.5f * ((v & 1) ? hi2(acc[u][v >> 1]) : lo2(acc[u][v >> 1]));
          cost[ra * kWardCost + cb] = c;
          cost[cb * kWardCost + ra] = c;
        }
      }
    if (threadIdx.x < 96) {
      // pairs (u, v), u < v, inside diagonal tile 16 + t / 6
      const int t = threadIdx.x, jd = 16 + t / 6, q = t % 6;
      const int u = q < 3 ? 0 : (q < 5 ? 1 : 2);
      const int v = q < 3 ? q + 1 : (q < 5 ? q - 1 : 3);
      const int ra = 4 * jd + u, cb = 4 * jd + v;
      float s = 0.f;
      for (int d = 0; d < kHeadDim; ++d) {
        const float df = S[d * kWardRow + ra] - S[d * kWardRow + cb];
        s = fmaf(df, df, s);
      }
      if (cb < m) {
        cost[ra * kWardCost + cb] = 0.5f * s;
        cost[cb * kWardCost + ra] = 0.5f * s;
      }
    }
  }

  // rounds of mutual cheapest merges
  int alive = m;
  for (int round = 0; alive > a.nbk && round < m; ++round) {
    __syncthreads();
    {
      // the warp's 8 rows r = warp + 16 j side by side (their reductions
      // overlap); lane l holds candidates 4 l .. 4 l + 3, ascending
      constexpr int kRows = kWardMaxPool / kWardWarps;
      const int4 nn = *reinterpret_cast<const int4*>(n + 4 * lane);
      const int nv[4] = {nn.x, nn.y, nn.z, nn.w};
      float bc[kRows];
      int bi[kRows];
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        const int r = warp + kWardWarps * j;
        const int nr = r < m ? n[r] : 0;
        bc[j] = CUDART_INF_F;
        bi[j] = -1;
        if (nr > 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * lane + e;
            if (c != r && nv[e] > 0 && nr + nv[e] <= a.mcap) {
              const float v = cost[r * kWardCost + c];
              if (v < bc[j]) {
                bc[j] = v;
                bi[j] = c;
              }
            }
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const float ov = __shfl_xor_sync(0xffffffffu, bc[j], o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi[j], o);
          if (oi >= 0 && (bi[j] < 0 || ov < bc[j] || (ov == bc[j] && oi < bi[j]))) {
            bc[j] = ov;
            bi[j] = oi;
          }
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const int r = warp + kWardWarps * j;
          if (r < m && n[r] > 0) {
            best[r] = bi[j];
            bestc[r] = bc[j];
          }
        }
      }
    }
    if (threadIdx.x == 0) misc[0] = 0;
    __syncthreads();
    if (threadIdx.x < m) {
      const int r = threadIdx.x;
      if (n[r] > 0) {
        const int b = best[r];
        if (b > r && best[b] == r) {
          const int sidx = atomicAdd(&misc[0], 1);
          pa[sidx] = r;
          pb[sidx] = b;
          pc[sidx] = bestc[r];
        }
      }
    }
    __syncthreads();
    const int np = misc[0];
    if (np == 0) break;                  // no merge allowed (cannot happen below the bucket target)
    const int need = alive - a.nbk;
    if (threadIdx.x < np) {              // the cheapest `need` pairs: cost, then the lower index
      const int i = threadIdx.x;
      int rk = 0;
      for (int j = 0; j < np; ++j) rk += (pc[j] < pc[i]) || (pc[j] == pc[i] && pa[j] < pa[i]);
      keep[i] = rk < need;
    }
    __syncthreads();
    for (int item = threadIdx.x; item < np * kHeadDim; item += kWardThreads) {
      const int i = item >> 7, d = item & (kHeadDim - 1);
      if (keep[i]) S[d * kWardRow + pa[i]] += S[d * kWardRow + pb[i]];
    }
    if (threadIdx.x < np && keep[threadIdx.x]) {
      const int r = pa[threadIdx.x], c = pb[threadIdx.x];
      const int na = n[r], nb2 = n[c];
      uint8_t merged[kWardMaxMembers];
      int x = 0, y = 0;
      for (int k = 0; k < na + nb2; ++k) {
        const uint8_t va = x < na ? mem[r * kWardMaxMembers + x] : 0xffu;
        const uint8_t vb = y < nb2 ? mem[c * kWardMaxMembers + y] : 0xffu;
        if (va < vb) {
          merged[k] = va;
          ++x;
        } else {
          merged[k] = vb;
          ++y;
        }
      }
      for (int k = 0; k < na + nb2; ++k) mem[r * kWardMaxMembers + k] = merged[k];
      n[r] = na + nb2;
      n[c] = 0;
      inv[r] = 1.f / static_cast<float>(na + nb2);
    }
    __syncthreads();
    for (int item = threadIdx.x; item < np * kHeadDim; item += kWardThreads) {
      const int i = item >> 7, d = item & (kHeadDim - 1);
      if (keep[i]) M[d * kWardRow + pa[i]] = S[d * kWardRow + pa[i]] / static_cast<float>(n[pa[i]]);
    }
    __syncthreads();
    // costs of every merged bucket against every live one from the means
    // (both halves of the symmetric matrix; two merged buckets compute their
    // shared entry twice, to the same value); lane l takes buckets 4 l .. 4 l + 3
    {
      // costs of every merged bucket against every live one from the means
      // (both halves of the symmetric matrix; two merged buckets compute
      // their shared entry twice, to the same value); lane l takes buckets
      // 4 l .. 4 l + 3
      const u64 neg1 = pk2(-1.f, -1.f);
      for (int i = warp; i < np; i += kWardWarps) {
        if (!keep[i]) continue;
        const int r = pa[i];
        const int nr = n[r];
        u64 acc0 = 0ull, acc1 = 0ull;
#pragma unroll 4
        for (int d = 0; d < kHeadDim; ++d) {
          const float* row = M + d * kWardRow;
          const float mr = row[r];
          const float4 mc = *reinterpret_cast<const float4*>(row + 4 * lane);
          const u64 r2 = pk2(mr, mr);
          const u64 d0 = fma2(pk2(mc.x, mc.y), neg1, r2), d1 = fma2(pk2(mc.z, mc.w), neg1, r2);
          acc0 = fma2(d0, d0, acc0);
          acc1 = fma2(d1, d1, acc1);
        }
        const float accv[4] = {lo2(acc0), hi2(acc0), lo2(acc1), hi2(acc1)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * lane + e;
          if (c < m && c != r && n[c] > 0) {
            const float w = static_cast<float>(nr * n[c]) / static_cast<float>(nr + n[c]);
            const float v = w * accv[e];
            cost[r * kWardCost + c] = v;
            cost[c * kWardCost + r] = v;
          }
        }
      }
    }
    alive -= min(np, need);
  }
  __syncthreads();

  // buckets in the order of their lowest member (the slot index)
  if (warp < kWardMaxPool / 32) {
    const int t = threadIdx.x;
    const bool al = t < m && n[t] > 0;
    const unsigned bal = __ballot_sync(0xffffffffu, al);
    if (lane == 0) misc[1 + warp] = __popc(bal);
    rank[t] = al ? __popc(bal & ((1u << lane) - 1u)) : -1;
  }
  __syncthreads();
  if (threadIdx.x < kWardMaxPool && rank[threadIdx.x] >= 0) {
    int base = 0;
    for (int w = 0; w < warp; ++w) base += misc[1 + w];
    rank[threadIdx.x] += base;
  }
  __syncthreads();
  const int64_t row_base = pair * a.rows_per_pair + blk * a.nbk;
  if (threadIdx.x < m && rank[threadIdx.x] >= 0 && rank[threadIdx.x] < a.nbk) {
    const int t = threadIdx.x;
    int32_t* out = a.members + (row_base + rank[t]) * a.mcap;
    for (int k = 0; k < a.mcap; ++k)
      out[k] = k < n[t] ? static_cast<int32_t>(blk * m + mem[t * kWardMaxMembers + k]) : -1;
  }
  for (int t = warp; t < m; t += kWardWarps) {
    if (rank[t] < 0 || rank[t] >= a.nbk) continue;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = S[(lane + 32 * e) * kWardRow + t];
    const float s2 = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
    const float sc = s2 > 0.f ? 1.f / sqrtf(s2) : 0.f;
    float* out = a.cents + (row_base + rank[t]) * kHeadDim;
#pragma unroll
    for (int e = 0; e < 4; ++e) out[lane + 32 * e] = v[e] * sc;
  }
}

// ---- §2.3: centroid scores -----------------------------------------------------
// One warp takes 8 buckets at a time (a lane holds coordinates 4 lane ..
// 4 lane + 3 of the normalised index query and of each centroid row).
template <bool BF16>
__global__ void __launch_bounds__(256) bucket_score_kernel(BucketScoreArgs a) {
  __shared__ __align__(16) float qs[kHeadDim];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pair = blockIdx.y;
  if (warp == 0) {
    float qh[4];
    index_query_hat<BF16>(a.Q, pair, a.Hkv, a.Hq, a.G, a.n_q, lane, qh);
#pragma unroll
    for (int e = 0; e < 4; ++e) qs[lane + 32 * e] = qh[e];
  }
  __syncthreads();
  const float4 q4 = *reinterpret_cast<const float4*>(qs + 4 * lane);
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * a.rows_per_cta;
  const int64_t g1 = min(a.n_bkt, g0 + a.rows_per_cta);
  const float* cbase = a.cents + pair * a.rows_per_pair * kHeadDim;
  uint32_t* keys = a.keys + pair * a.n_bkt;
  for (int64_t base = g0 + warp * 8; base < g1; base += 8 * 8) {
    float dot[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
      if (base + j < g1) c = __ldg(reinterpret_cast<const float4*>(cbase + (base + j) * kHeadDim) + lane);
      dot[j] = q4.x * c.x + q4.y * c.y + q4.z * c.z + q4.w * c.w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) dot[j] = warp_sum(dot[j]);
    if (lane < 8 && base + lane < g1) {
      float mine = dot[0];
#pragma unroll
      for (int j = 1; j < 8; ++j)
        if (lane == j) mine = dot[j];
      const int64_t g = base + lane;
      // candidate: a raw key of the bucket outside sink and window
      const int64_t lo = (g / a.nbk) * a.b, hi = lo + a.b;
      bool cand;
      if (hi <= a.s_end || lo >= a.w_begin) {
        cand = false;
      } else if (lo >= a.s_end && hi <= a.w_begin) {
        cand = true;
      } else {
        cand = false;
        const int32_t* mm = a.members + (pair * a.rows_per_pair + g) * a.mcap;
        for (int k = 0; k < a.mcap; ++k) {
          const int32_t p = __ldg(mm + k);
          if (p < 0) continue;
          const int64_t r0 = static_cast<int64_t>(p) * a.stride, r1 = r0 + a.stride;
          if (max(r0, a.s_end) < min(r1, a.w_begin)) cand = true;
        }
      }
      keys[g] = cand ? float_key(mine) : 0u;
    }
  }
}

// ---- §2.3: top-k buckets -------------------------------------------------------
// Exact top-k of n order-preserving keys held in shared memory by one CTA of
// THREADS threads (key 0 = not a candidate): the k-th largest key tau by four
// 8-bit radix passes (lanes of a warp that fall into one bin add once), then
// the positions of the selected keys in ascending order: every key above
// tau and, of the keys equal to it, the lowest positions (a warp per
// contiguous segment, two scans over the warps).  Writes min(k, candidates)
// positions to out[0..), -1 up to k.
template <int THREADS>
__device__ void smem_topk(const uint32_t* keys, int n, int k, int32_t* out) {
  constexpr int W = THREADS / 32;
  constexpr int HG = 8;                // warps sharing one private histogram
  __shared__ unsigned hist[256];
  __shared__ unsigned phist[W / HG][256];
  __shared__ unsigned wgt[W], weq[W];
  __shared__ unsigned bc[3];     // prefix, keys equal to tau still to take, keff
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  unsigned remaining = 0, keff = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int t = threadIdx.x; t < (W / HG) * 256; t += THREADS) (&phist[0][0])[t] = 0;
    __syncthreads();
    // the scores crowd a few bins of the leading digits: lanes of a warp in
    // one bin add once, and groups of HG warps count into their own copy
    unsigned* my = phist[warp / HG];
    for (int b0 = warp * 32; b0 < n; b0 += THREADS) {
      const int i = b0 + lane;
      const uint32_t key = i < n ? keys[i] : 0u;
      const bool want = key != 0u && (key & pmask) == prefix;
      const unsigned bin = want ? (key >> shift) & 255u : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (want && lane == __ffs(peers) - 1) atomicAdd(&my[bin], static_cast<unsigned>(__popc(peers)));
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      unsigned t = 0;
#pragma unroll
      for (int g = 0; g < W / HG; ++g) t += phist[g][threadIdx.x];
      hist[threadIdx.x] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // bins 8 lane .. 8 lane + 7 per lane; suffix sums from the top
      unsigned c[8], own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[8 * lane + j];
        own += c[j];
      }
      if (pass == 0) {
        const unsigned nc = __reduce_add_sync(0xffffffffu, own);
        keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);
        remaining = keff;
      }
      unsigned above = own;        // sum over lanes >= lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += y;
      }
      const unsigned higher = above - own;
      int digit = -1;
      unsigned cnt_above_digit = 0;
      if (remaining > 0 && higher < remaining && above >= remaining) {
        unsigned acc = higher;
        for (int j = 7; j >= 0; --j) {
          if (acc + c[j] >= remaining) {
            digit = 8 * lane + j;
            cnt_above_digit = acc;
            break;
          }
          acc += c[j];
        }
      }
      const unsigned who = __ballot_sync(0xffffffffu, digit >= 0);
      if (who) {
        const int src = __ffs(who) - 1;
        digit = __shfl_sync(0xffffffffu, digit, src);
        cnt_above_digit = __shfl_sync(0xffffffffu, cnt_above_digit, src);
        if (lane == 0) {
          bc[0] = prefix | (static_cast<uint32_t>(digit) << shift);
          bc[1] = remaining - cnt_above_digit;
          bc[2] = keff;
        }
      } else if (lane == 0) {
        bc[0] = 0u;
        bc[1] = 0u;
        bc[2] = keff;
      }
    }
    __syncthreads();
    prefix = bc[0];
    remaining = bc[1];
    keff = bc[2];
    pmask |= 255u << shift;
    __syncthreads();             // bc is rewritten by the next pass
    if (keff == 0) break;
  }
  const uint32_t tau = prefix;
  const unsigned need = remaining;
  const int seg = (n + W - 1) / W;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  unsigned gt = 0, eq = 0;
  if (keff > 0)
    for (int i = s0 + lane; i < s1; i += 32) {
      const uint32_t key = keys[i];
      gt += key > tau;
      eq += key == tau;
    }
  gt = __reduce_add_sync(0xffffffffu, gt);
  eq = __reduce_add_sync(0xffffffffu, eq);
  if (lane == 0) {
    wgt[warp] = gt;
    weq[warp] = eq;
  }
  __syncthreads();
  if (warp == 0) {
    unsigned g = lane < W ? wgt[lane] : 0u, e = lane < W ? weq[lane] : 0u;
    const unsigned g0 = g, e0 = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned yg = __shfl_up_sync(0xffffffffu, g, o);
      const unsigned ye = __shfl_up_sync(0xffffffffu, e, o);
      if (lane >= o) {
        g += yg;
        e += ye;
      }
    }
    if (lane < W) {
      wgt[lane] = g - g0;
      weq[lane] = e - e0;
    }
  }
  __syncthreads();
  if (keff > 0) {
    unsigned gt_before = wgt[warp], eq_before = weq[warp];
    const unsigned lt = (1u << lane) - 1u;
    for (int b0 = s0; b0 < s1; b0 += 32) {
      const int i = b0 + lane;
      const uint32_t key = i < s1 ? keys[i] : 0u;
      const bool is_gt = i < s1 && key > tau;
      const bool is_eq = i < s1 && key == tau;
      const unsigned bg = __ballot_sync(0xffffffffu, is_gt), be = __ballot_sync(0xffffffffu, is_eq);
      const unsigned my_eq = eq_before + __popc(be & lt);
      if (is_gt || (is_eq && my_eq < need)) out[gt_before + __popc(bg & lt) + min(my_eq, need)] = i;
      gt_before += __popc(bg);
      eq_before += __popc(be);
    }
  }
  for (int i = keff + threadIdx.x; i < k; i += THREADS) out[i] = -1;
  __syncthreads();
}

// First level: the top min(k, 8192) of each chunk of kLocalKeys buckets (one
// CTA per (chunk, pair)).  Every key of the global top-k is among the top-k of
// its own chunk (same order), so the chunks' winners, kept in bucket order,
// are the candidates of the second level.
constexpr int kLocalKeys = kBucketChunk;
constexpr int kLocalThreads = 512;
__global__ void __launch_bounds__(kLocalThreads) bucket_local_topk_kernel(const uint32_t* keys_all, int64_t n, int kl,
                                                                          uint32_t* cand_key, int32_t* cand_id) {
  extern __shared__ __align__(16) uint32_t keys[];         // [kLocalKeys], then the positions
  int32_t* pos = reinterpret_cast<int32_t*>(keys + kLocalKeys);
  const int64_t pair = blockIdx.y;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * kLocalKeys;
  const int64_t left = n - g0;
  const int nl = left < kLocalKeys ? static_cast<int>(left) : kLocalKeys;
  const uint32_t* src = keys_all + pair * n + g0;
  for (int i = threadIdx.x; i < kLocalKeys; i += kLocalThreads) keys[i] = i < nl ? __ldg(src + i) : 0u;
  __syncthreads();
  smem_topk<kLocalThreads>(keys, nl, kl, pos);
  const int64_t ob = (pair * gridDim.x + blockIdx.x) * kl;
  for (int j = threadIdx.x; j < kl; j += kLocalThreads) {
    const int q = pos[j];
    cand_key[ob + j] = q >= 0 ? keys[q] : 0u;
    cand_id[ob + j] = q >= 0 ? static_cast<int32_t>(g0 + q) : -1;
  }
}

// Second level: one CTA per pair selects the top k of its chunks' candidates
// (in shared memory, bucket order), ties to the lower bucket.
constexpr int kSelThreads = 1024;
__global__ void __launch_bounds__(kSelThreads) bucket_select_kernel(const uint32_t* cand_key, const int32_t* cand_id,
                                                                     int nc, int k, int32_t* sel_all) {
  extern __shared__ __align__(16) uint32_t ck[];
  int32_t* pos = reinterpret_cast<int32_t*>(ck + nc);
  const int64_t pair = blockIdx.x;
  for (int i = threadIdx.x; i < nc; i += kSelThreads) ck[i] = __ldg(cand_key + pair * nc + i);
  __syncthreads();
  smem_topk<kSelThreads>(ck, nc, k, pos);
  int32_t* sel = sel_all + pair * static_cast<int64_t>(k);
  for (int j = threadIdx.x; j < k; j += kSelThreads) {
    const int q = pos[j];
    sel[j] = q >= 0 ? __ldg(cand_id + pair * nc + q) : -1;
  }
}

// ---- §2.3: expansion by within-bucket merit ------------------------------------
// Own cosine of every member pool key of the selected buckets: entry e of a
// pair is member e % mcap of selected bucket e / mcap; a warp takes two
// entries at a time.  Writes a 64-bit key per entry: the order-preserving
// cosine above the complemented pool-key id (larger key = better, then the
// lower position), 0 for empty entries.
template <bool BF16>
__global__ void __launch_bounds__(256) bucket_own_kernel(BucketExpandArgs a) {
  __shared__ __align__(16) float qs[kHeadDim];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pair = blockIdx.y;
  if (warp == 0) {
    float qh[4];
    index_query_hat<BF16>(a.Q, pair, a.Hkv, a.Hq, a.G, a.n_q, lane, qh);
#pragma unroll
    for (int e = 0; e < 4; ++e) qs[lane + 32 * e] = qh[e];
  }
  __syncthreads();
  float qh[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) qh[e] = qs[lane + 32 * e];
  const int n_ent = a.top_k * a.mcap;
  const int e0 = blockIdx.x * kOwnPerCta;
  const int e1 = min(n_ent, e0 + kOwnPerCta);
  for (int e = e0 + 2 * warp; e < e1; e += 16) {
    int32_t mm[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      mm[t] = -1;
      if (e + t < e1) {
        const int32_t bk = __ldg(a.sel + pair * a.top_k + (e + t) / a.mcap);
        if (bk >= 0) mm[t] = __ldg(a.members + (pair * a.rows_per_pair + bk) * a.mcap + (e + t) % a.mcap);
      }
    }
    float p[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int64_t m0 = mm[t] < 0 ? 0 : mm[t];
      pool_key<BF16>(a.K, (pair * a.cap + m0 * a.stride) * kHeadDim, mm[t] < 0 ? 0 : a.stride, lane, p[t]);
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float dot = warp_sum(p[t][0] * qh[0] + p[t][1] * qh[1] + p[t][2] * qh[2] + p[t][3] * qh[3]);
      const float s2 = warp_sum(p[t][0] * p[t][0] + p[t][1] * p[t][1] + p[t][2] * p[t][2] + p[t][3] * p[t][3]);
      const float own = s2 > 0.f ? dot / sqrtf(s2) : 0.f;
      if (lane == 0 && e + t < e1)
        a.own[pair * n_ent + e + t] =
            mm[t] < 0 ? 0ull : (static_cast<u64>(float_key(own)) << 32) | static_cast<u64>(~static_cast<uint32_t>(mm[t]));
    }
  }
}

// Bitonic sort of n (a power of two) 64-bit keys in shared memory, descending.
__device__ void bitonic_desc(u64* v, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const u64 x = v[lo], y = v[hi];
        if ((x < y) == desc) {
          v[lo] = y;
          v[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

// One CTA per pair: the kept pool keys, ascending, -1 padded to kept_cap.
// keep_pool == 0 keeps every member of the selected buckets; else the
// keep_pool entries with the largest keys of bucket_own_kernel.
__global__ void __launch_bounds__(512) bucket_keep_kernel(BucketExpandArgs a) {
  extern __shared__ __align__(16) u64 buf[];
  const int64_t pair = blockIdx.x;
  const int n_ent = a.top_k * a.mcap;
  int L = 1;
  while (L < n_ent) L <<= 1;
  for (int e = threadIdx.x; e < L; e += blockDim.x) {
    u64 v = 0ull;
    if (e < n_ent) {
      if (a.keep_pool > 0) {
        v = a.own[pair * n_ent + e];
      } else {
        const int32_t bk = __ldg(a.sel + pair * a.top_k + e / a.mcap);
        const int32_t mm = bk >= 0 ? __ldg(a.members + (pair * a.rows_per_pair + bk) * a.mcap + e % a.mcap) : -1;
        v = mm < 0 ? 0ull : (1ull << 32) | static_cast<u64>(~static_cast<uint32_t>(mm));
      }
    }
    buf[e] = v;
  }
  bitonic_desc(buf, L);
  // the best keep_pool (or all) entries; their ids, larger key = lower id
  // within equal cosines, re-sorted ascending by id
  const int take = a.keep_pool > 0 ? min(a.keep_pool, n_ent) : n_ent;
  for (int e = threadIdx.x; e < L; e += blockDim.x) {     // each element read and written by one thread
    const u64 v = buf[e];
    buf[e] = (e < take && v != 0ull) ? static_cast<u64>(static_cast<uint32_t>(v)) + 1ull : 0ull;   // ~id + 1
  }
  bitonic_desc(buf, L);                  // descending ~id = ascending id
  int32_t* out = a.kept + pair * a.kept_cap;
  for (int e = threadIdx.x; e < a.kept_cap; e += blockDim.x) {
    const u64 v = e < L ? buf[e] : 0ull;
    out[e] = v == 0ull ? -1 : static_cast<int32_t>(~static_cast<uint32_t>(v - 1ull));
  }
}

}  // namespace

size_t ward_smem_bytes() {
  return sizeof(float) * (2 * kHeadDim * kWardRow + kWardMaxPool * kWardCost + 2 * kWardMaxPool + kWardMaxPool / 2) +
         sizeof(int) * (3 * kWardMaxPool + 3 * (kWardMaxPool / 2) + 8) + kWardMaxPool * kWardMaxMembers +
         sizeof(uint64_t);
}

cudaError_t launch_ward(const WardArgs& a, int pairs, int64_t n_blocks, bool bf16, cudaStream_t s) {
  if (pairs == 0 || n_blocks == 0) return cudaSuccess;
  const size_t smem = ward_smem_bytes();
  auto kern = bf16 ? ward_kernel<true> : ward_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(static_cast<unsigned>(n_blocks), static_cast<unsigned>(pairs)), kWardThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bucket_select(const BucketScoreArgs& sa_, const BucketExpandArgs& ea, int pairs, bool bf16,
                                 cudaStream_t s) {
  if (pairs == 0) return cudaSuccess;
  if (sa_.n_bkt > 0) {
    const int64_t chunks = (sa_.n_bkt + sa_.rows_per_cta - 1) / sa_.rows_per_cta;
    auto sk = bf16 ? bucket_score_kernel<true> : bucket_score_kernel<false>;
    sk<<<dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(pairs)), 256, 0, s>>>(sa_);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (ea.top_k > 0) {
    const int chunks = static_cast<int>((sa_.n_bkt + kLocalKeys - 1) / kLocalKeys);
    const int kl = ea.top_k < kLocalKeys ? ea.top_k : kLocalKeys;
    const int nc = chunks * kl;
    constexpr size_t kLocalSmem = static_cast<size_t>(kLocalKeys) * 8;
    cudaError_t e = cudaFuncSetAttribute(bucket_local_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kLocalSmem));
    if (e != cudaSuccess) return e;
    bucket_local_topk_kernel<<<dim3(chunks, pairs), kLocalThreads, kLocalSmem, s>>>(sa_.keys, sa_.n_bkt, kl,
                                                                                     sa_.cand_key, sa_.cand_id);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = static_cast<size_t>(nc) * 8;     // keys and positions
    e = cudaFuncSetAttribute(bucket_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bucket_select_kernel<<<pairs, kSelThreads, smem, s>>>(sa_.cand_key, sa_.cand_id, nc, ea.top_k, ea.sel);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_bucket_expand(const BucketExpandArgs& a, int pairs, bool bf16, cudaStream_t s) {
  if (pairs == 0 || a.kept_cap == 0) return cudaSuccess;
  const int n_ent = a.top_k * a.mcap;
  if (a.keep_pool > 0 && n_ent > 0) {
    auto ok = bf16 ? bucket_own_kernel<true> : bucket_own_kernel<false>;
    ok<<<dim3((n_ent + kOwnPerCta - 1) / kOwnPerCta, pairs), 256, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  int L = 1;
  while (L < n_ent) L <<= 1;
  bucket_keep_kernel<<<pairs, 512, static_cast<size_t>(L) * 8, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sa
