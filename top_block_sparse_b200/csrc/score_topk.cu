// Steps 2-3 for decode and draft chunks: GQA-shared block scoring and top-k
// selection with sink / window exclusion.
//
// Scoring (LSA review §2.4 and SparDA "方法": one index query per GQA
// group, here the sum of the group's queries of the first new token):
//   mean pooling: s_j = qbar . Kc_j * scale
//   LSA         : s_j = (qbar / |qbar|) . Kc_j   (cosine, LSA review §2.3)
// Candidates: complete blocks not wholly inside sink [0, s_end) or window
// [w_begin, C) (SparDA "方法": initial + local + top-k blocks).
// Selection: the k largest by (score desc, block id asc), written in
// ascending block order, -1 padded.
//
// Grid (chunks, pairs): every CTA streams a chunk of one pair's compressed
// keys (fp32, 128-bit loads, a warp per row with a shuffle reduction) and
// writes scores; the CTA that finishes last for a pair (atomic ticket, no
// waiting) runs the radix select over the pair's scores.
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;

// Block-wide exclusive scan of one value per thread (kScoreThreads threads).
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* warp_tot,
                                                         unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned t = lane < kScoreWarps ? warp_tot[lane] : 0u;
    unsigned s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kScoreWarps) warp_tot[lane] = s - t;   // exclusive warp offsets
    if (lane == kScoreWarps - 1) *total = s;
  }
  __syncthreads();
  const unsigned r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

// Exact top-k of `nb` keys in shared memory (key 0 = not a candidate;
// candidates have keys >= 1).  Writes ascending block ids to out[0..k).
__device__ void radix_select_write(const uint32_t* keys, int nb, int k, int32_t* out,
                                   unsigned* hist, unsigned* scratch) {
  const int tid = threadIdx.x;
  unsigned* warp_tot = scratch;          // [kScoreWarps]
  unsigned* total = scratch + 16;
  unsigned* bcast = scratch + 20;        // digit, count above

  // number of candidates
  unsigned nc = 0;
  for (int j = tid; j < nb; j += kScoreThreads) nc += keys[j] != 0u;
  block_exclusive_scan(nc, warp_tot, total);
  const unsigned n_cand = *total;
  const unsigned keff = n_cand < static_cast<unsigned>(k) ? n_cand : static_cast<unsigned>(k);

  uint32_t tau = 0u;          // keff-th largest key
  unsigned need = keff;       // how many keys equal to tau are taken
  if (keff > 0u) {
    uint32_t prefix = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kScoreThreads) hist[i] = 0u;
      __syncthreads();
      for (int j = tid; j < nb; j += kScoreThreads) {
        const uint32_t key = keys[j];
        if (key == 0u) continue;
        const bool match = (shift == 24) || ((key ^ prefix) >> (shift + 8)) == 0u;
        if (match) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // lane owns bins [8*lane, 8*lane + 8); find the digit holding the need-th largest
        unsigned own = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) own += hist[8 * tid + q];
        unsigned suf = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          unsigned y = __shfl_down_sync(0xffffffffu, suf, o);
          if (tid + o < 32) suf += y;
        }
        unsigned above = suf - own;    // keys with a digit in a higher lane's bins
        if (above < need && need <= above + own) {
          unsigned c = above;
          for (int q = 7; q >= 0; --q) {
            const unsigned h = hist[8 * tid + q];
            if (c + h >= need) {
              bcast[0] = static_cast<unsigned>(8 * tid + q);
              bcast[1] = c;
              break;
            }
            c += h;
          }
        }
      }
      __syncthreads();
      prefix |= bcast[0] << shift;
      need -= bcast[1];
      __syncthreads();
    }
    tau = prefix;
  }

  // Each thread owns a contiguous run of block ids so that scans follow id order.
  const int per = (nb + kScoreThreads - 1) / kScoreThreads;
  const int j0 = tid * per, j1 = min(nb, j0 + per);
  unsigned eq = 0;
  for (int j = j0; j < j1; ++j) eq += (keff > 0u && keys[j] == tau) ? 1u : 0u;
  unsigned eq_before = block_exclusive_scan(eq, warp_tot, total);
  unsigned sel = 0;
  {
    unsigned e = eq_before;
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = keys[j];
      bool s = false;
      if (keff > 0u && key != 0u) {
        if (key > tau) s = true;
        else if (key == tau) { s = e < need; ++e; }
      }
      sel += s;
    }
  }
  unsigned pos = block_exclusive_scan(sel, warp_tot, total);
  {
    unsigned e = eq_before;
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = keys[j];
      bool s = false;
      if (keff > 0u && key != 0u) {
        if (key > tau) s = true;
        else if (key == tau) { s = e < need; ++e; }
      }
      if (s) out[pos++] = j;
    }
  }
  for (int s = static_cast<int>(keff) + tid; s < k; s += kScoreThreads) out[s] = -1;
}

template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads) score_topk_query0_kernel(ScoreArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);                        // [nb] (last CTA)
  __shared__ __align__(16) float qs[kHeadDim];
  __shared__ unsigned hist[256];
  __shared__ unsigned scratch[32];
  __shared__ int is_last;

  const int pair = blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bi = pair / a.Hkv, h = pair % a.Hkv;

  // index query of the first new token: sum over the GQA group
  if (tid < kHeadDim) {
    float s = 0.f;
    for (int g = 0; g < a.G; ++g) {
      const int64_t off = ((static_cast<int64_t>(bi) * a.n_q + 0) * a.Hq + h * a.G + g) * kHeadDim + tid;
      if constexpr (BF16) s += __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(a.Q)[off]) << 16);
      else s += static_cast<const float*>(a.Q)[off];
    }
    qs[tid] = s;
  }
  __syncthreads();
  if (a.lsa) {
    if (warp == 0) {
      float ss = 0.f;
      for (int i = lane; i < kHeadDim; i += 32) ss += qs[i] * qs[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) scratch[0] = __float_as_uint(ss > 0.f ? rsqrtf(ss) : 0.f);
    }
    __syncthreads();
    const float inv = __uint_as_float(scratch[0]);
    __syncthreads();
    if (tid < kHeadDim) qs[tid] *= inv;
  } else {
    if (tid < kHeadDim) qs[tid] *= a.scale;
  }
  __syncthreads();

  const float4 q4 = reinterpret_cast<const float4*>(qs)[lane];
  const int64_t j_begin = static_cast<int64_t>(chunk) * a.blocks_per_chunk;
  const int64_t j_end = min(a.nb, j_begin + a.blocks_per_chunk);
  const float* kc = a.Kc + static_cast<int64_t>(pair) * a.nb * kHeadDim;
  float* sc = a.scores + static_cast<int64_t>(pair) * a.nb;
  for (int64_t j0 = j_begin + warp * 4; j0 < j_end; j0 += kScoreWarps * 4) {
    float4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      r[u] = (j0 + u < j_end) ? __ldcs(reinterpret_cast<const float4*>(kc + (j0 + u) * kHeadDim) + lane)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    float d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) d[u] = r[u].x * q4.x + r[u].y * q4.y + r[u].z * q4.z + r[u].w * q4.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) d[u] += __shfl_xor_sync(0xffffffffu, d[u], o);
    }
    if (lane < 4 && j0 + lane < j_end)
      sc[j0 + lane] = lane == 0 ? d[0] : lane == 1 ? d[1] : lane == 2 ? d[2] : d[3];
  }

  // ticket: the last CTA of this pair selects
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&a.counters[pair], 1u);
    is_last = (t == static_cast<unsigned>(a.chunks - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (tid == 0) a.counters[pair] = 0u;

  const int nb = static_cast<int>(a.nb);
  for (int j = tid; j < nb; j += kScoreThreads) {
    const int64_t lo = static_cast<int64_t>(j) * a.b, hi = lo + a.b;
    const bool cand = (lo < a.w_begin) && (hi > a.s_end);
    const float s = __ldcg(sc + j);
    uint32_t key = float_key(s);
    keys[j] = cand ? (key == 0u ? 1u : key) : 0u;
  }
  __syncthreads();
  radix_select_write(keys, nb, a.top_k, a.idx + static_cast<int64_t>(pair) * a.top_k, hist, scratch);
}

}  // namespace

cudaError_t launch_score_topk_query0(const ScoreArgs& a, bool bf16, cudaStream_t s) {
  if (a.B * a.Hkv == 0) return cudaSuccess;
  dim3 grid(a.chunks, a.B * a.Hkv), blk(kScoreThreads);
  const size_t smem = align_up(static_cast<size_t>(a.nb) * 4, 16);
  cudaError_t e;
  if (bf16) {
    e = cudaFuncSetAttribute(score_topk_query0_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_topk_query0_kernel<true><<<grid, blk, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(score_topk_query0_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_topk_query0_kernel<false><<<grid, blk, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
