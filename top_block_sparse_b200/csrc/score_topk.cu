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
#include "select.cuh"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;

template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads) score_topk_query0_kernel(ScoreArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);                        // [nb] (last CTA)
  __shared__ __align__(16) float qs[kHeadDim];
  __shared__ unsigned hist[256];
  __shared__ unsigned scratch[4];
  __shared__ int is_last;

  const int pair = blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bi = pair / a.Hkv, h = pair % a.Hkv;

  static_assert(kScoreBlocksPerChunk % kScoreWarps == 0 && kScoreBlocksPerChunk / kScoreWarps <= 32,
                "rows per warp");
  const int64_t j_begin = static_cast<int64_t>(chunk) * a.blocks_per_chunk;
  const int64_t j_end = min(a.nb, j_begin + a.blocks_per_chunk);
  const float* kc = a.Kc + static_cast<int64_t>(pair) * a.nb * kHeadDim;
  float* sc = a.scores + static_cast<int64_t>(pair) * a.nb;
  // every warp streams kRowsPerWarp rows; their loads are issued first, before
  // the index query is formed, so the two latencies overlap
  constexpr int kRowsPerWarp = kScoreBlocksPerChunk / kScoreWarps;
  const int64_t jw = j_begin + static_cast<int64_t>(warp) * kRowsPerWarp;
  float4 r[kRowsPerWarp];
#pragma unroll
  for (int u = 0; u < kRowsPerWarp; ++u)
    r[u] = (jw + u < j_end) ? __ldcs(reinterpret_cast<const float4*>(kc + (jw + u) * kHeadDim) + lane)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
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
  float d[kRowsPerWarp];
#pragma unroll
  for (int u = 0; u < kRowsPerWarp; ++u) d[u] = r[u].x * q4.x + r[u].y * q4.y + r[u].z * q4.z + r[u].w * q4.w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int u = 0; u < kRowsPerWarp; ++u) d[u] += __shfl_xor_sync(0xffffffffu, d[u], o);
  }
  float mine = d[0];
#pragma unroll
  for (int u = 1; u < kRowsPerWarp; ++u) mine = (lane == u) ? d[u] : mine;
  if (lane < kRowsPerWarp && jw + lane < j_end) sc[jw + lane] = mine;

  // ticket: the last CTA of this pair selects (one warp; the others leave).
  // The barrier orders the CTA's score stores before thread 0's release fence.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&a.counters[pair], 1u);
    is_last = (t == static_cast<unsigned>(a.chunks - 1));
  }
  __syncthreads();
  if (!is_last || warp != 0) return;
  __threadfence();
  if (lane == 0) a.counters[pair] = 0u;

  const int nb = static_cast<int>(a.nb);
  // the pair's scores come from L2; keep 8 loads per lane in flight
  for (int j0 = 0; j0 < nb; j0 += 8 * 32) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      v[u] = j < nb ? __ldcg(sc + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < nb) {
        const int64_t lo = static_cast<int64_t>(j) * a.b, hi = lo + a.b;
        const bool cand = (lo < a.w_begin) && (hi > a.s_end);
        const uint32_t key = float_key(v[u]);
        keys[j] = cand ? (key == 0u ? 1u : key) : 0u;
      }
    }
  }
  __syncwarp();
  warp_topk(keys, nb, a.top_k, a.idx + static_cast<int64_t>(pair) * a.top_k);
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
