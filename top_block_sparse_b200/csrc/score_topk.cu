// Steps 2-3 for decode and draft chunks: GQA-shared block scoring and top-k
// selection with sink / window exclusion.
//
// Scoring (LSA review §2.4 and SparDA "方法": one index query per GQA
// group, here the sum of the group's queries of the first new token):
//   mean pooling: s_j = qbar . Kc_j * scale
//   LSA         : s_j = (qbar / |qbar|) . Kc_j   (cosine, LSA review §2.3)
// Overlapping compressed keys (SparDA "方法": InfLLM-V2 pools keys into
// overlapping compressed representations, coarse to fine): every window is
// scored the same way and block j takes the max over the windows that share
// a key with it.
// Candidates: complete blocks not wholly inside sink [0, s_end) or window
// [w_begin, C) (SparDA "方法": initial + local + top-k blocks).
// Selection: the k largest by (score desc, block id asc), written in
// ascending block order, -1 padded.
//
// Grid (chunks, pairs), every CTA resident at once (2 per SM): each CTA
// streams a contiguous chunk of one pair's compressed keys (fp32 rows of 512
// bytes) through a 3-stage shared-memory ring of 64-row stages filled by
// cp.async.bulk (the TMA engine keeps far more bytes in flight per SM than
// per-thread loads); a warp scores 8 rows of a stage with a shuffle reduction
// per row.  With one chunk per pair the CTA builds the selection keys in
// shared memory (windows: an atomicMax of the order-preserving key into each
// block they touch) and selects; with several, CTAs write scores and the CTA
// that finishes last for the pair (atomic ticket, no waiting) reads them back
// and selects.
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kStageRows = kScoreRowsPerPass;                 // 64 rows = 32 KB
constexpr int kStageBytes = kStageRows * kHeadDim * 4;
constexpr int kScoreStages = 3;
constexpr int kRowsPerWarp = kStageRows / kScoreWarps;        // 8
constexpr size_t kRingBytes = static_cast<size_t>(kScoreStages) * kStageBytes;

__device__ __forceinline__ uint32_t block_key(const ScoreArgs& a, int64_t j, float s) {
  const int64_t lo = j * a.b, hi = lo + a.b;
  const bool cand = (lo < a.w_begin) && (hi > a.s_end);
  const uint32_t key = float_key(s);
  return cand ? (key == 0u ? 1u : key) : 0u;
}

template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads, 2) score_topk_query0_kernel(ScoreArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;                                           // kScoreStages x 32 KB
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kRingBytes);     // [nb] (selecting CTA)
  __shared__ uint64_t full[kScoreStages];
  __shared__ __align__(16) float qs[kHeadDim];
  __shared__ float qinv;
  __shared__ int is_last;
  __shared__ volatile int abort_flag;

  // the attention kernel launched after this one may take SMs as they drain
  pdl_launch_dependents();

  const int pair = blockIdx.y;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bi = pair / a.Hkv, h = pair % a.Hkv;
  const bool single = a.chunks == 1;

  const bool ovl = a.ov_s > 0;
  const int64_t j_begin = min(a.n_rows, static_cast<int64_t>(chunk) * a.rows_per_chunk);
  const int64_t j_end = min(a.n_rows, j_begin + a.rows_per_chunk);
  const int nrows = static_cast<int>(j_end - j_begin);
  const int nst = (nrows + kStageRows - 1) / kStageRows;
  const float* kc = a.Kc + (static_cast<int64_t>(pair) * a.kc_rows + j_begin) * kHeadDim;
  float* sc = a.scores ? a.scores + static_cast<int64_t>(pair) * a.nb : nullptr;
  float* csc = a.cscores ? a.cscores + static_cast<int64_t>(pair) * a.n_rows : nullptr;

  if (tid == 0) {
    for (int s = 0; s < kScoreStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int st) {
    const int s = st % kScoreStages;
    const int rows = min(kStageRows, nrows - st * kStageRows);
    const uint32_t bytes = static_cast<uint32_t>(rows) * kHeadDim * 4;
    mbar_arrive_expect_tx(&full[s], bytes);
    bulk_g2s(ring + static_cast<size_t>(s) * kStageBytes, kc + static_cast<int64_t>(st) * kStageRows * kHeadDim,
             bytes, &full[s]);
  };
  // the first stages are requested before the index query is formed, so the
  // two latencies overlap
  if (tid == 0)
    for (int st = 0; st < min(kScoreStages, nst); ++st) issue(st);
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
  if (ovl && single)
    for (int64_t j = tid; j < a.nb; j += kScoreThreads) keys[j] = 0u;
  __syncthreads();
  if (a.lsa) {
    if (warp == 0) {
      float ss = 0.f;
      for (int i = lane; i < kHeadDim; i += 32) ss += qs[i] * qs[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) qinv = ss > 0.f ? rsqrtf(ss) : 0.f;
    }
    __syncthreads();
  }
  const float qmul = a.lsa ? qinv : a.scale;
  float4 q4 = reinterpret_cast<const float4*>(qs)[lane];
  q4.x *= qmul;
  q4.y *= qmul;
  q4.z *= qmul;
  q4.w *= qmul;

  bool aborted = false;
  for (int st = 0; st < nst; ++st) {
    const int s = st % kScoreStages;
    const bool ok = mbar_wait_bounded(&full[s], (st / kScoreStages) & 1, &abort_flag);
    if (ok) {
      const float* rows = reinterpret_cast<const float*>(ring + static_cast<size_t>(s) * kStageBytes);
      const int r0 = warp * kRowsPerWarp;
      float d[kRowsPerWarp];
#pragma unroll
      for (int u = 0; u < kRowsPerWarp; ++u) {
        const float4 r = reinterpret_cast<const float4*>(rows + (r0 + u) * kHeadDim)[lane];
        d[u] = r.x * q4.x + r.y * q4.y + r.z * q4.z + r.w * q4.w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int u = 0; u < kRowsPerWarp; ++u) d[u] += __shfl_xor_sync(0xffffffffu, d[u], o);
      }
      float mine = d[0];
#pragma unroll
      for (int u = 1; u < kRowsPerWarp; ++u) mine = (lane == u) ? d[u] : mine;
      const int64_t j = j_begin + static_cast<int64_t>(st) * kStageRows + r0 + lane;
      if (lane < kRowsPerWarp && j < j_end) {
        if (!ovl) {
          if (sc) sc[j] = mine;
          if (single) keys[j] = block_key(a, j, mine);
        } else {
          if (csc) csc[j] = mine;
          if (single) {
            // window j covers keys [j*s, j*s + l): blocks t0/b .. (t0+l-1)/b
            const uint32_t key = float_key(mine);
            const int64_t t0 = j * a.ov_s;
            const int64_t last = min(a.nb - 1, (t0 + a.ov_l - 1) / a.b);
            for (int64_t jb = t0 / a.b; jb <= last; ++jb) atomicMax(&keys[jb], key);
          }
        }
      }
    } else if (lane == 0) {
      report(a.status, kStatusTimeout);
      abort_flag = 1;
    }
    // every warp is done with stage s before it is refilled
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (tid == 0 && st + kScoreStages < nst) issue(st + kScoreStages);
  }
  if (aborted) {
    // do not leave while copies into this CTA's shared memory may be in flight
    if (tid == 0)
      for (int st = 0; st < nst; ++st) mbar_wait_bounded(&full[st % kScoreStages], (st / kScoreStages) & 1, nullptr);
    return;
  }

  if (!single) {
    // ticket: the last CTA of this pair selects.  The barrier orders the
    // CTA's score stores before thread 0's release fence.
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned t = atomicAdd(&a.counters[pair], 1u);
      is_last = (t == static_cast<unsigned>(a.chunks - 1));
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (tid == 0) a.counters[pair] = 0u;
    // the pair's scores come back from L2
    if (!ovl) {
      for (int64_t j = tid; j < a.nb; j += kScoreThreads) keys[j] = block_key(a, j, __ldcg(sc + j));
    } else {
      // block j: windows c_lo = ceil((jb - l + 1) / s) .. c_hi = ((j+1)b - 1) / s
      for (int64_t j = tid; j < a.nb; j += kScoreThreads) {
        const int64_t lo = j * a.b - a.ov_l + 1;
        const int64_t c_lo = lo <= 0 ? 0 : (lo + a.ov_s - 1) / a.ov_s;
        const int64_t c_hi = min(a.n_rows - 1, ((j + 1) * a.b - 1) / a.ov_s);
        float m = -CUDART_INF_F;
        for (int64_t c = c_lo; c <= c_hi; ++c) m = fmaxf(m, __ldcg(csc + c));
        if (sc) sc[j] = m;
        keys[j] = block_key(a, j, m);
      }
    }
  } else if (ovl) {
    __syncthreads();
    for (int64_t j = tid; j < a.nb; j += kScoreThreads) {
      const float m = key_float(keys[j]);
      if (sc) sc[j] = m;
      keys[j] = block_key(a, j, m);
    }
  }
  __syncthreads();
  const int nb = static_cast<int>(a.nb);
  int32_t* out = a.idx + static_cast<int64_t>(pair) * a.top_k;
  // the ring is idle now: its first words hold the selection's histograms
  unsigned* scratch = reinterpret_cast<unsigned*>(ring);
  // keys per thread sized to the table (the radix passes loop over them)
  if (nb <= kScoreThreads) block_radix_topk<1>(keys, nb, a.top_k, out, scratch);
  else if (nb <= 2 * kScoreThreads) block_radix_topk<2>(keys, nb, a.top_k, out, scratch);
  else if (nb <= 2048) block_radix_topk<2048 / kScoreThreads>(keys, nb, a.top_k, out, scratch);
  else block_radix_topk<kMaxSelectBlocks / kScoreThreads>(keys, nb, a.top_k, out, scratch);
}

}  // namespace

cudaError_t launch_score_topk_query0(const ScoreArgs& a, bool bf16, cudaStream_t s) {
  if (a.B * a.Hkv == 0) return cudaSuccess;
  dim3 grid(a.chunks, a.B * a.Hkv), blk(kScoreThreads);
  const size_t smem = kRingBytes + align_up(static_cast<size_t>(a.nb) * 4, 16);
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
