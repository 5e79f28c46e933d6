// Dense verify of a draft chunk: the attention mass of each complete
// context block and the block selection it refreshes (S3R review, section
// "稠密验证": one causal forward of the chunk over the dense cache, whose
// attention weights refresh the subset the drafts read; section "稀疏起草",
// KV-selection formula: recent window plus the top-K positions by those
// scores).
//
//   mass[pair][j] = sum over the pair's rows r (chunk tokens x query heads of
//                   the KV head) and the keys t of block j of
//                   exp(q_r . k_t * scale - lse_r)
//
// The dense attention is the decode attention kernel with the whole context
// as its window; its dense-verify instantiation also stores, for every
// 32-key half-tile of the complete blocks and every row, the sum of the
// row's probabilities 2^(x - m) and the running max m they were taken
// against.  Once lse is known, mass_finalize_kernel turns those into block
// masses (sum of part.sum * 2^(part.m - lse * log2 e)), so K and V are read
// once; mass_topk_kernel then takes each pair's top-k candidates by mass.
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace sa {
namespace {

// Block masses from the half-tile partial sums: one CTA per (pair, run of
// blocks), the pair's lse rows in shared memory.
__global__ void __launch_bounds__(128) mass_finalize_kernel(const float2* __restrict__ part,
                                                            const float* __restrict__ lse, float* __restrict__ mass,
                                                            int Hkv, int G, int n_q, int nb, int hpb) {
  __shared__ float l2[16];
  const int pair = blockIdx.y;
  const int bi = pair / Hkv, h = pair - bi * Hkv;
  const int R = n_q * G, Hq = Hkv * G;
  if (threadIdx.x < 16) {
    const int r = threadIdx.x;
    l2[r] = r < R ? lse[(static_cast<int64_t>(bi) * n_q + r / G) * Hq + h * G + r % G] * 1.4426950408889634f
                  : CUDART_INF_F;
  }
  __syncthreads();
  const int64_t hts = static_cast<int64_t>(nb) * hpb;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < nb; j += gridDim.x * blockDim.x) {
    float m = 0.f;
    for (int hh = 0; hh < hpb; ++hh) {
      const float2* pp = part + (pair * hts + static_cast<int64_t>(j) * hpb + hh) * 16;
      for (int r = 0; r < R; ++r) {
        const float2 v = __ldg(pp + r);
        m += v.x * exp2f(v.y - l2[r]);
      }
    }
    mass[static_cast<int64_t>(pair) * nb + j] = m;
  }
}

// Top-k of each pair's candidate blocks by mass (ties: lower block first),
// ascending ids, -1 padded: one warp per pair, keys in shared memory.
__global__ void __launch_bounds__(32) mass_topk_kernel(const float* __restrict__ mass, int nb, int b,
                                                       int64_t s_end, int64_t w_begin, int k,
                                                       int32_t* __restrict__ idx) {
  extern __shared__ uint32_t keys[];
  const int pair = blockIdx.x;
  const float* m = mass + static_cast<int64_t>(pair) * nb;
  for (int j = threadIdx.x; j < nb; j += 32) {
    const int64_t lo = static_cast<int64_t>(j) * b, hi = lo + b;
    const uint32_t key = float_key(__ldg(m + j));
    keys[j] = (lo < w_begin && hi > s_end) ? (key == 0u ? 1u : key) : 0u;
  }
  __syncwarp();
  warp_topk(keys, nb, k, idx + static_cast<int64_t>(pair) * k);
}

}  // namespace

cudaError_t launch_mass_finalize(const float2* part, const float* lse, float* mass, int B, int Hkv, int G, int n_q,
                                 int nb, int b, cudaStream_t s) {
  if (nb == 0 || B * Hkv == 0) return cudaSuccess;
  const dim3 grid((nb + 127) / 128, B * Hkv);
  mass_finalize_kernel<<<grid, 128, 0, s>>>(part, lse, mass, Hkv, G, n_q, nb, b / 32);
  return cudaGetLastError();
}

cudaError_t launch_mass_topk(const float* mass, int pairs, int nb, int b, int64_t s_end, int64_t w_begin, int k,
                             int32_t* idx, cudaStream_t s) {
  if (pairs == 0 || k == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(nb > 0 ? nb : 1) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(mass_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  mass_topk_kernel<<<pairs, 32, smem, s>>>(mass, nb, b, s_end, w_begin, k, idx);
  return cudaGetLastError();
}

}  // namespace sa
