// Exact top-k selection of block scores by one warp (radix select on
// order-preserving float keys), shared by the decode and prefill selectors.
#pragma once

#include "common.cuh"

namespace sa {

__device__ __forceinline__ unsigned warp_sum(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned warp_exclusive_scan(unsigned v) {
  const int lane = threadIdx.x & 31;
  unsigned x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// Exact top-k of `nb` keys (in shared memory) by ONE warp.  Key 0 marks a
// non-candidate; candidates have keys >= 1 (order-preserving float keys).
// Key j is held by lane j % 32 as element j / 32.  The k-th largest key tau
// is found bit by bit from the most significant bit: tau is the largest value
// with at least k keys >= tau (32 steps of a warp-wide count).  Keys above tau
// are taken, and keys equal to tau in ascending block order until k are taken
// (the lower-index tie rule).  Selected ids are written ascending to
// out[0..k), -1 padded.  PER (keys per lane) bounds nb <= 32 * PER.
template <int PER>
__device__ inline void warp_topk_bits(const uint32_t* keys, int nb, int k, int32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t kr[PER];
  unsigned nc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    kr[i] = j < nb ? keys[j] : 0u;
    nc += kr[i] != 0u;
  }
  nc = __reduce_add_sync(0xffffffffu, nc);
  const unsigned keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);
  uint32_t tau = 0xffffffffu;
  unsigned need = 0;
  if (keff > 0u) {
    uint32_t prefix = 0u;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      unsigned c = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) c += kr[i] >= cand;
      if (__reduce_add_sync(0xffffffffu, c) >= keff) prefix = cand;
    }
    tau = prefix;
    unsigned gt = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) gt += kr[i] > tau;
    need = keff - __reduce_add_sync(0xffffffffu, gt);
  }
  const unsigned lt_mask = (1u << lane) - 1u;
  unsigned base = 0, eq_base = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const bool eq = keff > 0u && kr[i] == tau;
    const unsigned b_eq = __ballot_sync(0xffffffffu, eq);
    const bool take_eq = eq && (eq_base + __popc(b_eq & lt_mask)) < need;
    eq_base += __popc(b_eq);
    const bool sel = (keff > 0u && kr[i] > tau && kr[i] != 0u) || take_eq;
    const unsigned b = __ballot_sync(0xffffffffu, sel);
    if (sel) out[base + __popc(b & lt_mask)] = i * 32 + lane;
    base += __popc(b);
  }
  for (int s = static_cast<int>(keff) + lane; s < k; s += 32) out[s] = -1;
}

// Dispatch on the number of keys per lane; nb <= 2048.
__device__ inline void warp_topk(const uint32_t* keys, int nb, int k, int32_t* out) {
  if (nb <= 256) warp_topk_bits<8>(keys, nb, k, out);
  else if (nb <= 512) warp_topk_bits<16>(keys, nb, k, out);
  else if (nb <= 1024) warp_topk_bits<32>(keys, nb, k, out);
  else warp_topk_bits<64>(keys, nb, k, out);
}

}  // namespace sa
