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

// Exact top-k of `nb` keys in shared memory by ONE warp (key 0 = not a
// candidate, candidates have keys >= 1): a 4-pass, 8-bit-digit radix select
// finds the k-th largest key tau and how many keys equal to tau are taken
// (the lowest block ids first); a prefix scan in block-id order then writes
// the selected ids ascending to out[0..k), -1 padded.
__device__ inline void warp_radix_select(const uint32_t* keys, int nb, int k, int32_t* out, unsigned* hist) {
  const int lane = threadIdx.x & 31;
  unsigned nc = 0;
#pragma unroll 8
  for (int j = lane; j < nb; j += 32) nc += keys[j] != 0u;
  nc = warp_sum(nc);
  const unsigned keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);

  uint32_t tau = 0u;          // keff-th largest key
  unsigned need = keff;       // keys equal to tau that are taken
  if (keff > 0u) {
    uint32_t prefix = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[lane + 32 * i] = 0u;
      __syncwarp();
      // scores cluster in a few digit values (sign and exponent bits first), so
      // lanes with equal digits are merged and one of them adds their count
#pragma unroll 8
      for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < nb ? keys[j] : 0u;
        const bool take = key != 0u && (shift == 24 || ((key ^ prefix) >> (shift + 8)) == 0u);
        const unsigned digit = take ? ((key >> shift) & 255u) : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, digit);
        if (take && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], static_cast<unsigned>(__popc(peers)));
      }
      __syncwarp();
      // lane owns bins [8*lane, 8*lane + 8): find the digit holding the need-th largest
      unsigned h8[8], own = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        h8[q] = hist[8 * lane + q];
        own += h8[q];
      }
      unsigned suf = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
      }
      const unsigned above = suf - own;          // keys in higher lanes' bins
      unsigned digit = 0, cnt_above = 0;
      const bool mine = above < need && need <= above + own;
      if (mine) {
        unsigned c = above;
        bool found = false;
#pragma unroll
        for (int q = 7; q >= 0; --q) {
          if (!found && c + h8[q] >= need) {
            digit = static_cast<unsigned>(8 * lane + q);
            cnt_above = c;
            found = true;
          }
          c += h8[q];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      digit = __shfl_sync(0xffffffffu, digit, src);
      cnt_above = __shfl_sync(0xffffffffu, cnt_above, src);
      prefix |= digit << shift;
      need -= cnt_above;
      __syncwarp();
    }
    tau = prefix;
  }

  // Each lane owns a contiguous run of block ids so that scans follow id order.
  const int per = (nb + 31) / 32;
  const int j0 = lane * per, j1 = min(nb, j0 + per);
  unsigned eq = 0;
  if (keff > 0u) {
#pragma unroll 8
    for (int j = j0; j < j1; ++j) eq += keys[j] == tau;
  }
  const unsigned eq_before = warp_exclusive_scan(eq);
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
  unsigned pos = warp_exclusive_scan(sel);
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
  for (int s = static_cast<int>(keff) + lane; s < k; s += 32) out[s] = -1;
}

}  // namespace sa
