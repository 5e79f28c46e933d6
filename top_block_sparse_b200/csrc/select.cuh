// Exact top-k selection of block scores by one warp (radix select on
// order-preserving float keys), shared by the decode and prefill selectors.
#pragma once

#include "common.cuh"

namespace sa {

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
// warp_topk_regs takes the keys in registers (0 also past nb);
// warp_topk_bits loads them from shared memory first.
template <int PER>
__device__ inline void warp_topk_regs(const uint32_t (&kr)[PER], int k, int32_t* out) {
  const int lane = threadIdx.x & 31;
  unsigned nc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) nc += kr[i] != 0u;
  nc = __reduce_add_sync(0xffffffffu, nc);
  const unsigned keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);
  uint32_t tau = 0xffffffffu;
  unsigned need = 0;
  if (keff > 0u) {
    // tau = the largest value with at least keff keys >= tau.  When some
    // prefix already has exactly keff keys at or above it, those keys are the
    // selection: stop there (tau = prefix - 1, nothing taken at equality).
    uint32_t prefix = 0u;
    bool exact = false;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      unsigned c = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) c += kr[i] >= cand;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= keff) prefix = cand;
      if (c == keff) {
        exact = true;
        break;
      }
    }
    if (exact) {
      tau = prefix - 1u;            // prefix >= 1: it has a bit set
      need = 0u;
    } else {
      tau = prefix;
      unsigned gt = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) gt += kr[i] > tau;
      need = keff - __reduce_add_sync(0xffffffffu, gt);
    }
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

template <int PER>
__device__ inline void warp_topk_bits(const uint32_t* keys, int nb, int k, int32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t kr[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    kr[i] = j < nb ? keys[j] : 0u;
  }
  warp_topk_regs<PER>(kr, k, out);
}

// The same selection for any nb, by one warp, with the keys left in shared
// memory (every step of the search re-reads them).
__device__ inline void warp_topk_smem(const uint32_t* keys, int nb, int k, int32_t* out) {
  const int lane = threadIdx.x & 31;
  unsigned nc = 0;
  for (int j = lane; j < nb; j += 32) nc += keys[j] != 0u;
  nc = __reduce_add_sync(0xffffffffu, nc);
  const unsigned keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);
  uint32_t tau = 0xffffffffu;
  unsigned need = 0;
  if (keff > 0u) {
    uint32_t prefix = 0u;
    bool exact = false;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      unsigned c = 0;
#pragma unroll 4
      for (int j = lane; j < nb; j += 32) c += keys[j] >= cand;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= keff) prefix = cand;
      if (c == keff) {
        exact = true;
        break;
      }
    }
    if (exact) {
      tau = prefix - 1u;
      need = 0u;
    } else {
      tau = prefix;
      unsigned gt = 0;
      for (int j = lane; j < nb; j += 32) gt += keys[j] > tau;
      need = keff - __reduce_add_sync(0xffffffffu, gt);
    }
  }
  const unsigned lt_mask = (1u << lane) - 1u;
  unsigned base = 0, eq_base = 0;
  if (keff > 0u) {
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < nb ? keys[j] : 0u;
      const bool eq = key == tau;
      const unsigned b_eq = __ballot_sync(0xffffffffu, eq);
      const bool take_eq = eq && (eq_base + __popc(b_eq & lt_mask)) < need;
      eq_base += __popc(b_eq);
      const bool sel = (key > tau) || take_eq;
      const unsigned b = __ballot_sync(0xffffffffu, sel);
      if (sel) out[base + __popc(b & lt_mask)] = j;
      base += __popc(b);
    }
  }
  for (int s = static_cast<int>(keff) + lane; s < k; s += 32) out[s] = -1;
}

// Dispatch on the number of keys per lane: registers up to 2048 keys, shared
// memory beyond.
__device__ inline void warp_topk(const uint32_t* keys, int nb, int k, int32_t* out) {
  if (nb <= 256) warp_topk_bits<8>(keys, nb, k, out);
  else if (nb <= 512) warp_topk_bits<16>(keys, nb, k, out);
  else if (nb <= 1024) warp_topk_bits<32>(keys, nb, k, out);
  else if (nb <= 2048) warp_topk_bits<64>(keys, nb, k, out);
  else warp_topk_smem(keys, nb, k, out);
}

// Ascending ids of the keys above tau plus the first `need` keys equal to
// tau (lowest ids first), -1 padded to k; the CTA's keys are in registers
// (thread t holds keys t, t + NT, ...).  The keys array (nb words) is reused
// for two bitmaps: the 32 keys of word w sit in one warp's lanes, so a ballot
// builds the word; warp 0 then turns the bitmaps into ids.  Every thread must
// call it after a barrier that follows its last read of `keys`.
template <int NT, int PER>
__device__ inline void block_emit(const uint32_t (&kr)[PER], uint32_t* keys, int nb, int k, unsigned keff,
                                  uint32_t tau, unsigned need, int32_t* out) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = (nb + 31) / 32;
  uint32_t* gbits = keys;
  uint32_t* ebits = keys + W;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int w = i * NW + warp;
    const unsigned g = __ballot_sync(0xffffffffu, keff > 0u && kr[i] > tau);
    const unsigned e = __ballot_sync(0xffffffffu, keff > 0u && kr[i] == tau);
    if (lane == 0 && w < W) {
      gbits[w] = g;
      ebits[w] = e;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  // lane l owns words [l * WL, (l + 1) * WL)
  const int WL = (W + 31) / 32;
  const int w0 = min(W, lane * WL), w1 = min(W, w0 + WL);
  unsigned eq_cnt = 0;
  for (int w = w0; w < w1; ++w) eq_cnt += __popc(ebits[w]);
  unsigned eq_before = warp_exclusive_scan(eq_cnt);
  unsigned n_sel = 0;
  for (int w = w0; w < w1; ++w) {
    unsigned e = ebits[w];
    unsigned take = 0u;
    while (e && eq_before < need) {
      const unsigned low = e & (0u - e);
      take |= low;
      e ^= low;
      ++eq_before;
    }
    eq_before += __popc(e);
    const unsigned sel = gbits[w] | take;
    gbits[w] = sel;
    n_sel += __popc(sel);
  }
  unsigned pos = warp_exclusive_scan(n_sel);
  for (int w = w0; w < w1; ++w) {
    unsigned m = gbits[w];
    while (m) {
      const int b = __ffs(m) - 1;
      out[pos++] = w * 32 + b;
      m &= m - 1u;
    }
  }
  for (int s = static_cast<int>(keff) + lane; s < k; s += 32) out[s] = -1;
}

// Exact top-k of nb <= 256 * PER keys (in shared memory) by a whole CTA of
// 256 threads, with the rules of warp_topk_bits and an 8-bit radix search for
// tau: four passes, each a histogram of the next 8 bits of the keys that
// still agree with tau on the bits above (one private histogram per warp,
// then one bin per thread), and a suffix scan over the 256 bins that picks
// the digit holding the k-th largest.  `scratch` is NW * 256 + NW + 4 words
// of shared memory (not the keys array).
template <int PER>
__device__ inline void block_radix_topk(uint32_t* keys, int nb, int k, int32_t* out, unsigned* scratch) {
  constexpr int NT = 256, NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned* hist = scratch;                 // [NW][256]
  unsigned* wtot = scratch + NW * 256;      // [NW]
  unsigned* ctl = wtot + NW;                // digit, need
  uint32_t kr[PER];
  unsigned nc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * NT + tid;
    kr[i] = j < nb ? keys[j] : 0u;
    nc += kr[i] != 0u;
  }
  nc = __reduce_add_sync(0xffffffffu, nc);
  if (lane == 0) wtot[warp] = nc;
  __syncthreads();
  nc = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) nc += wtot[w];
  const unsigned keff = nc < static_cast<unsigned>(k) ? nc : static_cast<unsigned>(k);
  uint32_t prefix = 0u, pmask = 0u;
  unsigned need = keff;
  if (keff > 0u) {
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      __syncthreads();                      // the previous pass has read hist, wtot and ctl
#pragma unroll
      for (int w = 0; w < NW; ++w) hist[w * 256 + tid] = 0u;
      __syncthreads();
      unsigned* my = hist + warp * 256;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (kr[i] != 0u && (kr[i] & pmask) == prefix) atomicAdd(&my[(kr[i] >> shift) & 255u], 1u);
      __syncthreads();
      // thread t takes bin b = 255 - t, so a prefix scan over t counts the
      // keys whose digit is >= b
      const int b = 255 - tid;
      unsigned hb = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) hb += hist[w * 256 + b];
      unsigned x = hb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) wtot[warp] = x;
      __syncthreads();
      unsigned off = 0;
      for (int w = 0; w < warp; ++w) off += wtot[w];
      const unsigned incl = x + off, excl = incl - hb;
      if (hb > 0u && excl < need && incl >= need) {
        ctl[0] = static_cast<unsigned>(b);
        ctl[1] = need - excl;
      }
      __syncthreads();
      prefix |= ctl[0] << shift;
      pmask |= 255u << shift;
      need = ctl[1];
    }
  }
  const uint32_t tau = keff > 0u ? prefix : 0xffffffffu;
  if (keff == 0u) need = 0u;
  block_emit<NT, PER>(kr, keys, nb, k, keff, tau, need, out);
}

}  // namespace sa
