// Work units of the decode / draft-chunk attention kernels: the key ranges
// of the tiles of one (sequence, KV head) pair, shared by the CUDA-core and
// the tensor-core kernels.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace sa {

// Key ranges of the two tiles of one ring stage (n == 0: empty tile).
struct StageInfo {
  int64_t ks0, ks1;
  int n0, n1;
  int64_t pad;
};

// Key range of tile u (0 <= u < MT) of a pair; nkeys == 0 means empty.  The
// index table holds valid ids or -1 (caller tables are sanitised first).
// COHERENT: the table was written during this launch (read through L2).
template <bool COHERENT = false>
__device__ __forceinline__ void tile_range(const DecodeAttnArgs& a, int64_t pair, int u, int64_t* ks,
                                           int* nk) {
  int64_t s = 0, e = 0;
  const int T = a.tile;
  if (u < a.n_sink_tiles) {
    s = static_cast<int64_t>(u) * T;
    e = min(s + T, a.s_end);
  } else if ((u -= a.n_sink_tiles) < a.idx_stride * a.tpb) {
    const int sl = u / a.tpb, sub = u - sl * a.tpb;
    const int32_t j = COHERENT ? __ldcg(a.idx + pair * a.idx_stride + sl) : __ldg(a.idx + pair * a.idx_stride + sl);
    if (j >= 0) {
      const int64_t lo = max(static_cast<int64_t>(j) * a.b, a.s_end);
      const int64_t hi = min(static_cast<int64_t>(j + 1) * a.b, a.w_begin);
      s = lo + static_cast<int64_t>(sub) * T;
      e = min(s + T, hi);
    }
  } else {
    u -= a.idx_stride * a.tpb;
    s = a.w_begin + static_cast<int64_t>(u) * T;
    e = min(s + T, a.kv_end);
  }
  *ks = s;
  *nk = e > s ? static_cast<int>(e - s) : 0;
}

// ---- tensor-core kernel work order (TcOrder) --------------------------------

// CTA that runs unit u of a list of tot units split evenly over g CTAs.
__device__ __forceinline__ int64_t list_owner(int64_t u, int64_t tot, int g) {
  return ((u + 1) * g - 1) / tot;
}

// CTA c's share of such a list: returns its unit count, *first its first unit.
__device__ __forceinline__ int list_share(int64_t tot, int g, int c, int64_t* first) {
  if (c >= g) {
    *first = 0;
    return 0;
  }
  const int64_t s = tot * c / g, e = tot * (c + 1) / g;
  *first = s;
  return static_cast<int>(e - s);
}

// Runs of a CTA's units: local units [0, nI) are list I from global unit i0,
// [nI, n) list D from global unit d0.  A run is the CTA's consecutive units of
// one pair in one list; the divisions happen once per run.
struct RunCursor {
  int64_t i0, d0, pD0;
  int nI, n, mI, mD;
  int run_start, next_start, ordinal;
  int64_t pair;
  bool in_d;
  __device__ void start(int i) {
    run_start = i;
    if (i < nI) {
      in_d = false;
      pair = (i0 + i) / mI;
      const int64_t e = (pair + 1) * mI - i0;
      next_start = static_cast<int>(e < nI ? e : nI);
    } else {
      in_d = true;
      const int64_t pd = (d0 + (i - nI)) / mD;         // pair index within list D
      pair = pD0 + pd;
      next_start = nI + static_cast<int>((pd + 1) * mD - d0);
    }
  }
  __device__ void init(const TcOrder& o, int64_t i0_, int nI_, int64_t d0_, int n_) {
    i0 = i0_;
    d0 = d0_;
    pD0 = o.pD0;
    nI = nI_;
    n = n_;
    mI = o.mI;
    mD = o.mD;
    ordinal = 0;
    pair = 0;
    in_d = false;
    run_start = 0;
    next_start = 0;
    if (n > 0) start(0);
  }
  // call with i ascending by at most one run at a time, before using unit i
  __device__ void at(int i) {
    if (i >= next_start && i < n) {
      ++ordinal;
      start(next_start);
    }
  }
  __device__ bool first(int i) const { return i == run_start; }
  __device__ bool last(int i) const { return i == n - 1 || i + 1 == next_start; }
};

// Key range of tile e (0 or 1) of local unit i, which lies in the cursor's
// current run (nk == 0: empty).
template <bool COHERENT>
__device__ __forceinline__ void unit_tile(const DecodeAttnArgs& a, const RunCursor& c, int i, int e, int64_t* ks,
                                          int* nk) {
  const TcOrder& o = a.ord;
  const int64_t u = c.in_d ? c.d0 + (i - c.nI) : c.i0 + i;
  const int M = c.in_d ? o.mD : o.mI, nt = c.in_d ? o.ntD : o.ntI;
  const int64_t lp = c.in_d ? c.pair - o.pD0 : c.pair;   // pair index within the list
  const int t = 2 * static_cast<int>(u - lp * M) + e;
  if (t >= nt) {
    *ks = 0;
    *nk = 0;
    return;
  }
  const int tt = t + (c.in_d ? o.dD : (t >= a.n_sink_tiles ? o.dI : 0));
  tile_range<COHERENT>(a, c.pair, tt, ks, nk);
}

// Partial-result slots of `pair`: *n CTAs hold a share of it; *mine is this
// CTA's slot for its run in list D (in_d) or list I.
__device__ __forceinline__ void pair_slots(const TcOrder& o, int64_t pair, bool in_d, int* n, int* mine) {
  int nI = 0, nD = 0;
  int64_t fI = 0, fD = 0;
  if (o.mI > 0 && pair < o.pI) {
    fI = list_owner(pair * o.mI, o.totI, o.gI);
    nI = static_cast<int>(list_owner(pair * o.mI + o.mI - 1, o.totI, o.gI) - fI) + 1;
  }
  if (o.mD > 0 && pair >= o.pD0) {
    const int64_t pd = pair - o.pD0;
    fD = list_owner(pd * o.mD, o.totD, o.gD);
    nD = static_cast<int>(list_owner(pd * o.mD + o.mD - 1, o.totD, o.gD) - fD) + 1;
  }
  *n = nI + nD;
  *mine = in_d ? nI + static_cast<int>(blockIdx.x - fD) : static_cast<int>(blockIdx.x - fI);
}

}  // namespace sa
