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

}  // namespace sa
