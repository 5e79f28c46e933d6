// Dense verify of a draft chunk: the attention mass of each complete
// context block and the block selection it refreshes (S3R review, section
// "稠密验证": one causal forward of the chunk over the dense cache, whose
// attention weights refresh the subset the drafts read; section "稀疏起草",
// KV-selection formula: recent window plus the top-K positions by those
// scores).  The dense attention itself (O, lse) is the decode attention
// kernel with the whole context as its window; this file adds, once lse is
// known,
//
//   mass[pair][j] = sum over the pair's rows r (chunk tokens x query heads of
//                   the KV head) and the keys t of block j of
//                   exp(q_r . k_t * scale - lse_r)
//
// and the top-k of the candidate blocks by mass.
//
// block_mass_kernel: one CTA per run of 128-key units of one pair.  Warp 0
// loads the pair's R <= 16 query rows (one 3-D box per d-half) and streams K
// (two 64-row boxes per d-half, 128-byte swizzle) through a 3-stage ring of
// 32 KB; warp 1 owns 32 TMEM columns and issues S^T = K Q^T (M 128 keys x N
// 16 rows x K 128) into one of two 16-column buffers; warps 2-5 (one key per
// thread, TMEM lane = key) read the unit's S rows, sum exp2(s * scale*log2e
// - lse_r*log2e) over the rows, reduce each 64-key tile over its two warps
// and add it to its block.  Keys of complete blocks precede the chunk, so
// every row sees them: no mask.  V is never read.  All waits are bounded.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace sa {
namespace {

constexpr int kVN = 16;                          // query rows on the MMA N axis
constexpr int kVHalf = 16384;                    // one d-half of a unit: 128 keys x 128 B
constexpr int kVStage = 2 * kVHalf;              // K only
constexpr int kVNS = 3;                          // ring stages
constexpr int kVQBuf = 2 * kVN * 128;            // two d-halves of 16 rows x 128 B
constexpr int kVThreads = 192;
constexpr int kVReduceThreads = 128;
constexpr uint32_t kVIdescS = tc::idesc_bf16(128, kVN, false, false);
constexpr size_t kVSmemBytes = 1024 + static_cast<size_t>(kVNS) * kVStage + kVQBuf + 256;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void reduce_bar() {
  asm volatile("bar.sync 1, %0;" ::"r"(kVReduceThreads) : "memory");
}
// The same barrier, returning whether any of the four warps passed true (a
// wait that gave up in one warp ends the loop in all of them).
__device__ __forceinline__ bool reduce_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(kVReduceThreads)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kVThreads, 1)
    block_mass_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                      BlockMassArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;                                   // kVNS x 32 KB
  unsigned char* Qs = ring + kVNS * kVStage;                    // 4 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(Qs + kVQBuf);
  uint64_t* kv_full = bars;                                     // [3]
  uint64_t* kv_empty = bars + 3;                                // [3]
  uint64_t* q_full = bars + 6;
  uint64_t* s_full = bars + 7;                                  // [2]
  uint64_t* s_free = bars + 9;                                  // [2]
  uint64_t* mma_done = bars + 11;
  float* red = reinterpret_cast<float*>(bars + 12);             // [2 units][4 warps]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = static_cast<int>(blockIdx.x / a.cpp);
  const int chunk = static_cast<int>(blockIdx.x - static_cast<int64_t>(pair) * a.cpp);
  const int u0 = chunk * a.upc;
  const int nunits = min(a.units, u0 + a.upc) - u0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kVNS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kVReduceThreads);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  {
    // Q rows past R only feed MMA columns that are never read; clear once
    uint4* q = reinterpret_cast<uint4*>(Qs);
    for (int i = threadIdx.x; i < kVQBuf / 16; i += kVThreads) q[i] = make_uint4(0u, 0u, 0u, 0u);
    tc::fence_proxy_async_smem();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 32);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  auto fail = [&]() {
    report(a.status, kStatusTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nunits > 0) {
      const int bi = pair / a.Hkv, h = pair - bi * a.Hkv;
      mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(2 * a.R * 128));
      tc::tma_load_3d(Qs, &q_map, 0, h * a.G, bi * a.n_q, q_full);
      tc::tma_load_3d(Qs + kVN * 128, &q_map, 64, h * a.G, bi * a.n_q, q_full);
      int i = 0;
      for (; i < nunits; ++i) {
        const int s = i % kVNS;
        if (i >= kVNS && !mbar_wait_bounded(&kv_empty[s], ((i / kVNS) & 1) ^ 1, abort_flag)) {
          fail();
          break;
        }
        unsigned char* st = ring + s * kVStage;
        mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(kVStage));
        for (int e = 0; e < 2; ++e) {
          // tile 2u + e; past the complete blocks: a box past the map, zeros
          const int tile = 2 * (u0 + i) + e;
          const int row = tile < a.tiles ? tile * 64 : static_cast<int>(a.kv_end);
          tc::tma_load_3d(st + e * 8192, &k_map, 0, row, pair, &kv_full[s]);
          tc::tma_load_3d(st + kVHalf + e * 8192, &k_map, 64, row, pair, &kv_full[s]);
        }
      }
      // do not leave while copies into shared memory may be in flight
      for (int r = max(0, i - kVNS); r < i; ++r) mbar_wait_bounded(&kv_full[r % kVNS], (r / kVNS) & 1, nullptr);
      mbar_wait_bounded(q_full, 0, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t ring_a = smem_u32(ring), qa = smem_u32(Qs);
    bool ok = nunits == 0 || mbar_wait_warp(q_full, 0, abort_flag);
    for (int i = 0; i < nunits && ok; ++i) {
      const int s = i % kVNS;
      ok = mbar_wait_warp(&kv_full[s], (i / kVNS) & 1, abort_flag) &&
           (i < 2 || mbar_wait_warp(&s_free[i & 1], ((i >> 1) + 1) & 1, abort_flag));
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t kst = ring_a + s * kVStage;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_bf16_elect(tbase + (i & 1) * kVN, tc::smem_desc(kst + (kk >> 2) * kVHalf + (kk & 3) * 32, 16, 1024),
                           tc::smem_desc(qa + (kk >> 2) * (kVN * 128) + (kk & 3) * 32, 16, 1024), kVIdescS, kk > 0);
      tc::mma_commit_elect(&s_full[i & 1]);
      tc::mma_commit_elect(&kv_empty[s]);
    }
    if (!ok && lane == 0) fail();
    tc::mma_commit_elect(mma_done);
    mbar_wait_warp(mma_done, 0, nullptr);
    __syncwarp();
  } else {
    // ---------------------------------------------- exp, row sum, block sums
    const int qq = warp & 3;                      // TMEM lane quarter
    const int t = qq * 32 + lane;                 // key slot of the unit
    const uint32_t tl = tbase + (static_cast<uint32_t>(qq * 32) << 16);
    // lse of the pair's rows in base 2 (row r = token r / G, head r % G)
    const int bi = pair / a.Hkv, h = pair - bi * a.Hkv;
    float l2[kVN];
#pragma unroll
    for (int r = 0; r < kVN; ++r) {
      l2[r] = CUDART_INF_F;                       // rows past R contribute exp2(-inf) = 0
      if (r < a.R) {
        const int j = r / a.G, g = r - (r / a.G) * a.G;
        l2[r] = a.lse[(static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * a.G + g] * 1.4426950408889634f;
      }
    }
    for (int i = 0; i < nunits; ++i) {
      const int sb = i & 1;
      const bool got = mbar_wait_bounded(&s_full[sb], (i >> 1) & 1, abort_flag);
      if (reduce_bar_or(!got)) {
        if (t == 0) fail();
        break;
      }
      tc::fence_after_sync();
      float sv[kVN];
      tmem_ld16(tl + sb * kVN, sv);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&s_free[sb]);
      float v = 0.f;
#pragma unroll
      for (int r = 0; r < kVN; ++r) v += ex2f(sv[r] * a.qscale - l2[r]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[sb * 4 + qq] = v;
      reduce_bar();
      // warps of key slots 0-63 (qq 0, 1) and 64-127 (qq 2, 3): one tile each
      if (lane == 0 && (qq & 1) == 0) {
        const int tile = 2 * (u0 + i) + (qq >> 1);
        if (tile < a.tiles)
          atomicAdd(a.mass + static_cast<int64_t>(pair) * a.nb + (tile * 64) / a.b, red[sb * 4 + qq] + red[sb * 4 + qq + 1]);
      }
    }
  }

  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 32);
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

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

}  // namespace

bool block_mass_supported(const BlockMassArgs& a) {
  return a.R >= 1 && a.R <= kVN && a.b % 64 == 0 && a.kv_end < (int64_t(1) << 31);
}

cudaError_t launch_block_mass(BlockMassArgs a, int num_sms, cudaStream_t s) {
  if (a.units == 0) return cudaSuccess;
  EncodeFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap qm, km;
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    // Q [B * n_q tokens][Hq heads][128]: box 64 columns x G heads x n_q tokens
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.Hq), static_cast<cuuint64_t>(a.B) * a.n_q};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(a.Hq) * 256};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(a.G), static_cast<cuuint32_t>(a.n_q)};
    if (enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.Q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // K [pairs][cap keys][128], rows at or past kv_end read as zeros
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.kv_end), static_cast<cuuint64_t>(a.B) * a.Hkv};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(a.cap) * 256};
    cuuint32_t box[3] = {64, 64, 1};
    if (enc(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.K), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // units of a pair per CTA: about eight CTAs per SM over the whole job
  const int64_t pairs = static_cast<int64_t>(a.B) * a.Hkv;
  const int64_t total = pairs * a.units;
  const int64_t want = static_cast<int64_t>(num_sms > 0 ? num_sms : 148) * 8;
  int64_t upc = (total + want - 1) / want;
  upc = upc < 4 ? 4 : upc;
  a.upc = static_cast<int>(upc < a.units ? upc : a.units);
  a.cpp = (a.units + a.upc - 1) / a.upc;
  cudaError_t e = cudaFuncSetAttribute(block_mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kVSmemBytes));
  if (e != cudaSuccess) return e;
  block_mass_kernel<<<static_cast<unsigned>(pairs * a.cpp), kVThreads, kVSmemBytes, s>>>(qm, km, a);
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
