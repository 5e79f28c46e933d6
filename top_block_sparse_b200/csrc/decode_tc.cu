// Step 4 for decode and draft chunks on the tensor cores (bf16 K, V and Q):
// softmax attention over the retained keys only (S3R review, section
// "稀疏起草": softmax over K_T and the weighted sum of V_T for the retained
// index set T; PulseCol §3.1 eq. (1)-(2): logits q.k/sqrt(d_h), keys outside
// the mask get zero weight).  The retained set, the work units (two 64-key
// tiles of one (sequence, KV head) pair), their stream-K split over one CTA
// per SM and the combine of partial results are those of decode_attn.cu.
//
// The keys of a unit sit on the MMA's M axis and the pair's <= 16 query rows
// (n_q tokens x G heads) on its N axis:
//   S^T  = K Q^T       tcgen05.mma M 128 keys x N 16 rows x K 128 (d), fp32 in TMEM
//   P    = softmax     4 warps, one key per thread (TMEM lane = key); the row
//                      max is exchanged through shared memory once per unit,
//                      the running max is raised lazily (only when a row's
//                      max grows by more than 2^8, which rescales O in TMEM)
//   O^T += V^T P^T     tcgen05.mma M 128 (d) x N 16 rows x K 128 keys; V is
//                      the MN-major operand straight from its TMA tile
// Every K/V byte is thus read from shared memory by the tensor cores alone;
// the CUDA cores do O(keys x rows) work per unit instead of O(keys x rows x d).
//
// CTA roles: warp 0 TMA producer (Q once per pair into a double buffer; K and
// V as 64-row x 128-byte boxes, two d-halves per tile, into a 3-stage ring of
// 64 KB units; rows at or past the end of the cache are zero-filled by the
// tensor map), warp 1 TMEM owner and MMA issuer, warps 2-5 softmax and
// epilogue.  With 9-16 rows (draft chunks, dense verify) warps 6-9 join as a
// second softmax warpgroup: warps w and w + 4 share a TMEM lane quarter (the
// same keys) and take rows 0-7 and 8-15, which halves each unit's softmax
// chain.  TMEM columns: S in [0,16) / [16,32) by unit parity, O^T in
// [32,48) / [48,64) by pair parity.  All waits are bounded.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <algorithm>

#include "common.cuh"
#include "decode_units.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace sa {
namespace {

constexpr int kN = 16;                          // query rows per pair on the MMA N axis
constexpr int kKVHalf = 16384;                  // one d-half of a unit: 128 keys x 128 B
constexpr int kStage = 4 * kKVHalf;             // K (two d-halves) + V (two d-halves)
constexpr int kNS = 3;                          // ring stages
constexpr int kQBuf = 2 * kN * 128;             // two d-halves of 16 rows x 128 B
constexpr int kPBuf = 2 * kN * 128;             // two key-halves of 16 rows x 128 B
constexpr int kThreads = 192;
constexpr int kThreadsFused = 256;              // fused: warps 6-7 select the top-k
constexpr int kThreadsSplit = 320;              // 9-16 rows: warps 6-9 are a second softmax warpgroup
constexpr int kSoftThreads = 128;
constexpr int kSelBarThreads = 192;             // softmax warps + selection warps
constexpr int kNumBars = 24;                    // 23 used; an even count keeps what follows 16-byte aligned
constexpr uint32_t kIdescS = tc::idesc_bf16(128, kN, false, false);
constexpr uint32_t kIdescO = tc::idesc_bf16(128, kN, true, false);
constexpr float kLazy = 8.f;                    // raise the running max when it grows by > 2^8
constexpr int kMaxSelPerCta = 64;               // fused: pairs one CTA may select
// wmax and lsum follow the barriers and the stage records and are read as float4
static_assert((kNumBars * 8 + kNS * sizeof(StageInfo)) % 16 == 0,
              "shared memory after the stage records must stay 16-byte aligned");
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kNS) * kStage + 2 * kQBuf + 2 * kPBuf +
                              kNumBars * 8 + kNS * sizeof(StageInfo) + (2 * 4 * kN + 4 * kN) * 4 + 32;
constexpr size_t kSmemFused = kSmemBytes;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float float_of_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync 1, %0;" ::"r"(kSoftThreads) : "memory");
}
// Split rows: barrier 1 (warps 2-5) or 3 (warps 6-9) for one warpgroup's
// rows, barrier 4 for both warpgroups.
__device__ __forceinline__ void group_bar(int grp) {
  asm volatile("bar.sync %0, %1;" ::"r"(grp ? 3 : 1), "r"(kSoftThreads) : "memory");
}
__device__ __forceinline__ void groups_bar() {
  asm volatile("bar.sync 4, %0;" ::"r"(2 * kSoftThreads) : "memory");
}

// Threads of an instantiation, and whether its softmax rows are split over
// two warpgroups.
template <int NR, int FUSED>
constexpr bool kSplitRows = NR == 16 && FUSED == 0;
template <int NR, int FUSED>
constexpr int kThreadsOf = FUSED ? kThreadsFused : (kSplitRows<NR, FUSED> ? kThreadsSplit : kThreads);
// The same barrier, returning whether any of the softmax threads passed true.
__device__ __forceinline__ bool softmax_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(kSoftThreads)
      : "memory");
  return r != 0;
}

// Named barrier 2: the softmax warps arrive once scoring is done, the
// selection warps of the fused kernel wait for them.
__device__ __forceinline__ void sel_bar_arrive() {
  asm volatile("bar.arrive 2, %0;" ::"r"(kSelBarThreads) : "memory");
}
__device__ __forceinline__ void sel_bar_sync() {
  asm volatile("bar.sync 2, %0;" ::"r"(kSelBarThreads) : "memory");
}


__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float (&v)[4]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
// Reduction of each of NR rows over the 32 lanes of a warp (max or sum) by a
// reduce-scatter: at each level a lane keeps half of the rows it still holds
// and trades the other half with the lane that differs in that bit, so NR
// rows take NR shuffles in all (not 5 NR); lane l ends with row l % NR.
template <int NR, bool MAX>
__device__ __forceinline__ float rows_reduce(float (&v)[NR], int lane) {
#pragma unroll
  for (int h = NR / 2; h >= 1; h >>= 1) {
    const bool up = (lane & h) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float keep = up ? v[i + h] : v[i];
      const float other = __shfl_xor_sync(0xffffffffu, up ? v[i] : v[i + h], h);
      v[i] = MAX ? fmaxf(keep, other) : keep + other;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = NR; o < 32; o <<= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, r, o);
    r = MAX ? fmaxf(r, other) : r + other;
  }
  return r;
}

// The first NR columns of this warp's 32 TMEM lanes.  A thread reads at
// most 8 rows: 16-row instantiations split their rows over two warpgroups.
template <int NR>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float (&v)[NR]) {
  static_assert(NR == 4 || NR == 8, "a thread reads at most 8 rows");
  if constexpr (NR == 4) tmem_ld4(taddr, v);
  else tmem_ld8(taddr, v);
}
template <int NR>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const float (&v)[NR]) {
  static_assert(NR == 4 || NR == 8, "a thread rescales at most 8 rows");
  if constexpr (NR == 4) tmem_st4(taddr, v);
  else tmem_st8(taddr, v);
}

template <bool OUT_BF16>
__device__ __forceinline__ void store_out(void* O, int64_t idx, float v) {
  if constexpr (OUT_BF16) static_cast<__nv_bfloat16*>(O)[idx] = __float2bfloat16_rn(v);
  else static_cast<float*>(O)[idx] = v;
}
// Four consecutive outputs v * s from element idx (a multiple of 4).
template <bool OUT_BF16>
__device__ __forceinline__ void store_out4(void* O, int64_t idx, float4 v, float s) {
  if constexpr (OUT_BF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * s, v.y * s), hi = __floats2bfloat162_rn(v.z * s, v.w * s);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&lo);
    w.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(O) + idx) = w;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(O) + idx) = make_float4(v.x * s, v.y * s, v.z * s, v.w * s);
  }
}

// Fused mode adds the step's scoring and selection in front of the
// attention: each CTA scores a contiguous run of the pair-major list of
// 128-key chunks of compressed keys (cp.async.bulk through the same ring),
// the CTA that finishes a pair's last chunk (atomic ticket) selects its top-k
// and publishes the table with a per-pair ready flag, and the producer waits
// for the flag of every pair before reading its table.  A cooperative launch
// keeps every CTA resident, so the waits end.
// FUSED: 0 attention only; 1 the whole step, each pair selected by the CTA
// that scored its last chunk (a warp bit search over <= kFusedMaxBlocks
// scores); 2 the whole step for long contexts and k <= kFusedSmallK: every
// CTA that scored chunks of a pair publishes the top k of its own rows, and
// the CTA completing the pair's count selects among those candidates.
template <bool OUT_BF16, int NR, int FUSED, bool MASS>
__global__ void __launch_bounds__(kThreadsOf<NR, FUSED>, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                     const __grid_constant__ CUtensorMap v_map, DecodeAttnArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;                                   // kNS x 64 KB
  unsigned char* Qs = ring + kNS * kStage;                      // 2 x 4 KB
  unsigned char* Ps = Qs + 2 * kQBuf;                           // 2 x 4 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(Ps + 2 * kPBuf);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 3;
  uint64_t* q_full = bars + 6;
  uint64_t* q_empty = bars + 8;
  uint64_t* s_full = bars + 10;
  uint64_t* s_free = bars + 12;
  uint64_t* p_full = bars + 14;
  uint64_t* p_free = bars + 16;
  uint64_t* o_full = bars + 18;
  uint64_t* o_free = bars + 20;
  uint64_t* score_done = bars + 22;      // fused: every score chunk consumed
  StageInfo* info = reinterpret_cast<StageInfo*>(bars + kNumBars);
  float* wmax = reinterpret_cast<float*>(info + kNS);          // [2][16 rows][4 warps]
  float* lsum = wmax + 2 * 4 * kN;                              // [16 rows][4 warps]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lsum + 4 * kN);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* ticket = reinterpret_cast<int*>(tmem_slot + 2);
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(tmem_slot + 4);    // 8-byte aligned
  __shared__ int sel_list[kMaxSelPerCta];                               // fused: pairs this CTA selects
  __shared__ int sel_first[kMaxSelPerCta];                              // FUSED 2: a run's first chunk
  __shared__ int sel_cnt[kMaxSelPerCta];                                // FUSED 2: its chunks
  __shared__ int n_sel;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's units: its share of list I, then its share of list D
  int64_t i0 = 0, d0 = 0;
  const int nI = list_share(a.ord.totI, a.ord.gI, blockIdx.x, &i0);
  const int nunits = nI + list_share(a.ord.totD, a.ord.gD, blockIdx.x, &d0);
  // fused: score chunks [c0, c1) of the pair-major chunk list come first and
  // take the ring's first r0 uses
  int c0 = 0, c1 = 0;
  if constexpr (FUSED) {
    const int total_chunks = a.B * a.Hkv * a.cpp;
    c0 = min(total_chunks, static_cast<int>(blockIdx.x) * a.cpc);
    c1 = min(total_chunks, c0 + a.cpc);
  }
  const int r0 = c1 - c0;

  if (threadIdx.x == 0) {
    n_sel = 0;
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSplitRows<NR, FUSED> ? 2 * kSoftThreads : kSoftThreads);
      mbar_init(&p_full[b], kSplitRows<NR, FUSED> ? 2 * kSoftThreads : kSoftThreads);
      mbar_init(&p_free[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], kSplitRows<NR, FUSED> ? 2 * kSoftThreads : kSoftThreads);
    }
    mbar_init(mma_done, 1);
    mbar_init(score_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Q rows past the pair's R and P rows past NR only feed MMA columns that
  // are never read; zero them once anyway.  (Every V row is written per
  // unit: see the producer.)
  {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    uint4* qp = reinterpret_cast<uint4*>(Qs);
    for (int i = threadIdx.x; i < (2 * kQBuf + 2 * kPBuf) / 16; i += blockDim.x) qp[i] = z;
    tc::fence_proxy_async_smem();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 64);
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
    // -------------------------------------------------------- TMA producer
    // the index table is written by the scoring kernel launched before this one
    if (a.pdl) pdl_wait_prior_grid();
    int issued = 0;
    RunCursor pc;
    pc.init(a.ord, i0, nI, d0, nunits);
    bool stop = false;
    if constexpr (FUSED) {
      // this CTA's score chunks: 128 compressed keys (64 KB of fp32) each
      for (int ci = 0; ci < r0 && !stop; ++ci) {
        const int gc = c0 + ci;
        const int pr = gc / a.cpp, ch = gc - pr * a.cpp;
        const int rows = min(128, static_cast<int>(a.nb) - ch * 128);
        const int s = ci % kNS;
        int ok = 1;
        if (lane == 0) {
          if (ci >= kNS && !mbar_wait_bounded(&kv_empty[s], ((ci / kNS) & 1) ^ 1, abort_flag)) ok = 0;
          if (ok) {
            const uint32_t bytes = static_cast<uint32_t>(rows) * kHeadDim * 4;
            mbar_arrive_expect_tx(&kv_full[s], bytes);
            bulk_g2s(ring + s * kStage, a.Kc + (static_cast<int64_t>(pr) * a.nb + ch * 128) * kHeadDim, bytes,
                     &kv_full[s]);
          } else {
            fail();
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) stop = true;
      }
    }
    // units in batches of up to 32 of one run: the lanes compute the key
    // ranges together, then lane 0 issues them in order
    for (int i = 0; i < nunits && !stop;) {
      pc.at(i);
      const int end = min(pc.next_start, min(nunits, i + 32));
      bool wait_ok = true;
      if constexpr (FUSED) {
        if (pc.in_d) {
          // the pair's table is published by the CTA that selected it
          const volatile unsigned* rdy = a.ready + pc.pair;
          const uint64_t tw = global_ns();
          for (uint32_t spin = 0; *rdy == 0u; ++spin) {
            if ((spin & 63u) == 0 && (*abort_flag || global_ns() - tw > kWaitLimitNs)) {
              wait_ok = false;
              break;
            }
          }
          __threadfence();
        }
      }
      if (__any_sync(0xffffffffu, !wait_ok)) {
        if (lane == 0) fail();
        stop = true;
        break;
      }
      int64_t ks0 = 0, ks1 = 0;
      int nk0 = 0, nk1 = 0;
      if (i + lane < end) {
        unit_tile<FUSED != 0>(a, pc, i + lane, 0, &ks0, &nk0);
        unit_tile<FUSED != 0>(a, pc, i + lane, 1, &ks1, &nk1);
      }
      const int64_t pair = pc.pair;
      const int pk = pc.ordinal;
      for (int l = 0; l < end - i; ++l) {
        const int64_t k0 = __shfl_sync(0xffffffffu, ks0, l);
        const int64_t k1 = __shfl_sync(0xffffffffu, ks1, l);
        const int n0 = __shfl_sync(0xffffffffu, nk0, l);
        const int n1 = __shfl_sync(0xffffffffu, nk1, l);
        const int ri = r0 + i + l;               // ring use
        const int s = ri % kNS;
        int ok = 1;
        if (lane == 0) {
          if (l == 0 && pc.first(i)) {
            const int qb = pk & 1;
            if (pk >= 2 && !mbar_wait_bounded(&q_empty[qb], ((pk >> 1) + 1) & 1, abort_flag)) ok = 0;
            if (ok) {
              const int bi = static_cast<int>(pair / a.Hkv), h = static_cast<int>(pair % a.Hkv);
              mbar_arrive_expect_tx(&q_full[qb], static_cast<uint32_t>(2 * a.R * 128));
              tc::tma_load_3d(Qs + qb * kQBuf, &q_map, 0, h * a.G, bi * a.n_q, &q_full[qb]);
              tc::tma_load_3d(Qs + qb * kQBuf + kN * 128, &q_map, 64, h * a.G, bi * a.n_q, &q_full[qb]);
            }
          }
          if (ok && ri >= kNS && !mbar_wait_bounded(&kv_empty[s], ((ri / kNS) & 1) ^ 1, abort_flag)) ok = 0;
          if (ok) {
            info[s].ks0 = k0;
            info[s].ks1 = k1;
            info[s].n0 = n0;
            info[s].n1 = n1;
            // Every V row of the stage meets the P^T operand (zeros for the
            // keys of an empty tile), so an empty tile still gets V: a box
            // at row kv_end, past the tensor map, which the copy fills with
            // zeros without reading memory.  Stale rows could be anything
            // (in the fused kernel, bytes of compressed keys), and 0 times a
            // NaN is a NaN.  Its K rows are masked out of the softmax.
            const int t0 = n0 > 0, t1 = n1 > 0;
            unsigned char* st = ring + s * kStage;
            const int p32 = static_cast<int>(pair);
            const int zr = static_cast<int>(a.kv_end);
            mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>((t0 + t1) * 2 * 8192 + 2 * 2 * 8192));
            const int r0 = t0 ? static_cast<int>(k0) : zr;
            if (t0) {
              tc::tma_load_3d(st, &k_map, 0, r0, p32, &kv_full[s]);
              tc::tma_load_3d(st + kKVHalf, &k_map, 64, r0, p32, &kv_full[s]);
            }
            tc::tma_load_3d(st + 2 * kKVHalf, &v_map, 0, r0, p32, &kv_full[s]);
            tc::tma_load_3d(st + 3 * kKVHalf, &v_map, 64, r0, p32, &kv_full[s]);
            const int r1 = t1 ? static_cast<int>(k1) : zr;
            if (t1) {
              tc::tma_load_3d(st + 8192, &k_map, 0, r1, p32, &kv_full[s]);
              tc::tma_load_3d(st + kKVHalf + 8192, &k_map, 64, r1, p32, &kv_full[s]);
            }
            tc::tma_load_3d(st + 2 * kKVHalf + 8192, &v_map, 0, r1, p32, &kv_full[s]);
            tc::tma_load_3d(st + 3 * kKVHalf + 8192, &v_map, 64, r1, p32, &kv_full[s]);
          } else {
            fail();
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          stop = true;
          break;
        }
        issued = i + l + 1;
      }
      i = end;
    }
    // do not leave while copies into this CTA's shared memory may be in flight
    if (lane == 0) {
      const int used = r0 + issued;
      for (int ri = max(0, used - kNS); ri < used; ++ri) mbar_wait_bounded(&kv_full[ri % kNS], (ri / kNS) & 1, nullptr);
      for (int k = max(0, pc.ordinal - 1); k <= pc.ordinal; ++k)
        if (issued > 0) mbar_wait_bounded(&q_full[k & 1], (k >> 1) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // S(i) needs unit i's K and Q and a free S buffer; PV(i) needs P(i).  The
    // thread polls both and issues whichever is ready, so a unit's ring stage
    // (released when PV(i) completes) never waits for the next unit's data.
    // The whole warp runs the loop in lock step (descriptors warp-uniform);
    // every readiness test is made warp-wide and one elected lane issues.
    {
      const uint32_t ring_a = smem_u32(ring), qa = smem_u32(Qs), pa = smem_u32(Ps);
      int ns = 0, npv = 0;                  // next S / PV to issue
      RunCursor cs, cp;                     // run bookkeeping of units ns / npv
      cs.init(a.ord, i0, nI, d0, nunits);
      cp.init(a.ord, i0, nI, d0, nunits);
      bool ok = true;
      // Fused: the ring's first r0 uses carry score chunks, which land in
      // order of use as far as the softmax warps' waits see them.  Only once
      // the last one has landed does each stage's full barrier stand at or
      // past its last score-chunk phase; polled earlier, a completed phase of
      // the same parity one use back would read as an attention unit's
      // arrival.
      if constexpr (FUSED) {
        if (!mbar_wait_warp(score_done, 0, abort_flag)) ok = false;
      }
      uint64_t t0 = global_ns();
      for (uint32_t spin = 0; ok && npv < nunits; ++spin) {
        bool did = false;
        if (ns < nunits) {
          const bool fi = cs.first(ns);
          const int pk = cs.ordinal, qb = pk & 1, s = (r0 + ns) % kNS;
          const bool ready = mbar_test_wait(&kv_full[s], ((r0 + ns) / kNS) & 1) &&
                             (!fi || mbar_test_wait(&q_full[qb], (pk >> 1) & 1)) &&
                             (ns < 2 || mbar_test_wait(&s_free[ns & 1], ((ns >> 1) + 1) & 1));
          if (__all_sync(0xffffffffu, ready)) {
            tc::fence_after_sync();
            const uint32_t kst = ring_a + s * kStage, qst = qa + qb * kQBuf;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc::mma_bf16_elect(tbase + (ns & 1) * kN,
                           tc::smem_desc(kst + (kk >> 2) * kKVHalf + (kk & 3) * 32, 16, 1024),
                           tc::smem_desc(qst + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024), kIdescS, kk > 0);
            tc::mma_commit_elect(&s_full[ns & 1]);
            // no later MMA reads this Q buffer for this pair
            if (cs.last(ns)) tc::mma_commit_elect(&q_empty[qb]);
            ++ns;
            cs.at(ns);
            did = true;
          }
        }
        if (npv < ns) {
          const bool fi = cp.first(npv);
          const int pk = cp.ordinal, ob = pk & 1;
          const bool ready = mbar_test_wait(&p_full[npv & 1], (npv >> 1) & 1) &&
                             (!fi || pk < 2 || mbar_test_wait(&o_free[ob], ((pk >> 1) + 1) & 1));
          if (__all_sync(0xffffffffu, ready)) {
            tc::fence_after_sync();
            const uint32_t vst = ring_a + ((r0 + npv) % kNS) * kStage + 2 * kKVHalf;
            const uint32_t pb = pa + (npv & 1) * kPBuf;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc::mma_bf16_elect(tbase + 32 + ob * kN, tc::smem_desc(vst + kk * 2048, kKVHalf, 1024),
                           tc::smem_desc(pb + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024), kIdescO,
                           !(fi && kk == 0));
            tc::mma_commit_elect(&kv_empty[(r0 + npv) % kNS]);
            tc::mma_commit_elect(&p_free[npv & 1]);
            if (cp.last(npv)) tc::mma_commit_elect(&o_full[ob]);
            ++npv;
            cp.at(npv);
            did = true;
          }
        }
        if (did) {
          t0 = global_ns();
        } else if ((spin & 63u) == 0) {
          if (__any_sync(0xffffffffu, *abort_flag || global_ns() - t0 > kWaitLimitNs)) {
            ok = false;
            break;
          }
        }
      }
      if (!ok && lane == 0) fail();
      // every MMA must be complete before TMEM is released
      tc::mma_commit_elect(mma_done);
      mbar_wait_warp(mma_done, 0, nullptr);
    }
    __syncwarp();
  } else if (FUSED && warp >= 6) {
    // ------------------------------------------ top-k selection (fused only)
    // the pairs whose last score chunk this CTA scored, a warp each, while
    // the softmax warps attend the index-independent units
    sel_bar_sync();
    const int nb = static_cast<int>(a.nb);
    const int nsel = n_sel;
    for (int e = warp - 6; e < nsel && !*abort_flag && FUSED == 2; e += 2) {
      // FUSED 2: this CTA's run of chunks of pair pr -> the top k of its own
      // rows into the pair's candidate slot, then the pair's chunk count
      const int pr = sel_list[e], first = sel_first[e], n = sel_cnt[e];
      const int row0 = (first - pr * a.cpp) * 128, row1 = min(nb, row0 + n * 128);
      const float* sc = a.scores + static_cast<int64_t>(pr) * nb;
      constexpr int PR = kFusedRunChunks * 128 / 32;
      uint32_t kr[PR];
#pragma unroll
      for (int i = 0; i < PR; ++i) {
        const int j = row0 + i * 32 + lane;
        const float v = j < row1 ? __ldcg(sc + j) : 0.f;
        const int64_t lo = static_cast<int64_t>(j) * a.b, hi = lo + a.b;
        const bool cand = j < row1 && (lo < a.w_begin) && (hi > a.s_end);
        const uint32_t key = float_key(v);
        kr[i] = cand ? (key == 0u ? 1u : key) : 0u;
      }
      const int slot = static_cast<int>(blockIdx.x) - (pr * a.cpp) / a.cpc;
      uint2* cs = a.cand + (static_cast<int64_t>(pr) * kFusedCandSlots + slot) * kFusedSmallK;
      // k passes, each taking the largest key left (the lowest id on ties)
#pragma unroll 1
      for (int q = 0; q < kFusedSmallK; ++q) {
        uint32_t best = 0u;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < PR; ++i) {
          const bool gt = kr[i] > best;
          best = gt ? kr[i] : best;
          bi = gt ? i : bi;
        }
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        unsigned jm = 0xffffffffu;
        if (m != 0u && q < a.top_k) {
          jm = __reduce_min_sync(0xffffffffu, best == m ? static_cast<unsigned>(bi * 32 + lane) : 0xffffffffu);
#pragma unroll
          for (int i = 0; i < PR; ++i) kr[i] = (static_cast<unsigned>(i * 32 + lane) == jm) ? 0u : kr[i];
        }
        if (lane == 0) cs[q] = make_uint2(jm == 0xffffffffu ? 0u : m, jm == 0xffffffffu ? 0u : row0 + jm);
      }
      __threadfence();
      __syncwarp();
      unsigned old = 0u;
      if (lane == 0) old = atomicAdd(&a.score_cnt[pr], static_cast<unsigned>(n));
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old + n != static_cast<unsigned>(a.cpp)) continue;
      // the last run of the pair: merge the slots' candidates
      __threadfence();
      if (lane == 0) a.score_cnt[pr] = 0u;
      const int nslots = ((pr + 1) * a.cpp - 1) / a.cpc - (pr * a.cpp) / a.cpc + 1;
      const uint2* cp = a.cand + static_cast<int64_t>(pr) * kFusedCandSlots * kFusedSmallK;
      constexpr int PM = kFusedCandSlots * kFusedSmallK / 32;
      uint32_t mk[PM], mi[PM];
#pragma unroll
      for (int i = 0; i < PM; ++i) {
        const int c = i * 32 + lane;
        const uint2 v = c < nslots * kFusedSmallK ? __ldcg(cp + c) : make_uint2(0u, 0u);
        mk[i] = v.x;
        mi[i] = v.y;
      }
      int got[kFusedSmallK];
      int ng = 0;
#pragma unroll
      for (int q = 0; q < kFusedSmallK; ++q) {
        got[q] = 0x7fffffff;
        uint32_t best = 0u, bid = 0xffffffffu;
#pragma unroll
        for (int i = 0; i < PM; ++i) {
          const bool better = mk[i] > best || (mk[i] == best && mk[i] != 0u && mi[i] < bid);
          best = better ? mk[i] : best;
          bid = better ? mi[i] : bid;
        }
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        if (m != 0u && q < a.top_k) {
          const unsigned jm = __reduce_min_sync(0xffffffffu, best == m ? bid : 0xffffffffu);
#pragma unroll
          for (int i = 0; i < PM; ++i) mk[i] = (mk[i] == m && mi[i] == jm) ? 0u : mk[i];
          got[q] = static_cast<int>(jm);
          ++ng;
        }
      }
      if (lane == 0) {
        // ascending ids (absent ones sort last)
#pragma unroll
        for (int q = 1; q < kFusedSmallK; ++q) {
#pragma unroll
          for (int r = q; r > 0; --r) {
            const int lo = min(got[r - 1], got[r]), hi = max(got[r - 1], got[r]);
            got[r - 1] = lo;
            got[r] = hi;
          }
        }
        int32_t* out = a.idx_w + static_cast<int64_t>(pr) * a.top_k;
#pragma unroll
        for (int q = 0; q < kFusedSmallK; ++q)
          if (q < a.top_k) out[q] = q < ng ? got[q] : -1;
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicExch(&a.ready[pr], 1u);
    }
    for (int e = warp - 6; e < nsel && !*abort_flag && FUSED == 1; e += 2) {
      const int pr = sel_list[e];
      __threadfence();
      if (lane == 0) a.score_cnt[pr] = 0u;
      const float* sc = a.scores + static_cast<int64_t>(pr) * nb;
      // the pair's keys in registers (all loads in flight at once)
      constexpr int PER = kFusedMaxBlocks / 32;
      float v[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int j = i * 32 + lane;
        v[i] = j < nb ? __ldcg(sc + j) : 0.f;
      }
      uint32_t kr[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int j = i * 32 + lane;
        const int64_t lo = static_cast<int64_t>(j) * a.b, hi = lo + a.b;
        const bool cand = j < nb && (lo < a.w_begin) && (hi > a.s_end);
        const uint32_t key = float_key(v[i]);
        kr[i] = cand ? (key == 0u ? 1u : key) : 0u;
      }
      warp_topk_regs<PER>(kr, a.top_k, a.idx_w + static_cast<int64_t>(pr) * a.top_k);
      // publish: every lane's table entries, then the flag
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicExch(&a.ready[pr], 1u);
    }
  } else {
    // ------------------------------------------------- softmax and epilogue
    const int qq = warp & 3;                  // TMEM lane quarter of this warp
    const int t = qq * 32 + lane;             // key slot of the unit; output column d in the epilogue
    constexpr bool SPLIT = kSplitRows<NR, FUSED>;
    constexpr int NH = SPLIT ? NR / 2 : NR;   // rows of this thread's warpgroup
    const int grp = SPLIT ? (warp - 2) >> 2 : 0;
    const int rb = grp * NH;                  // its first row
    // one warpgroup's barrier (its rows' maxima and sums), and the barrier of
    // every softmax thread (the pair's ticket)
    auto gbar = [&]() {
      if constexpr (SPLIT) group_bar(grp);
      else softmax_bar();
    };
    auto abar = [&]() {
      if constexpr (SPLIT) groups_bar();
      else softmax_bar();
    };
    const uint32_t tl = tbase + (static_cast<uint32_t>(qq * 32) << 16);
    const int R = a.R, G = a.G;
    const int C = static_cast<int>(a.C);
    const float qscale = a.qscale;
    const int tile = t >> 6, kc = t & 63;
    // byte offsets of this key's P^T entries (row r, key kc of its 64-key half)
    uint32_t poff[NH];
#pragma unroll
    for (int r = 0; r < NH; ++r) poff[r] = tile * (kN * 128) + tc::sw128_off(rb + r, kc >> 3) + (kc & 7) * 2;
    float m_run[NH], l_t[NH];
    RunCursor pc;
    pc.init(a.ord, i0, nI, d0, nunits);
    bool ok = true;

    auto epilogue = [&]() -> bool {
      // row sums over the unit's 128 key slots
      float mine = 0.f;
      if constexpr (NH >= 8) {
        float lt[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) lt[r] = l_t[r];
        mine = rows_reduce<NH, false>(lt, lane);
      } else {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          float v = l_t[r];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          mine = (lane == r) ? v : mine;
        }
      }
      if (lane < NH) lsum[(rb + lane) * 4 + qq] = mine;
      const int pkk = pc.ordinal, ob = pkk & 1;
      if (!mbar_wait_bounded(&o_full[ob], (pkk >> 1) & 1, abort_flag)) return false;
      tc::fence_after_sync();
      float ov[NH];
      tmem_ldn<NH>(tl + 32 + ob * kN + rb, ov);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&o_free[ob]);
      gbar();
      float L[NH];
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        const float4 v = reinterpret_cast<const float4*>(lsum)[rb + r];
        L[r] = (v.x + v.y) + (v.z + v.w);
      }
      const int64_t pair = pc.pair;
      int n_ctas, slot;
      pair_slots(a.ord, pair, pc.in_d, &n_ctas, &slot);
      const int bi = static_cast<int>(pair / a.Hkv), h = static_cast<int>(pair % a.Hkv);
      auto out_row = [&](int r) -> int64_t {
        const int j = r / G, g = r - (r / G) * G;
        return (static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * G + g;
      };
      if (n_ctas == 1) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          if (rb + r < R) {
            const int64_t orow = out_row(rb + r);
            store_out<OUT_BF16>(a.O, orow * kHeadDim + t, ov[r] * (L[r] > 0.f ? 1.f / L[r] : 0.f));
            if (t == r && a.lse)
              a.lse[orow] = L[r] > 0.f ? (m_run[r] + log2f(L[r])) * 0.69314718055994531f : -CUDART_INF_F;
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          if (rb + r < R) {
            const int64_t ps = (pair * a.n_slots + slot) * a.R4 + rb + r;
            a.part_O[ps * kHeadDim + t] = ov[r];
            if (t == r) {
              a.part_ml[ps * 2 + 0] = m_run[r];
              a.part_ml[ps * 2 + 1] = L[r];
            }
          }
        }
        // the barrier orders every thread's partial stores before thread 0's
        // release fence and ticket
        abar();
        if (t == 0 && grp == 0) {
          __threadfence();
          const unsigned tk = atomicAdd(&a.counters[pair], 1u);
          *ticket = (tk == static_cast<unsigned>(n_ctas - 1));
        }
        abar();
        if (*ticket) {
          __threadfence();
          // thread t merges columns 4 (t % 32) .. + 3 of its warpgroup's rows
          // t / 32 + 4 k; the loads of up to SG slots are all in flight
          // before their use
          constexpr int KR = NH / 4;
          constexpr int SG = NH >= 16 ? 2 : 4;
          const int c4 = (t & 31) * 4, r0w = rb + (t >> 5);
          float Mx[KR], Ls[KR];
          float4 acc[KR];
#pragma unroll
          for (int k = 0; k < KR; ++k) {
            Mx[k] = -CUDART_INF_F;
            Ls[k] = 0.f;
            acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          for (int s0 = 0; s0 < n_ctas; s0 += SG) {
            float2 ml[SG][KR];
            float4 po[SG][KR];
#pragma unroll
            for (int j = 0; j < SG; ++j) {
#pragma unroll
              for (int k = 0; k < KR; ++k) {
                const int r = r0w + 4 * k;
                ml[j][k] = make_float2(-CUDART_INF_F, 0.f);
                po[j][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s0 + j < n_ctas && r < R) {
                  const int64_t ps = (pair * a.n_slots + s0 + j) * a.R4 + r;
                  ml[j][k] = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + ps);
                  po[j][k] = __ldcg(reinterpret_cast<const float4*>(a.part_O + ps * kHeadDim + c4));
                }
              }
            }
#pragma unroll
            for (int k = 0; k < KR; ++k) {
              float mn = Mx[k];
#pragma unroll
              for (int j = 0; j < SG; ++j) mn = fmaxf(mn, ml[j][k].x);
              const float mr = (mn == -CUDART_INF_F) ? 0.f : mn;
              const float so = exp2f(Mx[k] - mr);
              Ls[k] *= so;
              acc[k].x *= so;
              acc[k].y *= so;
              acc[k].z *= so;
              acc[k].w *= so;
#pragma unroll
              for (int j = 0; j < SG; ++j) {
                const float sc = exp2f(ml[j][k].x - mr);
                Ls[k] += ml[j][k].y * sc;
                acc[k].x += po[j][k].x * sc;
                acc[k].y += po[j][k].y * sc;
                acc[k].z += po[j][k].z * sc;
                acc[k].w += po[j][k].w * sc;
              }
              Mx[k] = mn;
            }
          }
#pragma unroll
          for (int k = 0; k < KR; ++k) {
            const int r = r0w + 4 * k;
            if (r < R) {
              const int64_t orow = out_row(r);
              const float inv = Ls[k] > 0.f ? 1.f / Ls[k] : 0.f;
              store_out4<OUT_BF16>(a.O, orow * kHeadDim + c4, acc[k], inv);
              if (c4 == 0 && a.lse)
                a.lse[orow] = Ls[k] > 0.f ? (Mx[k] + log2f(Ls[k])) * 0.69314718055994531f : -CUDART_INF_F;
            }
          }
          if (t == 0 && grp == 0) a.counters[pair] = 0u;
        }
      }
      abar();            // lsum and the ticket are reused by the next pair
      return true;
    };

    if constexpr (FUSED) {
      // ---- scoring: warp w scores rows 32 w .. 32 w + 31 of every chunk
      // (q-bar = sum of the group's heads of the first new token, times the
      // softmax scale; 8 rows per batch, a float4 per lane, shuffle sums)
      const int sw = warp - 2;
      const int nb = static_cast<int>(a.nb);
      int cur = -1;
      int seg_cnt = 0;                           // chunks of pair `cur` scored by this CTA
      float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f);
      // count this CTA's chunks of a pair once its run of them ends (one
      // release fence and one atomic per run, not per chunk); the CTA that
      // completes the pair's count selects it
      int run_first = 0;                         // FUSED 2: the run's first chunk
      auto close_run = [&](int pr, int n) {
        if constexpr (FUSED == 1) {
          __threadfence();
          const unsigned old = atomicAdd(&a.score_cnt[pr], static_cast<unsigned>(n));
          if (old + n == static_cast<unsigned>(a.cpp)) {
            if (n_sel < kMaxSelPerCta) sel_list[n_sel++] = pr;
            else report(a.status, kStatusTimeout);
          }
        } else if (n_sel < kMaxSelPerCta) {
          // every run goes to the selection warps, which count it
          sel_list[n_sel] = pr;
          sel_first[n_sel] = run_first;
          sel_cnt[n_sel] = n;
          ++n_sel;
        } else {
          report(a.status, kStatusTimeout);
        }
      };
      for (int ci = 0; ci < r0; ++ci) {
        const int gc = c0 + ci;
        const int pr = gc / a.cpp, ch = gc - pr * a.cpp;
        const int rows = min(128, nb - ch * 128);
        const int s = ci % kNS;
        if (pr != cur) {
          if (t == 0 && cur >= 0) close_run(cur, seg_cnt);
          cur = pr;
          seg_cnt = 0;
          run_first = gc;
          const int bi = pr / a.Hkv, h = pr % a.Hkv;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int g = 0; g < G; ++g) {
            const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(
                static_cast<const uint16_t*>(a.Q) + (static_cast<int64_t>(bi) * a.n_q * a.Hq + h * G + g) * kHeadDim) + lane);
            acc.x += bf16lo(w2.x);
            acc.y += bf16hi(w2.x);
            acc.z += bf16lo(w2.y);
            acc.w += bf16hi(w2.y);
          }
          // mean pooling: qbar times the softmax scale; LSA centroids:
          // qbar / |qbar| (cosine scores)
          float mul = a.sscale;
          if (a.lsa) {
            float ss = acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            mul = ss > 0.f ? rsqrtf(ss) : 0.f;
          }
          q4 = make_float4(acc.x * mul, acc.y * mul, acc.z * mul, acc.w * mul);
        }
        const bool got = mbar_wait_bounded(&kv_full[s], (ci / kNS) & 1, abort_flag);
        // the last score chunk has landed, so every stage's full barrier has
        // passed its score-chunk phases: the MMA warp may poll the ring
        if (got && t == 0 && ci == r0 - 1) mbar_arrive(score_done);
        if (got) {
          const float* rowp = reinterpret_cast<const float*>(ring + s * kStage);
          float* sc = a.scores + static_cast<int64_t>(pr) * nb + ch * 128;
          // 16 rows at a time; a reduce-scatter over the lanes (each level
          // keeps half of the rows and sends the other half to the partner
          // lane) leaves row (lane & 15) summed over the lanes with bit 4
          // equal, and one more exchange completes it
          const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
#pragma unroll 1
          for (int grp = 0; grp < 2; ++grp) {
            const int rb = sw * 32 + grp * 16;
            float d[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              // rows past the chunk hold stale data; their sums are never stored
              const float4 v = reinterpret_cast<const float4*>(rowp + (rb + u) * kHeadDim)[lane];
              d[u] = v.x * q4.x + v.y * q4.y + v.z * q4.z + v.w * q4.w;
            }
            float e8[8], e4[4], e2[2];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              e8[i] = (b3 ? d[i + 8] : d[i]) + __shfl_xor_sync(0xffffffffu, b3 ? d[i] : d[i + 8], 8);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              e4[i] = (b2 ? e8[i + 4] : e8[i]) + __shfl_xor_sync(0xffffffffu, b2 ? e8[i] : e8[i + 4], 4);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              e2[i] = (b1 ? e4[i + 2] : e4[i]) + __shfl_xor_sync(0xffffffffu, b1 ? e4[i] : e4[i + 2], 2);
            float e1 = (b0 ? e2[1] : e2[0]) + __shfl_xor_sync(0xffffffffu, b0 ? e2[0] : e2[1], 1);
            e1 += __shfl_xor_sync(0xffffffffu, e1, 16);
            if (lane < 16 && rb + lane < rows) sc[rb + lane] = e1;
          }
        }
        // every warp is done with stage s and its score stores (uniform exit)
        if (softmax_bar_or(!got)) {
          ok = false;
          break;
        }
        if (t == 0) mbar_arrive(&kv_empty[s]);
        ++seg_cnt;
      }
      if (t == 0 && ok && cur >= 0) close_run(cur, seg_cnt);
      softmax_bar();
      if (t == 0 && r0 == 0) mbar_arrive(score_done);    // no score chunks
      // sel_list is complete: hand it to the selection warps and go on
      sel_bar_arrive();
    }

    for (int i = 0; i < nunits && ok; ++i) {
      pc.at(i);
      const bool fi = pc.first(i);
      if (fi) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          m_run[r] = -CUDART_INF_F;
          l_t[r] = 0.f;
        }
      }
      const int ri = r0 + i;                 // ring use
      const int s = ri % kNS, sb = i & 1;
      if (!mbar_wait_bounded(&s_full[sb], (i >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float sv[NH];
      tmem_ldn<NH>(tl + sb * kN + rb, sv);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&s_free[sb]);
      // the unit's key ranges, published with the stage's full barrier
      if (!mbar_wait_bounded(&kv_full[s], (ri / kNS) & 1, abort_flag)) {
        ok = false;
        break;
      }
      const int n = tile ? info[s].n1 : info[s].n0;
      const int64_t kst = tile ? info[s].ks1 : info[s].ks0;
      const int dnew = static_cast<int>(tile ? info[s].ks1 : info[s].ks0) + kc - C;   // >= 0: a new key
      const int dn = dnew < 0 ? -1 : min(dnew, 64);
      const bool kv = kc < n;
      float x[NH];
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        // new key C + dnew is seen by token row / G iff dnew <= row / G, i.e. dnew * G <= row
        const int row = rb + r;
        const bool v = kv && row < R && (dn < 0 || dn * G <= row);
        x[r] = v ? sv[r] * qscale : -CUDART_INF_F;
      }
      // unit max of every row: warp reduction, then the four warps through
      // shared memory (row r of this warp stored by lane r)
      float* wm = wmax + sb * (kN * 4);
      if constexpr (NH >= 8) {
        float xm[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) xm[r] = x[r];
        const float mx = rows_reduce<NH, true>(xm, lane);
        if (lane < NH) wm[(rb + lane) * 4 + qq] = mx;
      } else {
        uint32_t mk = 0u;
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          const uint32_t k = __reduce_max_sync(0xffffffffu, float_key(x[r]));
          mk = (lane == r) ? k : mk;
        }
        if (lane < NH) wm[(rb + lane) * 4 + qq] = float_of_key(mk);
      }
      gbar();
      float alpha[NH];
      bool grow_any = false;
      if constexpr (NH >= 8) {
        // lane l combines row l % NH alone (the unit max over the four
        // warps, the growth test, the factor); every lane then takes the
        // rows from their lanes
        const int rr = lane & (NH - 1);
        const float4 w4 = reinterpret_cast<const float4*>(wm)[rb + rr];
        const float M = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
        float mo = m_run[0];
#pragma unroll
        for (int r = 1; r < NH; ++r) mo = (rr == r) ? m_run[r] : mo;
        const bool grow = M > mo + kLazy;
        const float al = grow ? ex2(mo - M) : 1.f;     // 0 for the first keys of a row
        const float mn = grow ? M : mo;
        grow_any = __any_sync(0xffffffffu, grow);
#pragma unroll
        for (int r = 0; r < NH; ++r) m_run[r] = __shfl_sync(0xffffffffu, mn, r);
        if (grow_any) {
#pragma unroll
          for (int r = 0; r < NH; ++r) alpha[r] = __shfl_sync(0xffffffffu, al, r);
        } else {
#pragma unroll
          for (int r = 0; r < NH; ++r) alpha[r] = 1.f;
        }
      } else {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          const float4 w4 = reinterpret_cast<const float4*>(wm)[rb + r];
          const float M = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
          const bool grow = M > m_run[r] + kLazy;
          alpha[r] = grow ? ex2(m_run[r] - M) : 1.f;     // 0 for the first keys of a row
          m_run[r] = grow ? M : m_run[r];
          grow_any |= grow;
        }
      }
      if (grow_any) {
        if (!fi) {
          // O^T holds earlier units of this pair: wait for PV(i-1), rescale
          const int pj = i - 1;
          if (!mbar_wait_bounded(&p_free[pj & 1], (pj >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          float ov[NH];
          const uint32_t to = tl + 32 + (pc.ordinal & 1) * kN + rb;
          tmem_ldn<NH>(to, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < NH; ++r) ov[r] *= alpha[r];
          tmem_stn<NH>(to, ov);
          tc::tmem_wait_st();
          tc::fence_before_sync();
        }
#pragma unroll
        for (int r = 0; r < NH; ++r) l_t[r] *= alpha[r];
      }
      // P^T into this unit's P buffer once PV(i-2) has read it
      if (i >= 2 && !mbar_wait_bounded(&p_free[sb], ((i >> 1) + 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      unsigned char* pbuf = Ps + sb * kPBuf;
      float pm[NH];
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        const float p = ex2(x[r] - (m_run[r] == -CUDART_INF_F ? 0.f : m_run[r]));
        pm[r] = p;
        l_t[r] += p;
        *reinterpret_cast<__nv_bfloat16*>(pbuf + poff[r]) = __float2bfloat16_rn(p);
      }
      tc::fence_proxy_async_smem();
      mbar_arrive(&p_full[sb]);
      if constexpr (MASS) {
        // dense verify: this warp's 32 keys, when they are keys of the tile
        // (an empty tile has no key range) and lie in the complete blocks
        // (the dense mode's tiles start at multiples of 64): each row's
        // probability sum, reduce-scattered so that lane r holds the
        // warpgroup's row r (16 rows: lanes 0-15; at most 8: lanes 0-7)
        const int64_t k32 = kst + (qq & 1) * 32;
        if (n >= (qq & 1) * 32 + 32 && k32 + 32 <= a.mass_keys) {
          constexpr int W = NH > 8 ? 16 : 8;
          const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
          float e8[8], e4[4], e2[2];
          if constexpr (W == 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              e8[u] = (b3 ? pm[u + 8] : pm[u]) + __shfl_xor_sync(0xffffffffu, b3 ? pm[u] : pm[u + 8], 8);
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) e8[u] = u < NH ? pm[u < NH ? u : 0] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            e4[u] = (b2 ? e8[u + 4] : e8[u]) + __shfl_xor_sync(0xffffffffu, b2 ? e8[u] : e8[u + 4], 4);
#pragma unroll
          for (int u = 0; u < 2; ++u)
            e2[u] = (b1 ? e4[u + 2] : e4[u]) + __shfl_xor_sync(0xffffffffu, b1 ? e4[u] : e4[u + 2], 2);
          float e1 = (b0 ? e2[1] : e2[0]) + __shfl_xor_sync(0xffffffffu, b0 ? e2[0] : e2[1], 1);
          if constexpr (W == 8) e1 += __shfl_xor_sync(0xffffffffu, e1, 8);
          e1 += __shfl_xor_sync(0xffffffffu, e1, 16);
          const int r = lane & (W - 1);
          float mr = 0.f;
#pragma unroll
          for (int u = 0; u < NH; ++u) mr = (u == r && m_run[u] != -CUDART_INF_F) ? m_run[u] : mr;
          if (lane < W && r < NH && rb + r < R)
            a.mass_part[(pc.pair * a.mass_hts + k32 / 32) * 16 + rb + r] = make_float2(e1, mr);
        }
      }
      if (pc.last(i) && !epilogue()) {
        ok = false;
        break;
      }
    }
    if (!ok && lane == 0) fail();
  }

  // every warp reaches the final barrier converged (lane-0 drains above)
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 64);
  }
  if constexpr (FUSED) {
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned done = atomicAdd(a.exit_cnt, 1u);
      if (done == gridDim.x - 1) {
        // every CTA is past all its flag waits: clear the flags for the next call
        for (int p = 0; p < a.B * a.Hkv; ++p) a.ready[p] = 0u;
        __threadfence();
        *a.exit_cnt = 0u;
      }
    }
  }
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

size_t decode_tc_smem_bytes() { return kSmemBytes; }

TcOrder tc_order(int64_t pairs, int n_sink_tiles, int n_sel_tiles, int n_wc_tiles, bool split, int num_sms) {
  TcOrder o = {};
  const int64_t sms = std::max(num_sms, 1);
  int64_t pairs_i = pairs, pairs_d = pairs;
  if (split) {
    o.ntI = n_sink_tiles + n_wc_tiles;
    o.ntD = n_sel_tiles;
    o.dI = n_sel_tiles;
    o.dD = n_sink_tiles;
    o.pI = pairs;
  } else {
    // whole pairs first (the same number for every CTA), the rest split
    o.ntI = o.ntD = n_sink_tiles + n_sel_tiles + n_wc_tiles;
    o.pI = o.pD0 = (pairs / sms) * sms;
    pairs_i = o.pI;
    pairs_d = pairs - o.pI;
  }
  o.mI = (o.ntI + 1) / 2;
  o.mD = (o.ntD + 1) / 2;
  o.totI = pairs_i * o.mI;
  o.totD = pairs_d * o.mD;
  o.gI = static_cast<int>(std::min(sms, o.totI));
  o.gD = static_cast<int>(std::min(sms, o.totD));
  o.grid = std::max(std::max(o.gI, o.gD), 1);
  // CTAs a run of m units can touch when every CTA holds at least q units
  auto span = [](int m, int64_t tot, int g) -> int {
    if (m == 0 || g == 0) return 0;
    const int64_t q = tot / g;
    return 1 + static_cast<int>((m - 1 + q - 1) / q);
  };
  o.slots = std::max(span(o.mI, o.totI, o.gI) + span(o.mD, o.totD, o.gD), 1);
  return o;
}

bool decode_tc_supported(const DecodeAttnArgs& a) {
  return a.runs == nullptr && a.R >= 1 && a.R <= kN && a.kv_end < (int64_t(1) << 31) &&
         static_cast<int64_t>(a.B) * a.n_q < (int64_t(1) << 31) && encode_fn() != nullptr;
}

namespace {

bool encode_maps(const DecodeAttnArgs& a, CUtensorMap* qm, CUtensorMap* km, CUtensorMap* vm) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    // Q [B * n_q tokens][Hq heads][128]: box 64 columns x G heads x n_q tokens
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.Hq), static_cast<cuuint64_t>(a.B) * a.n_q};
    cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(a.Hq) * 256};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(a.G), static_cast<cuuint32_t>(a.n_q)};
    if (enc(qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.Q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  // K, V [pairs][cap keys][128], rows at or past kv_end read as zeros: box 64 columns x 64 keys
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.kv_end), static_cast<cuuint64_t>(a.B) * a.Hkv};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(a.cap) * 256};
  cuuint32_t box[3] = {64, 64, 1};
  if (enc(km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.K), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  return enc(vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.V), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FUSED>
cudaError_t launch_tc(const DecodeAttnArgs& a, const DecodePlan& p, bool out_bf16, cudaStream_t s) {
  CUtensorMap qm, km, vm;
  if (!encode_maps(a, &qm, &km, &vm)) return cudaErrorInvalidValue;
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, DecodeAttnArgs);
  // more than 8 rows: the 16-row instantiations, whose softmax rows are split
  // over two warpgroups
  const unsigned threads = FUSED ? kThreadsFused : (a.R > 8 ? kThreadsOf<16, false> : kThreads);
  if (!FUSED && a.mass_part) {
    // dense verify: the row sums of the complete blocks ride along
    if (a.R <= 4) kern = out_bf16 ? decode_tc_kernel<true, 4, false, true> : decode_tc_kernel<false, 4, false, true>;
    else if (a.R <= 8) kern = out_bf16 ? decode_tc_kernel<true, 8, false, true> : decode_tc_kernel<false, 8, false, true>;
    else kern = out_bf16 ? decode_tc_kernel<true, 16, false, true> : decode_tc_kernel<false, 16, false, true>;
  } else if (a.R <= 4) {
    kern = out_bf16 ? decode_tc_kernel<true, 4, FUSED, false> : decode_tc_kernel<false, 4, FUSED, false>;
  } else if constexpr (FUSED) {
    return cudaErrorInvalidValue;      // the fused step is built for at most 4 rows (decode_fused_supported)
  } else if (a.R <= 8) {
    kern = out_bf16 ? decode_tc_kernel<true, 8, false, false> : decode_tc_kernel<false, 8, false, false>;
  } else {
    kern = out_bf16 ? decode_tc_kernel<true, 16, false, false> : decode_tc_kernel<false, 16, false, false>;
  }
  const size_t smem = FUSED ? kSmemFused : kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.ord.grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (FUSED) {
    // every CTA resident at once: the per-pair flag waits depend on it
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = (FUSED || a.pdl) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, qm, km, vm, a);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeAttnArgs& a0, const DecodePlan& p, bool out_bf16, cudaStream_t s) {
  DecodeAttnArgs a = a0;
  a.ord = p.tc_plain;
  return launch_tc<0>(a, p, out_bf16, s);
}

bool decode_fused_supported(const DecodeAttnArgs& a, const DecodePlan& p, int64_t nb) {
  if (nb < 1 || nb > kMaxSelectBlocks || !decode_tc_supported(a)) return false;
  const int64_t pairs = static_cast<int64_t>(a.B) * a.Hkv;
  const int64_t cpp = (nb + 127) / 128;
  const int64_t chunks = pairs * cpp;
  const int grid = p.tc_split.grid;
  if (grid < 1) return false;
  if (nb > kFusedMaxBlocks) {
    // past 512 blocks: runs of at most kFusedRunChunks chunks publish their
    // own top k (k <= kFusedSmallK) into at most kFusedCandSlots slots a pair
    const int64_t cpc = (chunks + grid - 1) / grid;
    if (a.top_k > kFusedSmallK || cpc > kFusedRunChunks || (cpp + cpc - 1) / cpc + 1 > kFusedCandSlots) return false;
  }
  // Measured on B200: with more than 4 query rows per KV head (draft chunks)
  // or more than two pairs per CTA, the per-pair partial results of the two
  // split lists cost more than the second launch saves, and the scoring
  // kernel + attention kernel (whole pairs first) is faster.
  if (a.R > 4 || pairs > 2 * static_cast<int64_t>(grid)) return false;
  // at most one CTA per SM (shared memory), at most kMaxSelPerCta tickets per CTA
  return a.total_tiles > 0 && grid > 0 && (chunks + grid - 1) / grid <= kMaxSelPerCta;
}

cudaError_t launch_decode_fused(DecodeAttnArgs a, const DecodePlan& p, bool out_bf16, cudaStream_t s) {
  a.ord = p.tc_split;
  a.cpp = static_cast<int>((a.nb + 127) / 128);
  const int total_chunks = a.B * a.Hkv * a.cpp;
  a.cpc = (total_chunks + a.ord.grid - 1) / a.ord.grid;
  a.idx = a.idx_w;
  a.idx_stride = a.top_k;
  a.pdl = 0;
  return a.nb <= kFusedMaxBlocks ? launch_tc<1>(a, p, out_bf16, s) : launch_tc<2>(a, p, out_bf16, s);
}

}  // namespace sa
