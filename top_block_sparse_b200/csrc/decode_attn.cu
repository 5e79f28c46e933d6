// Step 4 for decode and draft chunks: softmax attention over the retained
// keys only (S3R review, section "稀疏起草": softmax over K_T and weighted sum
// of V_T for the retained index set T; PulseCol §3.1 eq. (1)-(2): logits
// q.k/sqrt(d_h), keys outside the mask get zero weight).
//
// Retained set of (sequence, KV head) for new token j:
//   sink [0, s_end)  U  selected blocks (minus keys already in sink/window)
//   U  window [w_begin, C)  U  new keys [C, C + j]
// (SparDA summary "方法": initial tokens + local window + top-k blocks; a
// draft chunk keeps one selection for all its tokens, S3R review).
//
// Work decomposition (B200): every (sequence, KV head) pair is a list of MT
// "tiles" of <= 64 contiguous keys: sink tiles, tpb tiles per selected block,
// window+new-key tiles.  The flattened list over all pairs is cut into equal
// contiguous ranges, one per CTA, one CTA per SM (stream-K), so every SM
// streams the same number of bytes whatever k, b or the batch are.
//
// Per CTA: one producer thread issues 1-D bulk copies (cp.async.bulk, the TMA
// engine) of each tile's K rows and V rows (contiguous in [B,Hkv,T,d]) into an
// n_stages-deep shared-memory ring guarded by mbarriers; RG*KG consumer warps
// compute.  Warp (rg, kg) owns query rows 4rg..4rg+3 of the pair and keys
// [kg*KPW, kg*KPW + KPW) of every tile, and keeps its own online-softmax
// state (fp32 max, sum, 4x128 accumulator).  QK: 8 lanes share a key, each
// lane holds 16 of the 128 coordinates of the 4 pre-scaled query rows in
// registers; a 3-level reduce-scatter leaves one (row, key) logit per lane.
// PV: each lane owns 4 output columns of the 4 rows.  No tensor cores: at
// 2*G FLOP per K/V byte the work is bound by HBM, not by FMA throughput.
//
// Combine: at the end of a pair segment the KG warps of a row group merge
// through shared memory (max / log-sum-exp rescaling).  A CTA that holds a
// whole pair writes O and lse; otherwise it writes an unnormalised partial
// (O, max, sum) to the workspace and takes an atomic ticket; the CTA that
// arrives last for the pair merges all partials and resets the ticket.
// Nothing ever waits on another CTA.
#include <algorithm>
#include <math_constants.h>

#include "common.cuh"
#include "decode_units.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kCombStride = 132;   // floats per (row) in the combine buffer: 128 O + m + l + pad

__device__ __forceinline__ void consumer_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

typedef unsigned long long u64;

// Packed fp32 pairs (sm_100 f32x2 arithmetic halves the FMA instruction count).
__device__ __forceinline__ u64 pk2(float x, float y) {
  u64 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float lo2(u64 v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(u64 v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// two bf16 (one 32-bit word) -> packed fp32 pair
__device__ __forceinline__ u64 bf2(uint32_t w) { return pk2(bf16lo(w), bf16hi(w)); }

// Loads this lane's 16 coordinates of one key row as packed fp32 pairs.
template <bool BF16>
__device__ __forceinline__ void load_key(const unsigned char* krow, int l8, u64 (&kp)[8]) {
  if constexpr (BF16) {
    const uint4 u0 = *reinterpret_cast<const uint4*>(krow + l8 * 16);
    const uint4 u1 = *reinterpret_cast<const uint4*>(krow + 128 + l8 * 16);
    kp[0] = bf2(u0.x); kp[1] = bf2(u0.y); kp[2] = bf2(u0.z); kp[3] = bf2(u0.w);
    kp[4] = bf2(u1.x); kp[5] = bf2(u1.y); kp[6] = bf2(u1.z); kp[7] = bf2(u1.w);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(krow + 128 * c + l8 * 16);
      kp[2 * c] = x.x;
      kp[2 * c + 1] = x.y;
    }
  }
}

// QK partial sums of two key rows over this lane's 16 coordinates for the 4
// query-row slots: v[4*key + x] = sum_e q[x][e] * k_key[e].  Even and odd
// coordinate pairs go to separate accumulators so that the two keys give 16
// independent FMA chains of length 4.
template <bool BF16>
__device__ __forceinline__ void qk_two_keys(const unsigned char* krow_a, const unsigned char* krow_b, int l8,
                                            const u64 (&q2)[4][8], float (&v)[8]) {
  u64 ka[8], kb[8];
  load_key<BF16>(krow_a, l8, ka);
  load_key<BF16>(krow_b, l8, kb);
  u64 acc[2][4][2];
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    acc[0][x][0] = 0ull; acc[0][x][1] = 0ull;
    acc[1][x][0] = 0ull; acc[1][x][1] = 0ull;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      acc[0][x][e & 1] = fma2(q2[x][e], ka[e], acc[0][x][e & 1]);
      acc[1][x][e & 1] = fma2(q2[x][e], kb[e], acc[1][x][e & 1]);
    }
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    v[x] = (lo2(acc[0][x][0]) + hi2(acc[0][x][0])) + (lo2(acc[0][x][1]) + hi2(acc[0][x][1]));
    v[4 + x] = (lo2(acc[1][x][0]) + hi2(acc[1][x][0])) + (lo2(acc[1][x][1]) + hi2(acc[1][x][1]));
  }
}

// Run mode: entry e of gathered tile `sl` of `pair` (rpt entries per tile).
// Returns the number of keys of its run inside [s_end, w_begin) and their
// first key in *start (0 keys for -1 entries and entries past the row).
__device__ __forceinline__ int run_entry(const DecodeAttnArgs& a, int64_t pair, int sl, int e, int rpt,
                                         int64_t* start) {
  const int64_t at = static_cast<int64_t>(sl) * rpt + e;
  const int32_t m = (e < rpt && at < a.runs_stride) ? __ldg(a.runs + pair * a.runs_stride + at) : -1;
  *start = 0;
  if (m < 0) return 0;
  const int64_t lo = max(static_cast<int64_t>(m) * a.run_len, a.s_end);
  const int64_t hi = min(static_cast<int64_t>(m) * a.run_len + a.run_len, a.w_begin);
  *start = lo;
  return hi > lo ? static_cast<int>(hi - lo) : 0;
}

// Key position given to gathered tiles: below every context key, so the
// causal rule of the new tokens never applies to them.
constexpr int64_t kRunTilePos = -(int64_t(1) << 40);

template <bool BF16, bool OUT_BF16, int RG, int KG>
__global__ void __launch_bounds__((RG * KG + 1) * 32, 1) decode_attn_kernel(DecodeAttnArgs a) {
  constexpr int NWC = RG * KG;                 // consumer warps
  constexpr int NCT = NWC * 32;                // consumer threads
  constexpr int HALF = BF16 ? 64 : 32;         // keys per tile; a ring stage holds two tiles
  constexpr int KPH = HALF / KG;               // keys per warp per tile
  constexpr int NITH = KPH / 8;                // QK iterations per tile (8 keys per warp-iteration)
  constexpr int NIT = 2 * NITH;
  constexpr int KPR = 2 * KPH;                 // keys per warp per round (two tiles)
  constexpr int ROWB = BF16 ? 256 : 512;       // bytes per K/V row
  constexpr int KBYTES = 2 * HALF * ROWB;      // K part of a stage
  constexpr int STAGE = 2 * KBYTES;
  static_assert(KPH % 8 == 0, "a warp takes a multiple of 8 keys of every tile");

  extern __shared__ __align__(1024) unsigned char smem[];
  const int NS = a.n_stages;
  unsigned char* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NS) * STAGE);
  uint64_t* empty = full + NS;
  StageInfo* info = reinterpret_cast<StageInfo*>(empty + NS);
  u64* pbuf = reinterpret_cast<u64*>(info + NS);                     // [NWC][KPR][4] (p, p) pairs
  float* rowbuf = reinterpret_cast<float*>(pbuf + NWC * KPR * 4);    // [NWC][4] row scale factors
  float* comb = rowbuf + NWC * 4;                                    // [KG][RG*4][kCombStride]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(comb + KG * RG * 4 * kCombStride);
  int* ticket = const_cast<int*>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * a.tpc;       // work units = tile pairs
  const int64_t u1 = min(a.total_tiles, u0 + a.tpc);
  const int nunits = static_cast<int>(u1 - u0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NWC);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // everything above overlaps the tail of the scoring kernel; the index table
  // it writes is read only after this point
  if (a.pdl) pdl_wait_prior_grid();

  if (warp == NWC) {
    // ------------------------------------------------------------ producer
    // The warp computes the key ranges of 32 units at a time (one per lane,
    // index loads in parallel); lane 0 then feeds them to the ring in order.
    int issued = 0;
    bool stop = false;
    for (int base = 0; base < nunits && !stop; base += 32) {
      int64_t ks0 = 0, ks1 = 0;
      int nk0 = 0, nk1 = 0;
      if (base + lane < nunits) {
        const int64_t u = u0 + base + lane;
        const int64_t pair = u / a.MT;
        const int v = static_cast<int>(u - pair * a.MT);
        tile_range(a, pair, 2 * v, &ks0, &nk0);
        if (2 * v + 1 < a.n_tiles) tile_range(a, pair, 2 * v + 1, &ks1, &nk1);
      }
      const int cnt = min(32, nunits - base);
      for (int l = 0; l < cnt; ++l) {
        const int64_t k0 = __shfl_sync(0xffffffffu, ks0, l);
        const int64_t k1 = __shfl_sync(0xffffffffu, ks1, l);
        const int n0 = __shfl_sync(0xffffffffu, nk0, l);
        const int n1 = __shfl_sync(0xffffffffu, nk1, l);
        const int i = base + l;
        const int s = i % NS;
        const int64_t pair = (u0 + i) / a.MT;
        unsigned char* st = stages + static_cast<size_t>(s) * STAGE;
        const unsigned char* kb = static_cast<const unsigned char*>(a.K) + pair * a.cap * ROWB;
        const unsigned char* vb = static_cast<const unsigned char*>(a.V) + pair * a.cap * ROWB;
        // run mode: tiles of the selected section are packed from key runs
        // by the whole warp (their sizes first, the copies after the barrier
        // expects their bytes)
        bool gat[2] = {false, false};
        int sl[2] = {0, 0};
        int tot[2] = {n0, n1};
        const int rpt = a.runs ? HALF / a.run_len : 0;
        if (a.runs) {
          const int v = static_cast<int>((u0 + i) - pair * a.MT);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            sl[h] = 2 * v + h - a.n_sink_tiles;
            gat[h] = (2 * v + h < a.n_tiles) && sl[h] >= 0 && sl[h] < a.idx_stride;
            if (!gat[h]) continue;
            int t = 0;
            for (int c0 = 0; c0 < rpt; c0 += 32) {
              int64_t st0;
              const int len = run_entry(a, pair, sl[h], c0 + lane, rpt, &st0);
              t += __reduce_add_sync(0xffffffffu, static_cast<unsigned>(len));
            }
            tot[h] = t;
          }
        }
        int ok = 1;
        if (lane == 0) {
          if (i >= NS && !mbar_wait_bounded(&empty[s], ((i / NS) & 1) ^ 1, abort_flag)) ok = 0;
          if (ok && *abort_flag) ok = 0;
          if (ok) {
            info[s].ks0 = gat[0] ? kRunTilePos : k0;
            info[s].ks1 = gat[1] ? kRunTilePos : k1;
            info[s].n0 = tot[0];
            info[s].n1 = tot[1];
            if (tot[0] + tot[1] > 0) {
              mbar_arrive_expect_tx(&full[s], 2u * static_cast<uint32_t>(tot[0] + tot[1]) * ROWB);
              if (!gat[0] && n0 > 0) {
                bulk_g2s(st, kb + k0 * ROWB, n0 * ROWB, &full[s]);
                bulk_g2s(st + KBYTES, vb + k0 * ROWB, n0 * ROWB, &full[s]);
              }
              if (!gat[1] && n1 > 0) {
                bulk_g2s(st + HALF * ROWB, kb + k1 * ROWB, n1 * ROWB, &full[s]);
                bulk_g2s(st + KBYTES + HALF * ROWB, vb + k1 * ROWB, n1 * ROWB, &full[s]);
              }
            } else {
              mbar_arrive(&full[s]);
            }
          } else {
            report(a.status, kStatusTimeout);
            *abort_flag = 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          stop = true;
          break;
        }
        __syncwarp();
        if (gat[0] || gat[1]) {
          // each lane copies its runs' K and V rows to the packed positions
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!gat[h]) continue;
            int carry = 0;
            for (int c0 = 0; c0 < rpt; c0 += 32) {
              int64_t ks;
              const int len = run_entry(a, pair, sl[h], c0 + lane, rpt, &ks);
              int incl = len;
#pragma unroll
              for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
              }
              const int off = carry + incl - len;
              if (len > 0) {
                const uint32_t by = static_cast<uint32_t>(len) * ROWB;
                bulk_g2s(st + (h * HALF + off) * ROWB, kb + ks * ROWB, by, &full[s]);
                bulk_g2s(st + KBYTES + (h * HALF + off) * ROWB, vb + ks * ROWB, by, &full[s]);
              }
              carry += __shfl_sync(0xffffffffu, incl, 31);
            }
          }
        }
        issued = i + 1;
      }
    }
    // do not leave while copies into this CTA's shared memory may be in flight
    if (lane == 0)
      for (int i = max(0, issued - NS); i < issued; ++i) mbar_wait_bounded(&full[i % NS], (i / NS) & 1, nullptr);
    return;
  }

  // ------------------------------------------------------------- consumers
  const int rg = warp / KG, kg = warp - (warp / KG) * KG;
  const int gi = lane >> 3, l8 = lane & 7;
  const int m8 = l8 & 3;             // this lane's row after the reduce-scatter
  const int b2 = l8 >> 2;            // this lane's key (of the group's pair) after it
  u64* my_p = pbuf + warp * KPR * 4;
  float* my_row = rowbuf + warp * 4;

  // q2[x] holds query row rg*4 + (x ^ m8): with the rows permuted per lane the
  // reduce-scatter below needs no selects.
  u64 q2[4][8];
  u64 o2[4][2];                      // rows rg*4+r, columns 4*lane..4*lane+3 as two pairs
  float m_own = -CUDART_INF_F;       // running max of row rg*4 + m8 (same on all its lanes)
  float l_own = 0.f;                 // this lane's share of that row's running sum
  int64_t cur_pair = -1;

  auto load_q = [&](int64_t pair) {
    const int bi = static_cast<int>(pair / a.Hkv), h = static_cast<int>(pair % a.Hkv);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int rr = rg * 4 + (x ^ m8);
      float qf[16];
      if (rr < a.R) {
        const int j = rr / a.G, g = rr - (rr / a.G) * a.G;
        const int64_t off = ((static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * a.G + g) * kHeadDim;
        if constexpr (BF16) {
          const uint16_t* qp = static_cast<const uint16_t*>(a.Q) + off;
          unpack8(__ldg(reinterpret_cast<const uint4*>(qp + 8 * l8)), qf);
          unpack8(__ldg(reinterpret_cast<const uint4*>(qp + 64 + 8 * l8)), qf + 8);
        } else {
          const float* qp = static_cast<const float*>(a.Q) + off;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(qp + 32 * c + 4 * l8));
            qf[4 * c + 0] = v.x; qf[4 * c + 1] = v.y; qf[4 * c + 2] = v.z; qf[4 * c + 3] = v.w;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) qf[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) q2[x][e] = pk2(qf[2 * e] * a.qscale, qf[2 * e + 1] * a.qscale);
    }
    m_own = -CUDART_INF_F;
    l_own = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      o2[r][0] = 0ull;
      o2[r][1] = 0ull;
    }
  };

  auto write_out = [&](int64_t orow, int c4, float4 acc, float inv) {
    if constexpr (OUT_BF16) {
      uint2 pk = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.O) + orow * kHeadDim + 4 * c4) = pk;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow * kHeadDim + 4 * c4) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
  };

  // Merge the KG warps of every row group and emit this CTA's result for `pair`.
  auto flush = [&](int64_t pair) {
    // the row sums are spread over the 8 lanes that hold each row
    float l_row = l_own;
    l_row += __shfl_xor_sync(0xffffffffu, l_row, 4);
    l_row += __shfl_xor_sync(0xffffffffu, l_row, 8);
    l_row += __shfl_xor_sync(0xffffffffu, l_row, 16);
    float* cb = comb + (kg * RG * 4) * kCombStride;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int rr = rg * 4 + r;
      *reinterpret_cast<float4*>(cb + rr * kCombStride + 4 * lane) =
          make_float4(lo2(o2[r][0]), hi2(o2[r][0]), lo2(o2[r][1]), hi2(o2[r][1]));
    }
    if (lane < 4) {                   // lane r holds row rg*4 + r (gi = 0, b2 = 0, m8 = r)
      cb[(rg * 4 + lane) * kCombStride + 128] = m_own;
      cb[(rg * 4 + lane) * kCombStride + 129] = l_row;
    }
    consumer_bar(NCT);
    const int64_t first = pair * a.MT, last = first + a.MT - 1;
    const bool whole = first >= u0 && last < u1;
    const int64_t first_cta = first / a.tpc, last_cta = last / a.tpc;
    const int n_ctas = static_cast<int>(last_cta - first_cta + 1);
    const int slot = static_cast<int>(blockIdx.x - first_cta);
    const int bi = static_cast<int>(pair / a.Hkv), h = static_cast<int>(pair % a.Hkv);
    for (int item = threadIdx.x; item < a.R * 32; item += NCT) {
      const int rr = item >> 5, c4 = item & 31;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < KG; ++w) M = fmaxf(M, comb[(w * RG * 4 + rr) * kCombStride + 128]);
      const float Mr = (M == -CUDART_INF_F) ? 0.f : M;
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < KG; ++w) {
        const float* e = comb + (w * RG * 4 + rr) * kCombStride;
        const float sc = exp2f(e[128] - Mr);
        L += e[129] * sc;
        const float4 v = *reinterpret_cast<const float4*>(e + 4 * c4);
        acc.x += v.x * sc; acc.y += v.y * sc; acc.z += v.z * sc; acc.w += v.w * sc;
      }
      if (whole) {
        const int j = rr / a.G, g = rr - (rr / a.G) * a.G;
        const int64_t orow = (static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * a.G + g;
        write_out(orow, c4, acc, L > 0.f ? 1.f / L : 0.f);
        if (c4 == 0 && a.lse)
          a.lse[orow] = L > 0.f ? (Mr + log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
      } else {
        const int64_t ps = (pair * a.n_slots + slot) * a.R4 + rr;
        *reinterpret_cast<float4*>(a.part_O + ps * kHeadDim + 4 * c4) = acc;
        if (c4 == 0) {
          a.part_ml[ps * 2 + 0] = M;
          a.part_ml[ps * 2 + 1] = L;
        }
      }
    }
    if (!whole) {
      // the barrier orders every consumer's partial stores before thread 0's
      // release fence and ticket
      consumer_bar(NCT);
      if (threadIdx.x == 0) {
        __threadfence();
        const unsigned t = atomicAdd(&a.counters[pair], 1u);
        *ticket = (t == static_cast<unsigned>(n_ctas - 1));
      }
      consumer_bar(NCT);
      if (*ticket) {
        __threadfence();
        for (int item = threadIdx.x; item < a.R * 32; item += NCT) {
          const int rr = item >> 5, c4 = item & 31;
          float M = -CUDART_INF_F;
          for (int s2 = 0; s2 < n_ctas; ++s2)
            M = fmaxf(M, __ldcg(a.part_ml + ((pair * a.n_slots + s2) * a.R4 + rr) * 2));
          const float Mr = (M == -CUDART_INF_F) ? 0.f : M;
          float L = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int s2 = 0; s2 < n_ctas; ++s2) {
            const int64_t ps = (pair * a.n_slots + s2) * a.R4 + rr;
            const float sc = exp2f(__ldcg(a.part_ml + ps * 2) - Mr);
            L += __ldcg(a.part_ml + ps * 2 + 1) * sc;
            const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_O + ps * kHeadDim) + c4);
            acc.x += v.x * sc; acc.y += v.y * sc; acc.z += v.z * sc; acc.w += v.w * sc;
          }
          const int j = rr / a.G, g = rr - (rr / a.G) * a.G;
          const int64_t orow = (static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * a.G + g;
          write_out(orow, c4, acc, L > 0.f ? 1.f / L : 0.f);
          if (c4 == 0 && a.lse)
            a.lse[orow] = L > 0.f ? (Mr + log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
        }
        if (threadIdx.x == 0) a.counters[pair] = 0u;
      }
    }
    consumer_bar(NCT);   // the combine buffer is reused by the next segment
  };

  const int tok = (rg * 4 + m8) / a.G;   // new-token index of this lane's row
  bool aborted = false;
  for (int i = 0; i < nunits; ++i) {
    const int64_t pair = (u0 + i) / a.MT;
    if (pair != cur_pair) {
      if (cur_pair >= 0) flush(cur_pair);
      cur_pair = pair;
      load_q(pair);
    }
    const int s = i % NS;
    if (!aborted && !mbar_wait_bounded(&full[s], (i / NS) & 1, abort_flag)) {
      aborted = true;
      if (lane == 0) {
        report(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
    }
    const int n0 = aborted ? 0 : info[s].n0;
    const int n1 = aborted ? 0 : info[s].n1;
    const int64_t ks0 = info[s].ks0, ks1 = info[s].ks1;
    const int kb = kg * KPH;                  // this warp's first key in each tile
    const int nk0 = min(KPH, n0 - kb), nk1 = min(KPH, n1 - kb);
    if (nk0 > 0 || nk1 > 0) {
      const unsigned char* kst = stages + static_cast<size_t>(s) * STAGE;
      const unsigned char* vst = kst + KBYTES;
      float sc[NIT];
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const int half = it / NITH;
        const int kl = kb + (it % NITH) * 8 + 2 * gi;    // group's first key within the tile
        const unsigned char* kt = kst + half * HALF * ROWB;
        // this lane computes its own key (kl + b2) first, so the first
        // reduce-scatter level keeps v[0..3] and sends v[4..7] on every lane
        float v[8];
        qk_two_keys<BF16>(kt + (kl + b2) * ROWB, kt + (kl + (b2 ^ 1)) * ROWB, l8, q2, v);
        float w4[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) w4[x] = v[x] + __shfl_xor_sync(0xffffffffu, v[4 + x], 4);
        float w2[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) w2[x] = w4[x] + __shfl_xor_sync(0xffffffffu, w4[2 + x], 2);
        const float w1 = w2[0] + __shfl_xor_sync(0xffffffffu, w2[1], 1);
        // this lane now holds the logit of key kl + b2 of tile `half`, row rg*4 + m8
        const int key = kl + b2;
        const int nh = half ? n1 : n0;
        const int64_t pos = (half ? ks1 : ks0) + key;
        bool valid = key < nh;
        if (pos >= a.C) valid = valid && (pos - a.C) <= tok;
        sc[it] = valid ? w1 : -CUDART_INF_F;
      }
      float mx = sc[0];
#pragma unroll
      for (int it = 1; it < NIT; ++it) mx = fmaxf(mx, sc[it]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_own, mx);
      const float m_ref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
      const float alpha = exp2f(m_own - m_ref);
      float ps = 0.f;
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const float p = exp2f(sc[it] - m_ref);
        ps += p;
        my_p[(it * 8 + 2 * gi + b2) * 4 + m8] = pk2(p, p);
      }
      l_own = l_own * alpha + ps;
      const bool grew = m_new != m_own;          // only then does a row's scale change
      m_own = m_new;
      if (lane < 4) my_row[lane] = alpha;
      __syncwarp();
      if (__any_sync(0xffffffffu, grew)) {
        const float4 al = *reinterpret_cast<const float4*>(my_row);
        const u64 a0 = pk2(al.x, al.x), a1 = pk2(al.y, al.y), a2 = pk2(al.z, al.z), a3 = pk2(al.w, al.w);
        o2[0][0] = mul2(o2[0][0], a0); o2[0][1] = mul2(o2[0][1], a0);
        o2[1][0] = mul2(o2[1][0], a1); o2[1][1] = mul2(o2[1][1], a1);
        o2[2][0] = mul2(o2[2][0], a2); o2[2][1] = mul2(o2[2][1], a2);
        o2[3][0] = mul2(o2[3][0], a3); o2[3][1] = mul2(o2[3][1], a3);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int nk = half ? nk1 : nk0;
        const unsigned char* vt = vst + half * HALF * ROWB + kb * ROWB;
        const u64* pt = my_p + half * KPH * 4;
#pragma unroll 4
        for (int kk = 0; kk < nk; ++kk) {
          const ulonglong2 p01 = *reinterpret_cast<const ulonglong2*>(pt + kk * 4);
          const ulonglong2 p23 = *reinterpret_cast<const ulonglong2*>(pt + kk * 4 + 2);
          const unsigned char* vrow = vt + kk * ROWB;
          u64 v0, v1;
          if constexpr (BF16) {
            const uint2 u = *reinterpret_cast<const uint2*>(vrow + lane * 8);
            v0 = bf2(u.x);
            v1 = bf2(u.y);
          } else {
            const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(vrow + lane * 16);
            v0 = x.x;
            v1 = x.y;
          }
          o2[0][0] = fma2(p01.x, v0, o2[0][0]); o2[0][1] = fma2(p01.x, v1, o2[0][1]);
          o2[1][0] = fma2(p01.y, v0, o2[1][0]); o2[1][1] = fma2(p01.y, v1, o2[1][1]);
          o2[2][0] = fma2(p23.x, v0, o2[2][0]); o2[2][1] = fma2(p23.x, v1, o2[2][1]);
          o2[3][0] = fma2(p23.y, v0, o2[3][0]); o2[3][1] = fma2(p23.y, v1, o2[3][1]);
        }
      }
      __syncwarp();
    }
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (cur_pair >= 0) flush(cur_pair);
}

// Caller index tables (sa_sparse_attn_given_idx): an entry is kept only if it
// is a complete-block id larger than every earlier in-range entry of its row,
// so no key is attended twice; other entries become -1 and, unless they were
// -1 already, set kStatusIndex.  One warp per row, a max-scan per 32 entries.
__global__ void __launch_bounds__(256) sanitize_idx_kernel(const int32_t* idx, int32_t* out, int rows,
                                                           int len, int64_t nb, unsigned* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int32_t* in = idx + static_cast<int64_t>(row) * len;
  int32_t* o = out + static_cast<int64_t>(row) * len;
  int carry = -1;
  bool bad = false;
  for (int base = 0; base < len; base += 32) {
    const int s = base + lane;
    const int32_t j = s < len ? __ldg(in + s) : -1;
    const bool in_range = j >= 0 && j < nb;
    int incl = in_range ? j : -1;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl = max(incl, y);
    }
    int excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = -1;
    excl = max(excl, carry);
    const bool ok = in_range && j > excl;
    if (s < len) {
      o[s] = ok ? j : -1;
      if (!ok && j != -1) bad = true;
    }
    carry = max(carry, __shfl_sync(0xffffffffu, incl, 31));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, kStatusIndex);
}

// Caller prefill tables: row (pair, tile t) may list blocks j < t (complete
// blocks before the tile); an entry is kept if it is above every earlier
// in-range entry of the row and is not one of the tile's sink / window blocks
// (their keys are attended anyway).  Entries >= t or < -1, and repeated or
// descending ones, set kStatusIndex.
__global__ void __launch_bounds__(256) sanitize_prefill_idx_kernel(const int32_t* idx, int32_t* out, int P,
                                                                   int n_tiles, int len, int64_t S, int64_t W,
                                                                   unsigned* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= P * n_tiles) return;
  const int t = row % n_tiles;
  const int64_t C = static_cast<int64_t>(t) * 64;
  const int64_t s_end = S < C ? S : C;
  const int64_t w_begin = (C - W) > s_end ? (C - W) : s_end;
  const int lo = static_cast<int>(s_end / 64), hi = static_cast<int>(w_begin / 64);
  const int32_t* in = idx + static_cast<int64_t>(row) * len;
  int32_t* o = out + static_cast<int64_t>(row) * len;
  int carry = -1;
  bool bad = false;
  for (int base = 0; base < len; base += 32) {
    const int s = base + lane;
    const int32_t j = s < len ? __ldg(in + s) : -1;
    const bool in_range = j >= 0 && j < t;
    int incl = in_range ? j : -1;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl = max(incl, y);
    }
    int excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = -1;
    excl = max(excl, carry);
    const bool ok = in_range && j > excl;
    if (s < len) {
      o[s] = (ok && j >= lo && j < hi) ? j : -1;
      if (!ok && j != -1) bad = true;
    }
    carry = max(carry, __shfl_sync(0xffffffffu, incl, 31));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, kStatusIndex);
}

template <bool BF16, bool OUT_BF16, int RG, int KG>
cudaError_t launch_one(const DecodeAttnArgs& a, const DecodePlan& p, cudaStream_t s) {
  auto kern = decode_attn_kernel<BF16, OUT_BF16, RG, KG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(p.smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(p.threads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool BF16, bool OUT_BF16>
cudaError_t launch_rg(const DecodeAttnArgs& a, const DecodePlan& p, cudaStream_t s) {
  constexpr int H = BF16 ? 64 : 32;
  switch (p.RG) {
    case 1: return launch_one<BF16, OUT_BF16, 1, H / 8>(a, p, s);
    case 2: return launch_one<BF16, OUT_BF16, 2, H / 16>(a, p, s);
    case 3: return launch_one<BF16, OUT_BF16, 3, H / 16>(a, p, s);
    case 4: return launch_one<BF16, OUT_BF16, 4, (H / 32 < 1 ? 1 : H / 32)>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_smem_bytes(int RG, int KG, bool bf16, int n_stages) {
  const int NWC = RG * KG;
  const int half = bf16 ? 64 : 32;
  const int KPR = 2 * (half / KG);
  const size_t stage = 2 * 2 * half * (bf16 ? 256 : 512);
  size_t b = stage * n_stages;
  b += 2 * sizeof(uint64_t) * n_stages;
  b += sizeof(StageInfo) * n_stages;
  b += sizeof(unsigned long long) * NWC * KPR * 4;
  b += sizeof(float) * NWC * 4;
  b += sizeof(float) * KG * RG * 4 * kCombStride;
  b += 16;
  return b;
}

// Consumer warp layout: RG groups of 4 query rows, KG warps per group; every
// warp takes 8, 16 or 32 keys of each tile.
static int kg_for(int RG, bool bf16) {
  const int half = bf16 ? 64 : 32;
  const int kg = RG == 1 ? half / 8 : (RG == 4 ? half / 32 : half / 16);
  return kg < 1 ? 1 : kg;
}

bool plan_decode(const DecodeGeom& g, int idx_slots, bool bf16, int num_sms, DecodePlan* p,
                 const char** why) {
  p->R = g.R;
  p->RG = (g.R + 3) / 4;
  if (p->RG < 1 || p->RG > 4) {
    *why = "n_q * (num_q_heads / num_kv_heads) must be in [1, 16]";
    return false;
  }
  p->R4 = p->RG * 4;
  p->KG = kg_for(p->RG, bf16);
  p->threads = (p->RG * p->KG + 1) * 32;
  p->tile = bf16 ? 64 : 32;
  const int T = p->tile;
  p->n_sink_tiles = static_cast<int>((g.s_end + T - 1) / T);
  p->tpb = (g.b + T - 1) / T;
  p->n_wc_tiles = static_cast<int>((g.kv_end - g.w_begin + T - 1) / T);
  const int64_t nt = static_cast<int64_t>(p->n_sink_tiles) + static_cast<int64_t>(idx_slots) * p->tpb +
                     p->n_wc_tiles;
  if (nt > (1 << 24)) {
    *why = "too many key tiles per (sequence, KV head)";
    return false;
  }
  p->n_tiles = static_cast<int>(nt);
  p->MT = static_cast<int>((nt + 1) / 2);            // work units (tile pairs) per pair
  p->total_tiles = static_cast<int64_t>(g.pairs) * p->MT;
  const int64_t max_grid = num_sms;
  int64_t grid = p->total_tiles < max_grid ? p->total_tiles : max_grid;
  if (grid < 1) grid = 1;
  int64_t tpc = (p->total_tiles + grid - 1) / grid;
  if (tpc < 1) tpc = 1;
  if (tpc > (1 << 30)) {
    *why = "problem too large";
    return false;
  }
  p->tpc = static_cast<int>(tpc);
  p->grid = static_cast<int>((p->total_tiles + tpc - 1) / tpc);
  if (p->grid < 1) p->grid = 1;
  p->n_slots = static_cast<int>((p->MT + tpc - 1) / tpc) + 1;
  const int sel_tiles = idx_slots * p->tpb;
  p->tc_plain = tc_order(g.pairs, p->n_sink_tiles, sel_tiles, p->n_wc_tiles, false, num_sms);
  p->tc_split = tc_order(g.pairs, p->n_sink_tiles, sel_tiles, p->n_wc_tiles, true, num_sms);
  p->n_slots = std::max(p->n_slots, std::max(p->tc_plain.slots, p->tc_split.slots));
  const size_t limit = 227 * 1024;
  int ns = 3;
  while (ns > 1 && decode_smem_bytes(p->RG, p->KG, bf16, ns) > limit) --ns;
  p->n_stages = ns;
  p->smem = decode_smem_bytes(p->RG, p->KG, bf16, ns);
  if (p->smem > limit) {
    *why = "shared memory plan exceeds 227 KB";
    return false;
  }
  return true;
}

cudaError_t launch_sanitize_idx(const int32_t* idx, int32_t* out, int rows, int len, int64_t nb,
                                unsigned* status, cudaStream_t s) {
  if (rows == 0 || len == 0) return cudaSuccess;
  sanitize_idx_kernel<<<(rows + 7) / 8, 256, 0, s>>>(idx, out, rows, len, nb, status);
  return cudaGetLastError();
}

cudaError_t launch_sanitize_prefill_idx(const int32_t* idx, int32_t* out, int P, int n_tiles, int len,
                                        int64_t S, int64_t W, unsigned* status, cudaStream_t s) {
  const int rows = P * n_tiles;
  if (rows == 0 || len == 0) return cudaSuccess;
  sanitize_prefill_idx_kernel<<<(rows + 7) / 8, 256, 0, s>>>(idx, out, P, n_tiles, len, S, W, status);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const DecodeAttnArgs& a, const DecodePlan& p, bool bf16, bool out_bf16,
                               cudaStream_t s) {
  if (p.total_tiles == 0) return cudaSuccess;
  if (bf16 && decode_tc_supported(a)) return launch_decode_tc(a, p, out_bf16, s);
  if (bf16) return out_bf16 ? launch_rg<true, true>(a, p, s) : launch_rg<true, false>(a, p, s);
  return out_bf16 ? launch_rg<false, true>(a, p, s) : launch_rg<false, false>(a, p, s);
}

}  // namespace sa
