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
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kCombStride = 132;   // floats per (row) in the combine buffer: 128 O + m + l + pad

struct TileInfo {
  int64_t key_start;
  int nkeys;
  int pad;
};

__device__ __forceinline__ void consumer_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Walks a CTA's tiles in order and yields each tile's key range.  For a
// caller's index table (check_idx) an entry is used only if it is a block id
// in [0, nb) larger than every earlier in-range entry of the row, so no key is
// ever attended twice; other non-negative entries set kStatusIndex and are
// skipped, -1 entries are empty.
struct TileWalker {
  int64_t pair = -1;
  int slot = -1;
  int32_t run_max = -1;   // largest in-range id of the row's earlier slots
  int32_t j = -1;         // id of the current slot, -1 if skipped

  __device__ __forceinline__ void range(const DecodeAttnArgs& a, int64_t pr, int u, int64_t* ks, int* nk) {
    int64_t s = 0, e = 0;
    if (u < a.n_sink_tiles) {
      s = static_cast<int64_t>(u) * kTileKeys;
      e = min(s + kTileKeys, a.s_end);
    } else if ((u -= a.n_sink_tiles) < a.idx_stride * a.tpb) {
      const int sl = u / a.tpb, sub = u - sl * a.tpb;
      const int32_t* row = a.idx + pr * a.idx_stride;
      if (pr != pair) { pair = pr; slot = -1; run_max = -1; }
      if (sl != slot) {
        for (int q = slot + 1; q < sl; ++q) {        // slots this CTA did not walk
          const int32_t pj = __ldg(row + q);
          if (pj >= 0 && pj < a.nb && pj > run_max) run_max = pj;
        }
        int32_t jj = __ldg(row + sl);
        if (a.check_idx && jj >= 0) {
          const bool in_range = jj < a.nb;
          const bool ok = in_range && jj > run_max;
          if (in_range && jj > run_max) run_max = jj;
          if (!ok) {
            if (sub == 0) report(a.status, kStatusIndex);
            jj = -1;
          }
        } else if (a.check_idx && jj < -1) {
          if (sub == 0) report(a.status, kStatusIndex);
          jj = -1;
        }
        j = jj;
        slot = sl;
      }
      if (j >= 0) {
        const int64_t lo = max(static_cast<int64_t>(j) * a.b, a.s_end);
        const int64_t hi = min(static_cast<int64_t>(j + 1) * a.b, a.w_begin);
        s = lo + static_cast<int64_t>(sub) * kTileKeys;
        e = min(s + kTileKeys, hi);
      }
    } else {
      u -= a.idx_stride * a.tpb;
      s = a.w_begin + static_cast<int64_t>(u) * kTileKeys;
      e = min(s + kTileKeys, a.kv_end);
    }
    *ks = s;
    *nk = e > s ? static_cast<int>(e - s) : 0;
  }
};

template <bool BF16, bool OUT_BF16, int RG, int KG>
__global__ void __launch_bounds__((RG * KG + 1) * 32, 1) decode_attn_kernel(DecodeAttnArgs a) {
  constexpr int NWC = RG * KG;            // consumer warps
  constexpr int NCT = NWC * 32;           // consumer threads
  constexpr int KPW = kTileKeys / KG;     // keys per warp per tile
  constexpr int NIT = KPW / 8;            // QK iterations (8 keys per warp-iteration)
  constexpr int ROWB = BF16 ? 256 : 512;  // bytes per K/V row
  constexpr int STAGE = 2 * kTileKeys * ROWB;
  static_assert(KPW % 8 == 0, "KG must divide 8");

  extern __shared__ __align__(1024) unsigned char smem[];
  const int NS = a.n_stages;
  unsigned char* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NS) * STAGE);
  uint64_t* empty = full + NS;
  TileInfo* info = reinterpret_cast<TileInfo*>(empty + NS);
  float* pbuf = reinterpret_cast<float*>(info + NS);                 // [NWC][KPW][4]
  float* rowbuf = pbuf + NWC * KPW * 4;                              // [NWC][3][4]
  float* comb = rowbuf + NWC * 12;                                   // [KG][RG*4][kCombStride]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(comb + KG * RG * 4 * kCombStride);
  int* ticket = const_cast<int*>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * a.tpc;
  const int64_t t1 = min(a.total_tiles, t0 + a.tpc);
  const int ntiles = static_cast<int>(t1 - t0);

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
    if (lane == 0) {
      int issued = 0;
      TileWalker walker;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % NS;
        if (i >= NS) {
          if (!mbar_wait_bounded(&empty[s], ((i / NS) & 1) ^ 1, abort_flag)) {
            report(a.status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
        }
        if (*abort_flag) break;
        const int64_t t = t0 + i;
        const int64_t pair = t / a.MT;
        int64_t ks;
        int nk;
        walker.range(a, pair, static_cast<int>(t - pair * a.MT), &ks, &nk);
        info[s].key_start = ks;
        info[s].nkeys = nk;
        if (nk > 0) {
          const uint32_t bytes = static_cast<uint32_t>(nk) * ROWB;
          mbar_arrive_expect_tx(&full[s], 2 * bytes);
          const int64_t row = pair * a.cap + ks;
          const unsigned char* kp = static_cast<const unsigned char*>(a.K) + row * ROWB;
          const unsigned char* vp = static_cast<const unsigned char*>(a.V) + row * ROWB;
          bulk_g2s(stages + static_cast<size_t>(s) * STAGE, kp, bytes, &full[s]);
          bulk_g2s(stages + static_cast<size_t>(s) * STAGE + kTileKeys * ROWB, vp, bytes, &full[s]);
        } else {
          mbar_arrive(&full[s]);
        }
        issued = i + 1;
      }
      // do not leave while copies into this CTA's shared memory may be in flight
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait_bounded(&full[i % NS], (i / NS) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  const int rg = warp / KG, kg = warp - (warp / KG) * KG;
  const int gi = lane >> 3, l8 = lane & 7;
  float* my_p = pbuf + warp * KPW * 4;
  float* my_row = rowbuf + warp * 12;

  float q[4][16];
  float o[4][4];
  float m_run[4], l_run[4];
  int64_t cur_pair = -1;

  auto load_q = [&](int64_t pair) {
    const int bi = static_cast<int>(pair / a.Hkv), h = static_cast<int>(pair % a.Hkv);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int rr = rg * 4 + r;
      if (rr < a.R) {
        const int j = rr / a.G, g = rr - (rr / a.G) * a.G;
        const int64_t off = ((static_cast<int64_t>(bi) * a.n_q + j) * a.Hq + h * a.G + g) * kHeadDim;
        if constexpr (BF16) {
          const uint16_t* qp = static_cast<const uint16_t*>(a.Q) + off;
          uint4 u0 = __ldg(reinterpret_cast<const uint4*>(qp + 8 * l8));
          uint4 u1 = __ldg(reinterpret_cast<const uint4*>(qp + 64 + 8 * l8));
          unpack8(u0, &q[r][0]);
          unpack8(u1, &q[r][8]);
        } else {
          const float* qp = static_cast<const float*>(a.Q) + off;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float4 x = __ldg(reinterpret_cast<const float4*>(qp + 32 * c + 4 * l8));
            q[r][4 * c + 0] = x.x; q[r][4 * c + 1] = x.y; q[r][4 * c + 2] = x.z; q[r][4 * c + 3] = x.w;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) q[r][e] *= a.qscale;
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) q[r][e] = 0.f;
      }
      m_run[r] = -CUDART_INF_F;
      l_run[r] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) o[r][c] = 0.f;
    }
  };

  // Merge the KG warps of every row group and emit this CTA's result for `pair`.
  auto flush = [&](int64_t pair) {
    float* cb = comb + (kg * RG * 4) * kCombStride;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int rr = rg * 4 + r;
      *reinterpret_cast<float4*>(cb + rr * kCombStride + 4 * lane) =
          make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
      if (lane == 0) {
        cb[rr * kCombStride + 128] = m_run[r];
        cb[rr * kCombStride + 129] = l_run[r];
      }
    }
    consumer_bar(NCT);
    const int64_t first = pair * a.MT, last = first + a.MT - 1;
    const bool whole = first >= t0 && last < t1;
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
        const float inv = L > 0.f ? 1.f / L : 0.f;
        if constexpr (OUT_BF16) {
          uint2 pk = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.O) + orow * kHeadDim + 4 * c4) = pk;
        } else {
          *reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow * kHeadDim + 4 * c4) =
              make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
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
      __threadfence();
      consumer_bar(NCT);
      if (threadIdx.x == 0) {
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
          const float inv = L > 0.f ? 1.f / L : 0.f;
          if constexpr (OUT_BF16) {
            uint2 pk = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.O) + orow * kHeadDim + 4 * c4) = pk;
          } else {
            *reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow * kHeadDim + 4 * c4) =
                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
          }
          if (c4 == 0 && a.lse)
            a.lse[orow] = L > 0.f ? (Mr + log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
        }
        if (threadIdx.x == 0) a.counters[pair] = 0u;
      }
    }
    consumer_bar(NCT);   // the combine buffer is reused by the next segment
  };

  bool aborted = false;
  for (int i = 0; i < ntiles; ++i) {
    const int64_t t = t0 + i;
    const int64_t pair = t / a.MT;
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
    const int nkeys = aborted ? 0 : info[s].nkeys;
    const int64_t kstart = info[s].key_start;
    const int kb = kg * KPW;                 // this warp's first key in the tile
    const int nk = min(KPW, nkeys - kb);     // keys of this warp (<= 0: none)
    if (nk > 0) {
      const unsigned char* kst = stages + static_cast<size_t>(s) * STAGE;
      const unsigned char* vst = kst + kTileKeys * ROWB;
      float sc[NIT];
      const int r_loc = l8 & 3;
      const int rr_loc = rg * 4 + r_loc;
      const int tok = rr_loc / a.G;          // new-token index of this lane's row
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const int kk0 = kb + it * 8 + 2 * gi;
        float v[8];
#pragma unroll
        for (int kq = 0; kq < 2; ++kq) {
          const unsigned char* krow = kst + (kk0 + kq) * ROWB;
          float kf[16];
          if constexpr (BF16) {
            const uint4 u0 = *reinterpret_cast<const uint4*>(krow + l8 * 16);
            const uint4 u1 = *reinterpret_cast<const uint4*>(krow + 128 + l8 * 16);
            unpack8(u0, kf);
            unpack8(u1, kf + 8);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 x = *reinterpret_cast<const float4*>(krow + 128 * c + l8 * 16);
              kf[4 * c + 0] = x.x; kf[4 * c + 1] = x.y; kf[4 * c + 2] = x.z; kf[4 * c + 3] = x.w;
            }
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) acc = fmaf(q[r][e], kf[e], acc);
            v[kq * 4 + r] = acc;
          }
        }
        // reduce-scatter over the 8 lanes of the group: lane l8 ends with value l8
        const bool b2 = l8 & 4, b1 = l8 & 2, b0 = l8 & 1;
        float w4[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float send = b2 ? v[x] : v[4 + x];
          const float keep = b2 ? v[4 + x] : v[x];
          w4[x] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
        float w2[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const float send = b1 ? w4[x] : w4[2 + x];
          const float keep = b1 ? w4[2 + x] : w4[x];
          w2[x] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
        float w1;
        {
          const float send = b0 ? w2[0] : w2[1];
          const float keep = b0 ? w2[1] : w2[0];
          w1 = keep + __shfl_xor_sync(0xffffffffu, send, 1);
        }
        // this lane: key kk0 + (l8 >> 2), row r_loc
        const int kl = kk0 + (l8 >> 2);
        const int64_t pos = kstart + kl;
        bool valid = kl < nkeys;
        if (pos >= a.C) valid = valid && (pos - a.C) <= tok;
        sc[it] = valid ? w1 : -CUDART_INF_F;
      }
      float mx = sc[0];
#pragma unroll
      for (int it = 1; it < NIT; ++it) mx = fmaxf(mx, sc[it]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      float m_old = m_run[0];
#pragma unroll
      for (int r = 1; r < 4; ++r) m_old = (r_loc == r) ? m_run[r] : m_old;
      const float m_new = fmaxf(m_old, mx);
      const float m_ref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
      float rs = 0.f;
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const float p = exp2f(sc[it] - m_ref);
        rs += p;
        my_p[(it * 8 + 2 * gi + (l8 >> 2)) * 4 + r_loc] = p;
      }
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      rs += __shfl_xor_sync(0xffffffffu, rs, 8);
      rs += __shfl_xor_sync(0xffffffffu, rs, 16);
      if (lane < 4) {
        my_row[0 + lane] = exp2f(m_old - m_ref);   // alpha
        my_row[4 + lane] = rs;
        my_row[8 + lane] = m_new;
      }
      __syncwarp();
      const float4 al = *reinterpret_cast<const float4*>(my_row);
      const float4 rsv = *reinterpret_cast<const float4*>(my_row + 4);
      const float4 mn = *reinterpret_cast<const float4*>(my_row + 8);
      const float alr[4] = {al.x, al.y, al.z, al.w};
      const float rsr[4] = {rsv.x, rsv.y, rsv.z, rsv.w};
      const float mnr[4] = {mn.x, mn.y, mn.z, mn.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        l_run[r] = l_run[r] * alr[r] + rsr[r];
        m_run[r] = mnr[r];
#pragma unroll
        for (int c = 0; c < 4; ++c) o[r][c] *= alr[r];
      }
      for (int kk = 0; kk < nk; ++kk) {
        const float4 p4 = *reinterpret_cast<const float4*>(my_p + kk * 4);
        const unsigned char* vrow = vst + (kb + kk) * ROWB;
        float vv[4];
        if constexpr (BF16) {
          const uint2 u = *reinterpret_cast<const uint2*>(vrow + lane * 8);
          vv[0] = bf16lo(u.x); vv[1] = bf16hi(u.x); vv[2] = bf16lo(u.y); vv[3] = bf16hi(u.y);
        } else {
          const float4 x = *reinterpret_cast<const float4*>(vrow + lane * 16);
          vv[0] = x.x; vv[1] = x.y; vv[2] = x.z; vv[3] = x.w;
        }
        const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
          for (int c = 0; c < 4; ++c) o[r][c] = fmaf(pr[r], vv[c], o[r][c]);
        }
      }
      __syncwarp();
    }
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (cur_pair >= 0) flush(cur_pair);
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
  switch (p.RG) {
    case 1: return launch_one<BF16, OUT_BF16, 1, 8>(a, p, s);
    case 2: return launch_one<BF16, OUT_BF16, 2, 4>(a, p, s);
    case 3: return launch_one<BF16, OUT_BF16, 3, 4>(a, p, s);
    case 4: return launch_one<BF16, OUT_BF16, 4, 2>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_smem_bytes(int RG, int KG, bool bf16, int n_stages) {
  const int NWC = RG * KG;
  const int KPW = kTileKeys / KG;
  const size_t stage = 2 * kTileKeys * (bf16 ? 256 : 512);
  size_t b = stage * n_stages;
  b += 2 * sizeof(uint64_t) * n_stages;
  b += sizeof(TileInfo) * n_stages;
  b += sizeof(float) * NWC * KPW * 4;
  b += sizeof(float) * NWC * 12;
  b += sizeof(float) * KG * RG * 4 * kCombStride;
  b += 16;
  return b;
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
  p->KG = p->RG == 1 ? 8 : (p->RG == 4 ? 2 : 4);
  p->threads = (p->RG * p->KG + 1) * 32;
  p->n_sink_tiles = static_cast<int>((g.s_end + kTileKeys - 1) / kTileKeys);
  p->tpb = (g.b + kTileKeys - 1) / kTileKeys;
  p->n_wc_tiles = static_cast<int>((g.kv_end - g.w_begin + kTileKeys - 1) / kTileKeys);
  const int64_t mt = static_cast<int64_t>(p->n_sink_tiles) + static_cast<int64_t>(idx_slots) * p->tpb +
                     p->n_wc_tiles;
  if (mt > (1 << 24)) {
    *why = "too many key tiles per (sequence, KV head)";
    return false;
  }
  p->MT = static_cast<int>(mt);
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
  const size_t limit = 227 * 1024;
  int ns = bf16 ? 6 : 3;
  while (ns > 2 && decode_smem_bytes(p->RG, p->KG, bf16, ns) > limit) --ns;
  p->n_stages = ns;
  p->smem = decode_smem_bytes(p->RG, p->KG, bf16, ns);
  if (p->smem > limit) {
    *why = "shared memory plan exceeds 227 KB";
    return false;
  }
  return true;
}

cudaError_t launch_decode_attn(const DecodeAttnArgs& a, const DecodePlan& p, bool bf16, bool out_bf16,
                               cudaStream_t s) {
  if (p.total_tiles == 0) return cudaSuccess;
  if (bf16) return out_bf16 ? launch_rg<true, true>(a, p, s) : launch_rg<true, false>(a, p, s);
  return out_bf16 ? launch_rg<false, true>(a, p, s) : launch_rg<false, false>(a, p, s);
}

}  // namespace sa
