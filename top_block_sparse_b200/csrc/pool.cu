// Cache maintenance: compression of complete key blocks (step 1 of the
// method) and the append of new tokens' keys and values.
//
//   mean : Kc[j] = (1/b) * sum of the b keys of block j
//          (SparDA summary, section "方法": keys average-pooled into
//          compressed keys)
//   overlapping windows: Kc[c] = (1/l) * sum of the l keys from c*s, for
//          every complete window (same section: InfLLM-V2 pools into
//          overlapping compressed representations); the same kernel with
//          row start c*s and row length l
//   LSA  : Kc[j] = normalise(sum_t K_t / |K_t|) over the block's keys, which
//          equals the normalised sum of its pool keys (each pool key being the
//          sum of 4 consecutive unit keys) (LSA review §2.2)
//
// One warp per row, one pass over K with 128-bit coalesced loads: for bf16
// a row of 128 elements is 256 B = 16 lanes x 16 B, so one warp load covers
// two rows; for fp32 a row is 512 B = 32 lanes x 16 B.  Sums are kept in
// fp32 registers; the output is fp32 (set parity of the later top-k needs
// compressed keys far more precise than bf16).
#include "common.cuh"
#include "cache_ops.h"
#include "internal.h"

namespace sa {
namespace {

constexpr int kPoolWarps = 8;

template <bool BF16, bool LSA>
__global__ void __launch_bounds__(kPoolWarps * 32) pool_kernel(PoolArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kPoolWarps + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(a.pairs) * a.nb;
  if (w >= total) return;
  const int64_t pair = w / a.nb;
  const int64_t j = w - pair * a.nb;
  const int len = a.len;
  float* out = a.Kc + (pair * a.nb + j) * kHeadDim;

  if constexpr (BF16) {
    // lane -> row parity (lane >> 4), 16-byte chunk (lane & 15) = elements 8c..8c+7
    const uint16_t* base = static_cast<const uint16_t*>(a.K) + (pair * a.cap + j * a.stride) * kHeadDim;
    const int half = lane >> 4, c = lane & 15;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const int rows2 = len >> 1;                    // row pairs
    int i = 0;
    for (; i + 4 <= rows2; i += 4) {
      uint4 u[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        u[k] = __ldg(reinterpret_cast<const uint4*>(base + (2 * (i + k) + half) * kHeadDim) + c);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float f[8];
        unpack8(u[k], f);
        if constexpr (LSA) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += f[e] * inv;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += f[e];
        }
      }
    }
    if constexpr (!LSA) {
      // an odd row count leaves one row for the lower half-warp
      if ((len & 1) && half == 0) {
        float f[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(base + (len - 1) * kHeadDim) + c), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
    for (; i < rows2; ++i) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(base + (2 * i + half) * kHeadDim) + c);
      float f[8];
      unpack8(u, f);
      if constexpr (LSA) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e] * inv;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    float mul;
    if constexpr (LSA) {
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += acc[e] * acc[e];
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      mul = ss > 0.f ? rsqrtf(ss) : 0.f;
    } else {
      mul = 1.f / static_cast<float>(len);
    }
    if (half == 0) {
      float4* o4 = reinterpret_cast<float4*>(out + 8 * c);
      o4[0] = make_float4(acc[0] * mul, acc[1] * mul, acc[2] * mul, acc[3] * mul);
      o4[1] = make_float4(acc[4] * mul, acc[5] * mul, acc[6] * mul, acc[7] * mul);
    }
  } else {
    // fp32: lane -> 16-byte chunk = elements 4*lane..4*lane+3 of every row
    const float* base = static_cast<const float*>(a.K) + (pair * a.cap + j * a.stride) * kHeadDim;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int i = 0;
    for (; i + 4 <= len; i += 4) {
      float4 u[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        u[k] = __ldg(reinterpret_cast<const float4*>(base + (i + k) * kHeadDim) + lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float inv = 1.f;
        if constexpr (LSA) {
          float ss = u[k].x * u[k].x + u[k].y * u[k].y + u[k].z * u[k].z + u[k].w * u[k].w;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          inv = ss > 0.f ? rsqrtf(ss) : 0.f;
        }
        acc[0] += u[k].x * inv; acc[1] += u[k].y * inv;
        acc[2] += u[k].z * inv; acc[3] += u[k].w * inv;
      }
    }
    for (; i < len; ++i) {
      float4 u = __ldg(reinterpret_cast<const float4*>(base + i * kHeadDim) + lane);
      float inv = 1.f;
      if constexpr (LSA) {
        float ss = u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        inv = ss > 0.f ? rsqrtf(ss) : 0.f;
      }
      acc[0] += u.x * inv; acc[1] += u.y * inv; acc[2] += u.z * inv; acc[3] += u.w * inv;
    }
    float mul;
    if constexpr (LSA) {
      float ss = acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      mul = ss > 0.f ? rsqrtf(ss) : 0.f;
    } else {
      mul = 1.f / static_cast<float>(len);
    }
    reinterpret_cast<float4*>(out)[lane] =
        make_float4(acc[0] * mul, acc[1] * mul, acc[2] * mul, acc[3] * mul);
  }
}

// Append of the new tokens' rows to the cache: row t of pair q in K_new goes
// to row C + t of pair q in K (the same for V).  One thread per 16 bytes,
// K's rows first, then V's.
__global__ void __launch_bounds__(256) append_kv_kernel(const uint4* __restrict__ kn, const uint4* __restrict__ vn,
                                                        uint4* __restrict__ K, uint4* __restrict__ V, int64_t rows,
                                                        int n_q, int64_t cap, int64_t C, int chunks) {
  const int64_t per = rows * chunks;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= 2 * per) return;
  const bool is_v = i >= per;
  const int64_t j = is_v ? i - per : i;
  const int64_t row = j / chunks, c = j - row * chunks;
  const int64_t pair = row / n_q, t = row - pair * n_q;
  const uint4 v = is_v ? __ldg(vn + j) : __ldg(kn + j);
  (is_v ? V : K)[(pair * cap + C + t) * chunks + c] = v;
}

}  // namespace

cudaError_t launch_append_kv(const void* K_new, const void* V_new, void* K, void* V, int pairs, int n_q, int64_t cap,
                             int64_t C, int row_bytes, cudaStream_t s) {
  const int chunks = row_bytes / 16;
  const int64_t total = 2 * static_cast<int64_t>(pairs) * n_q * chunks;
  if (total == 0) return cudaSuccess;
  const int64_t grid = (total + 255) / 256;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  append_kv_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(
      static_cast<const uint4*>(K_new), static_cast<const uint4*>(V_new), static_cast<uint4*>(K),
      static_cast<uint4*>(V), static_cast<int64_t>(pairs) * n_q, n_q, cap, C, chunks);
  return cudaGetLastError();
}

cudaError_t launch_pool(const PoolArgs& a, bool bf16, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(a.pairs) * a.nb;
  if (total == 0) return cudaSuccess;
  const int64_t grid = (total + kPoolWarps - 1) / kPoolWarps;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  dim3 g(static_cast<unsigned>(grid)), blk(kPoolWarps * 32);
  if (bf16) {
    if (a.lsa) pool_kernel<true, true><<<g, blk, 0, s>>>(a);
    else pool_kernel<true, false><<<g, blk, 0, s>>>(a);
  } else {
    if (a.lsa) pool_kernel<false, true><<<g, blk, 0, s>>>(a);
    else pool_kernel<false, false><<<g, blk, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
