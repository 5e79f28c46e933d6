// Host-side interface of the cache append kernel (pool.cu) for the C ABI
// layer.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// Rows [pairs * n_q] of row_bytes (a multiple of 16) from K_new / V_new to
// rows C.. of each pair's cap rows in K / V.
cudaError_t launch_append_kv(const void* K_new, const void* V_new, void* K, void* V, int pairs, int n_q, int64_t cap,
                             int64_t C, int row_bytes, cudaStream_t s);

}  // namespace sa
