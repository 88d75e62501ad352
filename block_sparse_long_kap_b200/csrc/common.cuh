// Shared device helpers for the CoSA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cosa.h"

namespace cosa {

// Per-device status word: the first in-kernel error since it was last read.
__device__ int g_status;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Causal pages of q-block qb: pages holding a key that a row of the block sees.
__host__ __device__ __forceinline__ int causal_pages(int qb, int q_block, int page_size) {
  return ((qb + 1) * q_block + page_size - 1) / page_size;
}

// Number of forced pages: the sink pages plus the pages overlapping the
// q-block's own token range (the "local" pages), without double counting.
__host__ __device__ __forceinline__ int forced_count(int qb, int q_block, int page_size, int sink) {
  int n_b = causal_pages(qb, q_block, page_size);
  int first_diag = (qb * q_block) / page_size;
  int s = sink < n_b ? sink : n_b;
  int overlap = s > first_diag ? s - first_diag : 0;
  return s + (n_b - first_diag) - overlap;
}

// k_b = min(n_b, max(|forced|, ceil(fl32(budget * n_b)))).  The product is the
// single-precision round-to-nearest product on host and device alike.
__host__ __device__ __forceinline__ int budget_count(int qb, int q_block, int page_size, int sink,
                                                     float budget) {
  int n_b = causal_pages(qb, q_block, page_size);
  int n_f = forced_count(qb, q_block, page_size, sink);
#ifdef __CUDA_ARCH__
  float prod = __fmul_rn(budget, (float)n_b);
#else
  volatile float vb = budget;
  float prod = vb * (float)n_b;
#endif
  int want = (int)ceilf(prod);
  int k = want > n_f ? want : n_f;
  return k < n_b ? k : n_b;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace cosa
