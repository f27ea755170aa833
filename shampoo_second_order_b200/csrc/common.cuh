// Device helpers shared by the kernels of the library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace shampoo {

// Gradient element as float: bf16 is widened exactly (upper half of an fp32).
__device__ __forceinline__ float grad_at(const void* p, int64_t i, int bf16) {
  if (bf16) {
    unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    return __uint_as_float(static_cast<unsigned>(u) << 16);
  }
  return __ldg(reinterpret_cast<const float*>(p) + i);
}

// Scaling s_k of Newton step k of matrix m (1 past the scaled steps).
__device__ __forceinline__ double newton_sched(const NewtonWork& w, int m, int k) {
  return k < w.nsched[m] ? w.sched[(size_t)m * kSched + k] : 1.0;
}

// Warp sum / max.
__device__ __forceinline__ double warp_sum(double v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum of one double per thread; result valid in thread 0.
// `red` must hold blockDim.x / 32 doubles.
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    s = (l < nw) ? red[l] : 0.0;
    s = warp_sum(s);
  }
  __syncthreads();
  return s;
}

__device__ __forceinline__ double block_max(double v, double* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    s = (l < nw) ? red[l] : 0.0;
    s = warp_max(s);
  }
  __syncthreads();
  return s;
}

}  // namespace shampoo
