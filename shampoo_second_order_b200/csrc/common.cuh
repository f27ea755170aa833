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

// A strided read-only view of a matrix: element (i, k) is p[i*si + k*sk]
// when i < mi and k < mk, and 0 outside (the zero padding of ragged blocks).
struct View {
  const void* p;
  int64_t si, sk;
  int mi, mk;
  int bf16;
};

__device__ __forceinline__ float view_at(const View& v, int i, int k) {
  if (i < v.mi && k < v.mk) return grad_at(v.p, i * v.si + k * v.sk, v.bf16);
  return 0.0f;
}

// One 64 x 64 fp32 output tile, C(i, j) = sum_k A(i, k) * Bt(j, k), on 256
// threads; thread (ty, tx) = (t / 16, t % 16) owns rows ty*4.., cols tx*4..
// The loads follow whichever stride of the view is 1, so each warp reads
// contiguous memory.  Exact fp32 FMA products and sums.
__device__ __forceinline__ void tile_gemm_f32(const View& A, const View& B, int i0, int j0,
                                              int K, float acc[4][4], float (*As)[68],
                                              float (*Bs)[68]) {
  const int t = threadIdx.x;
  const int ty = t >> 4, tx = t & 15;
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = t + r * 256;
      int i, k;
      if (A.sk == 1) { k = e & 15; i = e >> 4; } else { i = e & 63; k = e >> 6; }
      As[k][i] = view_at(A, i0 + i, k0 + k);
      if (B.sk == 1) { k = e & 15; i = e >> 4; } else { i = e & 63; k = e >> 6; }
      Bs[k][i] = view_at(B, j0 + i, k0 + k);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
}

}  // namespace shampoo
