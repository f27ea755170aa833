// Statistics accumulation, the CUDA-core part (transcript segment 10, first
// piece): S <- beta2 S + g g^T per 1-D segment, the graft's diagonal
// accumulator a <- beta2 a + g*g together with ||D||^2, D = g / sqrt(a + eps),
// and the non-finite check of 1-D gradients (2-D gradients are checked by the
// gather, which reads them anyway).  The 2-D blocks' L and R run on the
// tensor cores (k_tc.cu).
#include "common.cuh"

namespace shampoo {

namespace {

// Four consecutive gradient elements as floats; `aligned` selects one
// vector load (8 or 16 bytes) over four scalar ones.
__device__ __forceinline__ float4 grad4(const void* g, int64_t i, int bf16, bool aligned) {
  if (bf16) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(g) + i;
    if (aligned) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                         __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    return make_float4(__uint_as_float((uint32_t)__ldg(p) << 16), __uint_as_float((uint32_t)__ldg(p + 1) << 16),
                       __uint_as_float((uint32_t)__ldg(p + 2) << 16), __uint_as_float((uint32_t)__ldg(p + 3) << 16));
  }
  const float* p = reinterpret_cast<const float*>(g) + i;
  if (aligned) return __ldg(reinterpret_cast<const float4*>(p));
  return make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
}

__device__ __forceinline__ bool aligned16(const void* g, int64_t i, int bf16) {
  return ((reinterpret_cast<uintptr_t>(g) + (uint64_t)i * (bf16 ? 2 : 4)) & (bf16 ? 7 : 15)) == 0;
}

// 1-D parameters only: flag a parameter whose gradient holds NaN or Inf.
__global__ void check_finite_kernel(const ChunkDesc* __restrict__ chunks,
                                    const void* const* __restrict__ gptr, int bf16,
                                    int* __restrict__ flags) {
  const ChunkDesc c = chunks[blockIdx.x];
  const void* g = gptr[c.param];
  int bad = 0;
  for (int i = threadIdx.x; i < c.len; i += blockDim.x) bad |= !isfinite(grad_at(g, c.start + i, bf16));
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&flags[c.param], 1);
}

// a <- beta2 a + g*g and sum of (g / sqrt(a + eps))^2 per parameter.
__global__ void __launch_bounds__(256) diag_update_kernel(
    const ChunkDesc* __restrict__ chunks, const ParamDesc* __restrict__ params,
    const void* const* __restrict__ gptr, int bf16, const int* __restrict__ flags, float beta2,
    float eps, float* __restrict__ a, double* __restrict__ d2) {
  __shared__ double red[8];
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  const void* g = gptr[c.param];
  float* ap = a + params[c.param].offset + c.start;
  const bool al = aligned16(g, c.start, bf16);
  double s = 0.0;
  const int n4 = c.len >> 2;
#pragma unroll 4
  for (int v = threadIdx.x; v < n4; v += blockDim.x) {
    const float4 x = grad4(g, c.start + 4 * (int64_t)v, bf16, al);
    float4 o = reinterpret_cast<float4*>(ap)[v];
    o.x = fmaf(beta2, o.x, x.x * x.x);
    o.y = fmaf(beta2, o.y, x.y * x.y);
    o.z = fmaf(beta2, o.z, x.z * x.z);
    o.w = fmaf(beta2, o.w, x.w * x.w);
    reinterpret_cast<float4*>(ap)[v] = o;
    const float d0 = x.x / sqrtf(o.x + eps), d1 = x.y / sqrtf(o.y + eps);
    const float e0 = x.z / sqrtf(o.z + eps), e1 = x.w / sqrtf(o.w + eps);
    s += (double)d0 * d0 + (double)d1 * d1 + (double)e0 * e0 + (double)e1 * e1;
  }
  for (int i = 4 * n4 + threadIdx.x; i < c.len; i += blockDim.x) {
    const float x = grad_at(g, c.start + i, bf16);
    const float o = fmaf(beta2, ap[i], x * x);
    ap[i] = o;
    const float d = x / sqrtf(o + eps);
    s += (double)d * d;
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0 && s != 0.0) atomicAdd(&d2[c.param], s);
}

// S(i, j) <- beta2 S(i, j) + g_i g_j on the valid len x len corner (columns
// rounded up to 4; the extra columns see g_j = 0).  One warp per row.
// grid: x = group of 8 rows, y = segment.
__global__ void __launch_bounds__(256) stats_segments_kernel(
    const SegDesc* __restrict__ segs, int mat0, const void* const* __restrict__ gptr, int bf16,
    const int* __restrict__ flags, float beta2, float* __restrict__ stats, int S) {
  const SegDesc sd = segs[blockIdx.y];
  if (flags[sd.param]) return;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= sd.len) return;
  const void* g = gptr[sd.param];
  const float gi = grad_at(g, sd.s0 + i, bf16);
  float4* row = reinterpret_cast<float4*>(stats + (size_t)(mat0 + blockIdx.y) * S * S + (size_t)i * S);
  const int n4 = (sd.len + 3) >> 2;
  for (int v = lane; v < n4; v += 32) {
    float gj[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = 4 * v + q;
      gj[q] = j < sd.len ? grad_at(g, sd.s0 + j, bf16) : 0.0f;
    }
    float4 o = row[v];
    o.x = fmaf(beta2, o.x, gi * gj[0]);
    o.y = fmaf(beta2, o.y, gi * gj[1]);
    o.z = fmaf(beta2, o.z, gi * gj[2]);
    o.w = fmaf(beta2, o.w, gi * gj[3]);
    row[v] = o;
  }
}

}  // namespace

void launch_check_finite(const ChunkDesc* chunks, int nchunks, const void* const* gptr, int bf16,
                         int* flags, cudaStream_t s) {
  if (nchunks > 0) check_finite_kernel<<<nchunks, 256, 0, s>>>(chunks, gptr, bf16, flags);
}

void launch_diag_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                        const void* const* gptr, int bf16, const int* flags, float beta2, float eps,
                        float* a, double* d2, cudaStream_t s) {
  if (nchunks > 0)
    diag_update_kernel<<<nchunks, 256, 0, s>>>(chunks, params, gptr, bf16, flags, beta2, eps, a, d2);
}

void launch_stats_segments(const SegDesc* segs, int nseg, int mat0, const void* const* gptr,
                           int bf16, const int* flags, float beta2, float* stats, int S,
                           cudaStream_t s) {
  if (nseg <= 0) return;
  dim3 grid((S + 7) / 8, nseg);
  stats_segments_kernel<<<grid, 256, 0, s>>>(segs, mat0, gptr, bf16, flags, beta2, stats, S);
}

}  // namespace shampoo
