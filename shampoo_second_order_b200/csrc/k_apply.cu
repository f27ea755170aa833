// The preconditioned step (transcript segment 10, third piece), CUDA-core
// part, and the grafted update:
//   per segment   P = S^{-2/p} g                           (a matvec)
//   per parameter s = ||D||_F / ||P||_F, D = g / sqrt(a + eps)  (layer-wise)
//                 m <- mu m + s P,  W <- W - lr m
// The 2-D blocks' P = L^{-1/p} G R^{-1/p} runs on the tensor cores (k_tc.cu)
// and lands in the same parameter-shaped buffer with its sums of squares; the
// update pass then reads both.
#include "common.cuh"

namespace shampoo {

namespace {

__device__ __forceinline__ bool vec_ok(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// sum of D^2 per parameter, D = g / sqrt(a + eps); used when apply receives
// other gradients than the update_stats call that accumulated ||D||^2.
__global__ void __launch_bounds__(256) dnorm_kernel(const ChunkDesc* __restrict__ chunks,
                                                    const ParamDesc* __restrict__ params,
                                                    const void* const* __restrict__ gptr, int bf16,
                                                    const int* __restrict__ flags,
                                                    const float* __restrict__ a, float eps,
                                                    double* __restrict__ d2) {
  __shared__ double red[8];
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  const void* g = gptr[c.param];
  const float* ap = a + params[c.param].offset + c.start;
  double s = 0.0;
  for (int i = threadIdx.x; i < c.len; i += blockDim.x) {
    const float d = grad_at(g, c.start + i, bf16) / sqrtf(ap[i] + eps);
    s += (double)d * d;
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0 && s != 0.0) atomicAdd(&d2[c.param], s);
}

// P[s0 + i] = sum_j Sr[i][j] g[s0 + j]; one warp per row.  grid: x = 8-row
// group, y = segment.
__global__ void __launch_bounds__(256) precond_seg_kernel(
    const SegDesc* __restrict__ segs, int mat0, const ParamDesc* __restrict__ params,
    const void* const* __restrict__ gptr, int bf16, const int* __restrict__ flags,
    const float* __restrict__ roots, int S, float* __restrict__ P, double* __restrict__ p2) {
  __shared__ double red[8];
  const SegDesc sd = segs[blockIdx.y];
  if (flags[sd.param]) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * 8 + warp;
  const void* g = gptr[sd.param];
  double ss = 0.0;
  if (i < sd.len) {
    const float4* row = reinterpret_cast<const float4*>(roots + (size_t)(mat0 + blockIdx.y) * S * S +
                                                        (size_t)i * S);
    float acc = 0.0f;
    const int n4 = (sd.len + 3) >> 2;
    for (int v = lane; v < n4; v += 32) {
      const float4 r = row[v];
      const float rv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = 4 * v + q;
        if (j < sd.len) acc = fmaf(rv[q], grad_at(g, sd.s0 + j, bf16), acc);
      }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      P[params[sd.param].offset + sd.s0 + i] = acc;
      ss = (double)acc * acc;
    }
  }
  ss = block_sum(ss, red);
  if (threadIdx.x == 0 && ss != 0.0) atomicAdd(&p2[sd.param], ss);
}

// W <- W - lr (mu m + s P); graft scale s per parameter from the two norms.
__global__ void __launch_bounds__(256) update_kernel(
    const ChunkDesc* __restrict__ chunks, const ParamDesc* __restrict__ params,
    float* const* __restrict__ wptr, const int* __restrict__ flags, const float* __restrict__ P,
    const double* __restrict__ d2, const double* __restrict__ p2, int graft, float mu, float lr,
    float* __restrict__ mom) {
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  float s = 1.0f;
  if (graft) {
    const double dn = d2[c.param], pn = p2[c.param];
    s = pn > 0.0 ? (float)(sqrt(dn) / sqrt(pn)) : 0.0f;
  }
  const int64_t off = params[c.param].offset + c.start;
  float* w = wptr[c.param] + c.start;
  const float* pp = P + off;
  float* mm = mom ? mom + off : nullptr;
  int done = 0;
  if (vec_ok(w)) {
    const int n4 = c.len >> 2;
    float4* w4 = reinterpret_cast<float4*>(w);
    const float4* p4 = reinterpret_cast<const float4*>(pp);
    float4* m4 = reinterpret_cast<float4*>(mm);
#pragma unroll 4
    for (int v = threadIdx.x; v < n4; v += blockDim.x) {
      const float4 p = p4[v];
      float4 x = w4[v];
      if (mm) {
        float4 m = m4[v];
        m.x = fmaf(mu, m.x, s * p.x);
        m.y = fmaf(mu, m.y, s * p.y);
        m.z = fmaf(mu, m.z, s * p.z);
        m.w = fmaf(mu, m.w, s * p.w);
        m4[v] = m;
        x.x = fmaf(-lr, m.x, x.x);
        x.y = fmaf(-lr, m.y, x.y);
        x.z = fmaf(-lr, m.z, x.z);
        x.w = fmaf(-lr, m.w, x.w);
      } else {
        x.x = fmaf(-lr, s * p.x, x.x);
        x.y = fmaf(-lr, s * p.y, x.y);
        x.z = fmaf(-lr, s * p.z, x.z);
        x.w = fmaf(-lr, s * p.w, x.w);
      }
      w4[v] = x;
    }
    done = 4 * n4;
  }
  for (int i = done + threadIdx.x; i < c.len; i += blockDim.x) {
    if (mm) {
      const float m = fmaf(mu, mm[i], s * pp[i]);
      mm[i] = m;
      w[i] = fmaf(-lr, m, w[i]);
    } else {
      w[i] = fmaf(-lr, s * pp[i], w[i]);
    }
  }
}

}  // namespace

void launch_dnorm(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                  const void* const* gptr, int bf16, const int* flags, const float* a, float eps,
                  double* d2, cudaStream_t s) {
  if (nchunks > 0) dnorm_kernel<<<nchunks, 256, 0, s>>>(chunks, params, gptr, bf16, flags, a, eps, d2);
}

void launch_precondition_segments(const SegDesc* segs, int nseg, int mat0, const ParamDesc* params,
                                  const void* const* gptr, int bf16, const int* flags,
                                  const float* roots, int S, float* P, double* p2,
                                  cudaStream_t s) {
  if (nseg <= 0) return;
  precond_seg_kernel<<<dim3((S + 7) / 8, nseg), 256, 0, s>>>(segs, mat0, params, gptr, bf16, flags,
                                                            roots, S, P, p2);
}

void launch_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params, float* const* wptr,
                   const int* flags, const float* P, const double* d2, const double* p2, int graft,
                   float mu, float lr, float* mom, cudaStream_t s) {
  if (nchunks > 0)
    update_kernel<<<nchunks, 256, 0, s>>>(chunks, params, wptr, flags, P, d2, p2, graft, mu, lr, mom);
}

}  // namespace shampoo
