// The preconditioned step (transcript segment 10, third piece) and the
// grafted update:
//   per block     Y = G R^{-1/p},  P = L^{-1/p} Y          (two GEMMs)
//   per segment   P = S^{-2/p} g                           (a matvec)
//   per parameter s = ||D||_F / ||P||_F, D = g / sqrt(a + eps)  (layer-wise)
//                 m <- mu m + s P,  W <- W - lr m
// P goes to a parameter-shaped buffer (padding discarded) together with the
// per-parameter sums of squares; the update pass then reads both.
#include "common.cuh"

namespace shampoo {

namespace {

// sum of D^2 per parameter, D = g / sqrt(a + eps)
__global__ void dnorm_kernel(const ChunkDesc* __restrict__ chunks, const ParamDesc* __restrict__ params,
                             const void* const* __restrict__ gptr, int bf16,
                             const int* __restrict__ flags, const float* __restrict__ a, float eps,
                             double* __restrict__ norms) {
  __shared__ double red[8];
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  const void* g = gptr[c.param];
  const float* ap = a + params[c.param].offset + c.start;
  double s = 0.0;
  for (int i = threadIdx.x; i < c.len; i += blockDim.x) {
    const float v = grad_at(g, c.start + i, bf16);
    const float d = v / sqrtf(ap[i] + eps);
    s += (double)d * d;
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0) atomicAdd(&norms[2 * c.param], s);
}

// Y = G R^{-1/p} over the whole S x S slot.  grid: x = tile, y = block.
__global__ void __launch_bounds__(256) precond_y_kernel(
    const BlockDesc* __restrict__ blocks, const void* const* __restrict__ gptr, int bf16,
    const int* __restrict__ flags, const float* __restrict__ roots, int S, float* __restrict__ Y) {
  __shared__ __align__(16) float As[16][68];
  __shared__ __align__(16) float Bs[16][68];
  const BlockDesc bd = blocks[blockIdx.y];
  if (flags[bd.param]) return;
  const int T = S / kTile;
  const int ti = blockIdx.x / T, tj = blockIdx.x % T;
  float* Yb = Y + (size_t)blockIdx.y * S * S;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[4][4] = {};
  if (ti * kTile < bd.m && tj * kTile < bd.n) {
    const int esz = bf16 ? 2 : 4;
    View A;
    A.p = reinterpret_cast<const char*>(gptr[bd.param]) + (bd.r0 * bd.ld + bd.c0) * esz;
    A.si = bd.ld; A.sk = 1; A.mi = bd.m; A.mk = bd.n; A.bf16 = bf16;
    View B;   // Bt(j, k) = Rr[k][j]; Rr is symmetric
    B.p = roots + (size_t)(2 * blockIdx.y + 1) * S * S;
    B.si = 1; B.sk = S; B.mi = bd.n; B.mk = bd.n; B.bf16 = 0;
    tile_gemm_f32(A, B, ti * kTile, tj * kTile, bd.n, acc, As, Bs);
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = ti * kTile + ty * 4 + x;
    *reinterpret_cast<float4*>(Yb + (size_t)i * S + tj * kTile + tx * 4) =
        make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
  }
}

// P = L^{-1/p} Y, valid m x n corner scattered into the parameter layout,
// sum of P^2 per parameter.  grid: x = tile, y = block.
__global__ void __launch_bounds__(256) precond_p_kernel(
    const BlockDesc* __restrict__ blocks, const ParamDesc* __restrict__ params,
    const int* __restrict__ flags, const float* __restrict__ roots, int S,
    const float* __restrict__ Y, float* __restrict__ P, double* __restrict__ norms) {
  __shared__ __align__(16) float As[16][68];
  __shared__ __align__(16) float Bs[16][68];
  __shared__ double red[8];
  const BlockDesc bd = blocks[blockIdx.y];
  if (flags[bd.param]) return;
  const int T = S / kTile;
  const int ti = blockIdx.x / T, tj = blockIdx.x % T;
  if (ti * kTile >= bd.m || tj * kTile >= bd.n) return;
  View A;   // Lr[i][k]
  A.p = roots + (size_t)(2 * blockIdx.y) * S * S;
  A.si = S; A.sk = 1; A.mi = bd.m; A.mk = bd.m; A.bf16 = 0;
  View B;   // Bt(j, k) = Y[k][j]
  B.p = Y + (size_t)blockIdx.y * S * S;
  B.si = 1; B.sk = S; B.mi = bd.n; B.mk = bd.m; B.bf16 = 0;
  float acc[4][4] = {};
  tile_gemm_f32(A, B, ti * kTile, tj * kTile, bd.m, acc, As, Bs);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float* Pp = P + params[bd.param].offset;
  double ss = 0.0;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = ti * kTile + ty * 4 + x;
    if (i >= bd.m) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = tj * kTile + tx * 4 + y;
      if (j < bd.n) {
        const float v = acc[x][y];
        Pp[(bd.r0 + i) * bd.ld + bd.c0 + j] = v;
        ss += (double)v * v;
      }
    }
  }
  ss = block_sum(ss, red);
  if (threadIdx.x == 0) atomicAdd(&norms[2 * bd.param + 1], ss);
}

// P[s0 + i] = sum_j Sr[i][j] g[s0 + j]; one warp per row.  grid: x = 8-row
// group, y = segment.
__global__ void __launch_bounds__(256) precond_seg_kernel(
    const SegDesc* __restrict__ segs, int mat0, const ParamDesc* __restrict__ params,
    const void* const* __restrict__ gptr, int bf16, const int* __restrict__ flags,
    const float* __restrict__ roots, int S, float* __restrict__ P, double* __restrict__ norms) {
  __shared__ double red[8];
  const SegDesc sd = segs[blockIdx.y];
  if (flags[sd.param]) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * 8 + warp;
  const void* g = gptr[sd.param];
  const float* Sr = roots + (size_t)(mat0 + blockIdx.y) * S * S;
  double ss = 0.0;
  if (i < sd.len) {
    float acc = 0.0f;
    for (int j = lane; j < sd.len; j += 32) acc = fmaf(Sr[(size_t)i * S + j], grad_at(g, sd.s0 + j, bf16), acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      P[params[sd.param].offset + sd.s0 + i] = acc;
      ss = (double)acc * acc;
    }
  }
  ss = block_sum(ss, red);
  if (threadIdx.x == 0 && ss != 0.0) atomicAdd(&norms[2 * sd.param + 1], ss);
}

// W <- W - lr (mu m + s P); graft scale s per parameter from the two norms.
__global__ void update_kernel(const ChunkDesc* __restrict__ chunks, const ParamDesc* __restrict__ params,
                              float* const* __restrict__ wptr, const int* __restrict__ flags,
                              const float* __restrict__ P, const double* __restrict__ norms,
                              int graft, float mu, float lr, float* __restrict__ mom) {
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  float s = 1.0f;
  if (graft) {
    const double dn = norms[2 * c.param], pn = norms[2 * c.param + 1];
    s = pn > 0.0 ? (float)(sqrt(dn) / sqrt(pn)) : 0.0f;
  }
  const int64_t off = params[c.param].offset + c.start;
  float* w = wptr[c.param] + c.start;
  const float* pp = P + off;
  if (mom) {
    float* mm = mom + off;
    for (int i = threadIdx.x; i < c.len; i += blockDim.x) {
      const float m = fmaf(mu, mm[i], s * pp[i]);
      mm[i] = m;
      w[i] = fmaf(-lr, m, w[i]);
    }
  } else {
    for (int i = threadIdx.x; i < c.len; i += blockDim.x) w[i] = fmaf(-lr, s * pp[i], w[i]);
  }
}

}  // namespace

void launch_dnorm(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                  const void* const* gptr, int bf16, const int* flags, const float* a, float eps,
                  double* norms, cudaStream_t s) {
  if (nchunks > 0) dnorm_kernel<<<nchunks, 256, 0, s>>>(chunks, params, gptr, bf16, flags, a, eps, norms);
}

void launch_precond_y(const BlockDesc* blocks, int nblk, const void* const* gptr, int bf16,
                      const int* flags, const float* roots, int S, float* Y, cudaStream_t s) {
  if (nblk <= 0) return;
  const int T = S / kTile;
  precond_y_kernel<<<dim3(T * T, nblk), 256, 0, s>>>(blocks, gptr, bf16, flags, roots, S, Y);
}

void launch_precond_p(const BlockDesc* blocks, int nblk, const ParamDesc* params, const int* flags,
                      const float* roots, int S, const float* Y, float* P, double* norms,
                      cudaStream_t s) {
  if (nblk <= 0) return;
  const int T = S / kTile;
  precond_p_kernel<<<dim3(T * T, nblk), 256, 0, s>>>(blocks, params, flags, roots, S, Y, P, norms);
}

void launch_precondition_segments(const SegDesc* segs, int nseg, int mat0, const ParamDesc* params,
                                  const void* const* gptr, int bf16, const int* flags,
                                  const float* roots, int S, float* P, double* norms,
                                  cudaStream_t s) {
  if (nseg <= 0) return;
  precond_seg_kernel<<<dim3((S + 7) / 8, nseg), 256, 0, s>>>(segs, mat0, params, gptr, bf16, flags,
                                                            roots, S, P, norms);
}

void launch_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params, float* const* wptr,
                   const int* flags, const float* P, const double* norms, int graft, float mu,
                   float lr, float* mom, cudaStream_t s) {
  if (nchunks > 0)
    update_kernel<<<nchunks, 256, 0, s>>>(chunks, params, wptr, flags, P, norms, graft, mu, lr, mom);
}

}  // namespace shampoo
