// Statistics accumulation (transcript segment 10, first piece):
//   L <- beta2 L + G G^T,  R <- beta2 R + G^T G  per <= b x b block (segment 16),
//   S <- beta2 S + g g^T per 1-D segment,  a <- beta2 a + g*g (graft).
// The block partition is fused into the loads: a block is read in place from
// the caller's row-major gradient with out-of-range rows/cols read as zero,
// which is the zero padding of a ragged block.
#include "common.cuh"

namespace shampoo {

__global__ void check_finite_kernel(const ChunkDesc* __restrict__ chunks,
                                    const void* const* __restrict__ gptr, int bf16,
                                    int* __restrict__ flags) {
  const ChunkDesc c = chunks[blockIdx.x];
  const void* g = gptr[c.param];
  int bad = 0;
  for (int i = threadIdx.x; i < c.len; i += blockDim.x) {
    const float v = grad_at(g, c.start + i, bf16);
    bad |= !isfinite(v);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&flags[c.param], 1);
}

__global__ void diag_update_kernel(const ChunkDesc* __restrict__ chunks,
                                   const ParamDesc* __restrict__ params,
                                   const void* const* __restrict__ gptr, int bf16,
                                   const int* __restrict__ flags, float beta2,
                                   float* __restrict__ a) {
  const ChunkDesc c = chunks[blockIdx.x];
  if (flags[c.param]) return;
  const void* g = gptr[c.param];
  float* ap = a + params[c.param].offset + c.start;
  for (int i = threadIdx.x; i < c.len; i += blockDim.x) {
    const float v = grad_at(g, c.start + i, bf16);
    ap[i] = fmaf(beta2, ap[i], v * v);
  }
}

// grid: x = tile (ti, tj) of the S x S slot, y = block, z = 0 for L, 1 for R.
__global__ void __launch_bounds__(256) stats_blocks_kernel(
    const BlockDesc* __restrict__ blocks, const void* const* __restrict__ gptr, int bf16,
    const int* __restrict__ flags, float beta2, float* __restrict__ stats, int S) {
  __shared__ __align__(16) float As[16][68];
  __shared__ __align__(16) float Bs[16][68];
  const BlockDesc bd = blocks[blockIdx.y];
  if (flags[bd.param]) return;
  const int T = S / kTile;
  const int ti = blockIdx.x / T, tj = blockIdx.x % T;
  const int isR = blockIdx.z;
  const int side = isR ? bd.n : bd.m;
  if (ti * kTile >= side || tj * kTile >= side) return;  // all-padding tile stays 0
  const char* base = reinterpret_cast<const char*>(gptr[bd.param]);
  const int esz = bf16 ? 2 : 4;
  const void* g0 = base + (bd.r0 * bd.ld + bd.c0) * esz;
  View A;
  A.p = g0;
  A.bf16 = bf16;
  int K;
  if (!isR) {  // L(i, j) = sum_k G[i][k] G[j][k]
    A.si = bd.ld; A.sk = 1; A.mi = bd.m; A.mk = bd.n; K = bd.n;
  } else {     // R(i, j) = sum_k G[k][i] G[k][j]
    A.si = 1; A.sk = bd.ld; A.mi = bd.n; A.mk = bd.m; K = bd.m;
  }
  float acc[4][4] = {};
  tile_gemm_f32(A, A, ti * kTile, tj * kTile, K, acc, As, Bs);
  float* C = stats + (size_t)(2 * blockIdx.y + isR) * S * S;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = ti * kTile + ty * 4 + x;
    float4* row = reinterpret_cast<float4*>(C + (size_t)i * S + tj * kTile + tx * 4);
    float4 o = *row;
    o.x = fmaf(beta2, o.x, acc[x][0]);
    o.y = fmaf(beta2, o.y, acc[x][1]);
    o.z = fmaf(beta2, o.z, acc[x][2]);
    o.w = fmaf(beta2, o.w, acc[x][3]);
    *row = o;
  }
}

// S(i, j) <- beta2 S(i, j) + g_i g_j over the valid len x len corner.
// grid: x = tile, y = segment.
__global__ void __launch_bounds__(256) stats_segments_kernel(
    const SegDesc* __restrict__ segs, int mat0, const void* const* __restrict__ gptr, int bf16,
    const int* __restrict__ flags, float beta2, float* __restrict__ stats, int S) {
  const SegDesc sd = segs[blockIdx.y];
  if (flags[sd.param]) return;
  const int T = S / kTile;
  const int ti = blockIdx.x / T, tj = blockIdx.x % T;
  if (ti * kTile >= sd.len || tj * kTile >= sd.len) return;
  __shared__ float gi[kTile], gj[kTile];
  const void* g = gptr[sd.param];
  if (threadIdx.x < kTile) {
    const int i = ti * kTile + threadIdx.x;
    gi[threadIdx.x] = i < sd.len ? grad_at(g, sd.s0 + i, bf16) : 0.0f;
  } else if (threadIdx.x < 2 * kTile) {
    const int j = tj * kTile + threadIdx.x - kTile;
    gj[threadIdx.x - kTile] = j < sd.len ? grad_at(g, sd.s0 + j, bf16) : 0.0f;
  }
  __syncthreads();
  float* C = stats + (size_t)(mat0 + blockIdx.y) * S * S;
  for (int e = threadIdx.x; e < kTile * kTile; e += blockDim.x) {
    const int i = e / kTile, j = e % kTile;
    float* c = C + (size_t)(ti * kTile + i) * S + tj * kTile + j;
    *c = fmaf(beta2, *c, gi[i] * gj[j]);
  }
}

void launch_check_finite(const ChunkDesc* chunks, int nchunks, const void* const* gptr, int bf16,
                         int* flags, cudaStream_t s) {
  if (nchunks > 0) check_finite_kernel<<<nchunks, 256, 0, s>>>(chunks, gptr, bf16, flags);
}

void launch_diag_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                        const void* const* gptr, int bf16, const int* flags, float beta2, float* a,
                        cudaStream_t s) {
  if (nchunks > 0)
    diag_update_kernel<<<nchunks, 256, 0, s>>>(chunks, params, gptr, bf16, flags, beta2, a);
}

void launch_stats_blocks(const BlockDesc* blocks, int nblk, const void* const* gptr, int bf16,
                         const int* flags, float beta2, float* stats, int S, cudaStream_t s) {
  if (nblk <= 0) return;
  const int T = S / kTile;
  dim3 grid(T * T, nblk, 2);
  stats_blocks_kernel<<<grid, 256, 0, s>>>(blocks, gptr, bf16, flags, beta2, stats, S);
}

void launch_stats_segments(const SegDesc* segs, int nseg, int mat0, const void* const* gptr,
                           int bf16, const int* flags, float beta2, float* stats, int S,
                           cudaStream_t s) {
  if (nseg <= 0) return;
  const int T = S / kTile;
  dim3 grid(T * T, nseg);
  stats_segments_kernel<<<grid, 256, 0, s>>>(segs, mat0, gptr, bf16, flags, beta2, stats, S);
}

}  // namespace shampoo
