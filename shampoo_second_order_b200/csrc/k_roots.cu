// Batched inverse p-th roots by the coupled Newton iteration in float64
// (transcript segment 12: the root must be taken in double precision; this
// is the coupled Newton iteration it names, Guo & Higham 2006), with a scalar
// scaling of the first steps:
//
//   c^p >= lambda_max(A + eps I),  X0 = c^{-1} I,  M0 = (A + eps I) / c^p
//   step k:  T = ((p+1) I - s_k M) / p,  X <- s_k^{1/p} X T,  M <- s_k T^p M
//   until max|M - I| <= tol.
//
// Scaling X by mu and M by mu^p keeps the coupling M = X^p (A + eps I), so
// every s_k > 0 leaves the limit unchanged.  Each eigenvalue m of M moves by
// the scalar map m -> s m ((p+1 - s m)/p)^p, which for s = 1 (plain Newton)
// only multiplies small eigenvalues by ((p+1)/p)^p per step.  A short Lanczos
// run on M0 estimates its extreme eigenvalues [l, u]; s_k is then chosen so
// that the ends of the current interval land on the same value (equal
// oscillation), which roughly halves the steps for spread spectra.  s_k is
// capped at 0.98 (p+1) so that the true top eigenvalue (<= 1 by the choice
// of c) stays inside the map's convergence region whatever the estimate;
// a poor estimate costs steps, never the limit.  Once the tracked interval
// sits above 0.7 the plain iteration finishes quadratically: near 1 the map
// sends 1 - m to (p+1)/(2p) (1 - m)^2 + O((1 - m)^3), so when ||M - I||_F = f
// bounds every |1 - m| and 0.75 f^2 (1 + f) <= tol / 2, the next step's
// residual is certainly below tol and that step computes X <- X T alone.
//
// Every matrix the iteration touches is a polynomial in A, so all of them are
// symmetric and commute: each product is computed on the upper-triangular
// 64 x 64 tiles only and written to both (i, j) and (j, i).  The products run
// on the float64 tensor-core MMA (mma.sync m8n8k4 .f64).  A ragged statistic
// sits in the top-left corner of its S x S slot; the padding is set to the
// identity in M0, never mixes with the valid corner, and is left out of the
// residual.
#include <float.h>

#include "common.cuh"

namespace shampoo {

namespace {

constexpr int kNewtonThreads = 128;
constexpr int kBK = 16;
constexpr int kAStride = kBK + 4;     // doubles; 4 mod 16 keeps fragment loads conflict-free

enum : int { kRunning = 0, kConverged = 1, kFailed = 2, kDiverged = 3, kFinal = 4 };

__device__ __forceinline__ unsigned long long dbl_bits(double v) {
  return static_cast<unsigned long long>(__double_as_longlong(v));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void dmma884(double& c0, double& c1, double a, double b) {
  asm volatile(
      "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
      : "+d"(c0), "+d"(c1)
      : "d"(a), "d"(b));
}

// Tile (ti, tj) of the upper triangle of a T x T tile grid, from its index.
__device__ __forceinline__ void tri_tile(int idx, int T, int& ti, int& tj) {
  ti = 0;
  while (idx >= T - ti) {
    idx -= T - ti;
    ++ti;
  }
  tj = ti + idx;
}

// Tile side TT (64, or 32 for the last steps, when only a few matrices are
// left and 64 x 64 tiles would leave most SMs idle).
template <int TT>
struct NewtonSmem {
  double As[2][TT][kAStride];
  double Bs[2][kBK][TT + 4];   // row stride = 8 mod 32 words: conflict-free fragment loads
};

// acc = A[i0:i0+TT, :] * B[:, j0:j0+TT] for S x S row-major float64 A, B.
// 4 warps in a 2 x 2 arrangement, each a TT/2 x TT/2 sub-tile of FM x FM
// m8n8 fragments (FM = TT/16); lane (g, t) = (lane / 4, lane % 4) holds
// acc[mi][ni][e] at row 8 mi + g, column 8 ni + 2 t + e of its sub-tile.
template <int TT>
__device__ __forceinline__ void dmma_tile(const double* __restrict__ A, const double* __restrict__ B,
                                          int S, int i0, int j0, double (&acc)[TT / 16][TT / 16][2],
                                          NewtonSmem<TT>& sm) {
  constexpr int FM = TT / 16, HALF = TT / 2;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int wm = warp >> 1, wn = warp & 1;
  auto load = [&](int stage, int k0) {
#pragma unroll
    for (int r = 0; r < TT / 16; ++r) {
      const int c = tid + r * kNewtonThreads;          // TT * 8 16-byte chunks per operand
      const int ar = c >> 3, ac = (c & 7) * 2;         // A: TT rows x 8 chunks
      cp_async16(&sm.As[stage][ar][ac], A + (size_t)(i0 + ar) * S + k0 + ac);
      const int br = c / HALF, bc = (c % HALF) * 2;    // B: 16 rows x TT/2 chunks
      cp_async16(&sm.Bs[stage][br][bc], B + (size_t)(k0 + br) * S + j0 + bc);
    }
    cp_async_commit();
  };
  const int nk = S / kBK;
  // on a diagonal tile the lower-left sub-tile mirrors the upper-right one
  const bool idle = (i0 == j0) && wm == 1 && wn == 0;
  load(0, 0);
  for (int kt = 0; kt < nk; ++kt) {
    if (kt + 1 < nk) {
      load((kt + 1) & 1, (kt + 1) * kBK);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int st = kt & 1;
#pragma unroll
    for (int kk = 0; kk < kBK && !idle; kk += 4) {
      double a[FM], b[FM];
#pragma unroll
      for (int mi = 0; mi < FM; ++mi) a[mi] = sm.As[st][wm * HALF + mi * 8 + g][kk + t];
#pragma unroll
      for (int ni = 0; ni < FM; ++ni) b[ni] = sm.Bs[st][kk + t][wn * HALF + ni * 8 + g];
#pragma unroll
      for (int mi = 0; mi < FM; ++mi)
#pragma unroll
        for (int ni = 0; ni < FM; ++ni) dmma884(acc[mi][ni][0], acc[mi][ni][1], a[mi], b[ni]);
    }
    __syncthreads();
  }
}

// How a warp's sub-tile of a tile is stored: on a diagonal tile the
// lower-left warp computes nothing (its sub-tile mirrors the upper-right
// one); every sub-tile off the matrix diagonal is also written transposed.
__device__ __forceinline__ int warp_weight(int i0, int j0) {
  const int warp = threadIdx.x >> 5, wm = warp >> 1, wn = warp & 1;
  if (i0 != j0) return 2;            // off-diagonal tile: block and mirror
  if (wm == 1 && wn == 0) return 0;  // idle
  return (wm == 0 && wn == 1) ? 2 : 1;
}

// Store the tile to C at (i0, j0) and its mirror image where it has one.
template <int TT>
__device__ __forceinline__ void store_sym(double* __restrict__ C, int S, int i0, int j0,
                                          const double (&acc)[TT / 16][TT / 16][2]) {
  constexpr int FM = TT / 16, HALF = TT / 2;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int wm = warp >> 1, wn = warp & 1;
  const int wgt = warp_weight(i0, j0);
  if (wgt == 0) return;
#pragma unroll
  for (int mi = 0; mi < FM; ++mi)
#pragma unroll
    for (int ni = 0; ni < FM; ++ni) {
      const int r = i0 + wm * HALF + mi * 8 + g;
      const int c = j0 + wn * HALF + ni * 8 + 2 * t;
      *reinterpret_cast<double2*>(C + (size_t)r * S + c) = make_double2(acc[mi][ni][0], acc[mi][ni][1]);
      if (wgt == 2) {
        C[(size_t)c * S + r] = acc[mi][ni][0];
        C[(size_t)(c + 1) * S + r] = acc[mi][ni][1];
      }
    }
}

// ---------------------------------------------------------------------------
// Set-up: the eigenvalue bound, X0, M0, T0 and the first residual.
// ---------------------------------------------------------------------------
// Element (r, c) of a statistic stored as upper 128-tiles (upper = 1) or in
// full (upper = 0).
__device__ __forceinline__ float sym_at(const float* a, int lda, int upper, int r, int c) {
  if (upper && (r >> 7) > (c >> 7)) return a[(size_t)c * lda + r];
  return a[(size_t)r * lda + c];
}

// grid: x = band of 32 rows, y = matrix.  Partial sums of the bound over the
// valid corner: ||A + eps I||_F^2 into fro2[m] and the absolute row sums into
// rows[m][:].  A statistic stored as upper 128-tiles is read row by row: an
// entry of an off-diagonal tile stands for itself and its mirror, so it adds
// twice to the Frobenius sum and to the row sums of both its row and its
// column (the column part accumulated per lane, then per block in shared
// memory, then once per block in global memory).
__global__ void __launch_bounds__(256) newton_bound_partial_kernel(const float* __restrict__ A,
                                                                   int64_t a_stride, int lda, int upper,
                                                                   const NewtonMat* __restrict__ mats,
                                                                   int S, float eps,
                                                                   double* __restrict__ fro2,
                                                                   double* __restrict__ rows) {
  __shared__ double red[8];
  __shared__ double colsum[1024];
  const int m = blockIdx.y;
  const NewtonMat mt = mats[m];
  const float* a = A + (size_t)mt.slot * a_stride;
  const int n = mt.size;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int c = threadIdx.x; c < S; c += blockDim.x) colsum[c] = 0.0;
  __syncthreads();
  double* rsum = rows + (size_t)m * S;
  double fro = 0.0;
  double col[32];   // this lane's mirror contributions, columns lane + 32 k
#pragma unroll
  for (int k = 0; k < 32; ++k) col[k] = 0.0;
  for (int j = 0; j < 4; ++j) {
    const int r = blockIdx.x * 32 + warp + 8 * j;
    if (r >= n) continue;
    const float* row = a + (size_t)r * lda;
    double rs = 0.0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int c = lane + 32 * k;
      if (c >= n) continue;
      const bool mirror = upper && (c >> 7) > (r >> 7);
      if (upper && (c >> 7) < (r >> 7)) continue;   // a lower tile: never written
      double v = (double)row[c];
      if (r == c) v += (double)eps;
      rs += fabs(v);
      fro += (mirror ? 2.0 : 1.0) * v * v;
      if (mirror) col[k] += fabs(v);
    }
    rs = warp_sum(rs);
    if (lane == 0 && rs != 0.0) atomicAdd(&rsum[r], rs);
  }
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int c = lane + 32 * k;
    if (c < n && col[k] != 0.0) atomicAdd(&colsum[c], col[k]);
  }
  fro = block_sum(fro, red);
  __syncthreads();
  for (int c = threadIdx.x; c < n; c += blockDim.x)
    if (colsum[c] != 0.0) atomicAdd(&rsum[c], colsum[c]);
  if (threadIdx.x == 0 && fro != 0.0) atomicAdd(&fro2[m], fro);
}

// One warp per matrix: c^p = min(||A + eps I||_F, ||A + eps I||_inf), both
// bounds of the largest eigenvalue of a symmetric matrix, from the partial
// sums; then the residual and Frobenius slots are cleared for the iteration.
// On a retry (attempt k > 0) the ridge is raised to eps + 8^k 2^-24 c^p:
// rounding of a float32 statistic can leave eigenvalues of A + eps I below
// zero by about 2^-24 c^p, which the iteration cannot root.
__global__ void newton_bound_final_kernel(const NewtonMat* __restrict__ mats, int nm, int S, float eps,
                                          int attempt, NewtonWork w, const double* __restrict__ rows,
                                          double* __restrict__ cpow) {
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (m >= nm) return;
  const NewtonMat mt = mats[m];
  double rowmax = 0.0;
  for (int c = lane; c < mt.size; c += 32) rowmax = fmax(rowmax, rows[(size_t)m * S + c]);
  rowmax = warp_max(rowmax);
  if (lane == 0) {
    double cp = fmin(sqrt(w.fro2[m]), rowmax);
    if (!(cp > 0.0) || !(cp <= DBL_MAX)) cp = (cp > 0.0) ? cp : 1.0;  // NaN/Inf/0 caught later
    double rd = (double)eps;
    if (attempt > 0) {
      const double extra = ldexp(cp, 3 * attempt - 24);
      rd += extra;
      cp += extra;   // lambda_max grows by exactly the added ridge
    }
    w.ridge[m] = rd;
    cpow[m] = cp;
    w.cinv[m] = pow(cp, -1.0 / mt.p);
    w.fro2[m] = 0.0;
    w.resid[m] = 0ull;
  }
}

// grid: x = row of the S x S slot, y = matrix.  Writes X0, M0 into the
// parity-0 buffers and folds max|M0 - I| (valid corner) into the residual.
// Also writes the valid corner of the statistic itself, mirrored, as float32
// into T4 (unused until the first step B): the Lanczos run multiplies by it,
// which is M0 up to the ridge and the scale c^p, at half the bytes.
__global__ void __launch_bounds__(256) newton_init_kernel(const float* __restrict__ A,
                                                          int64_t a_stride, int lda, int upper,
                                                          const NewtonMat* __restrict__ mats,
                                                          int S, NewtonWork w,
                                                          const double* __restrict__ cpow) {
  __shared__ double red[8];
  const int m = blockIdx.y;
  const NewtonMat mt = mats[m];
  const float* a = A + (size_t)mt.slot * a_stride;
  const int r = blockIdx.x;
  const size_t off = (size_t)m * S * S + (size_t)r * S;
  const double inv_cp = 1.0 / cpow[m];
  const double rd = w.ridge[m];
  const double ci = w.cinv[m];
  double dev = 0.0;
  float* a32 = reinterpret_cast<float*>(w.T4 + (size_t)m * S * S) + (size_t)r * S;
  for (int c = threadIdx.x; c < S; c += blockDim.x) {
    double v;
    const bool valid = r < mt.size && c < mt.size;
    if (valid) {
      // a full input is read through its symmetric part (exact when symmetric)
      v = upper ? (double)sym_at(a, lda, upper, r, c)
                : 0.5 * ((double)a[(size_t)r * lda + c] + (double)a[(size_t)c * lda + r]);
      a32[c] = (float)v;
      if (r == c) v += rd;
      v *= inv_cp;
    } else {
      v = (r == c) ? 1.0 : 0.0;
      a32[c] = 0.f;
    }
    const double d = (r == c) ? 1.0 : 0.0;
    w.M[0][off + c] = v;
    w.X[0][off + c] = (r == c) ? ci : 0.0;
    double e = valid ? fabs(v - d) : 0.0;
    if (!(e <= DBL_MAX)) e = INFINITY;
    dev = fmax(dev, e);
  }
  dev = block_max(dev, red);
  if (threadIdx.x == 0) atomicMax(&w.resid[m], dbl_bits(dev));
}

// ---------------------------------------------------------------------------
// Scaling schedule
// ---------------------------------------------------------------------------
constexpr int kLanczos = 12;

// One scalar Newton step on an eigenvalue m of the scaled M: m ((p+1-m)/p)^p.
// p is 2 or 4, so the division is a multiplication by the exact 1/p.
__device__ __forceinline__ double newton_map(double m, int p) {
  const double t = (p + 1 - m) * (p == 4 ? 0.25 : 0.5);
  const double t2 = t * t;
  return m * (p == 4 ? t2 * t2 : t2);
}

// Number of eigenvalues of the symmetric tridiagonal (a, b) below x.
__device__ int sturm_count(const double* a, const double* b, int k, double x) {
  int cnt = 0;
  double d = a[0] - x;
  if (d < 0) ++cnt;
  for (int i = 1; i < k; ++i) {
    const double dd = (d == 0.0) ? 1e-300 : d;
    d = a[i] - x - b[i - 1] * b[i - 1] / dd;
    if (d < 0) ++cnt;
  }
  return cnt;
}

// Multisection over one warp: f is nondecreasing-true on [lo, hi] (false
// below the point sought, true at and above it).  Each round the 32 lanes
// test 32 evenly spaced interior points and the bracket shrinks 33-fold to
// the cell where f turns true; every lane ends with the same bracket.
template <class F>
__device__ void warp_multisect(double& lo, double& hi, int rounds, F f) {
  const int lane = threadIdx.x & 31;
  for (int r = 0; r < rounds; ++r) {
    const double h = (hi - lo) * (1.0 / 33.0);
    const unsigned hit = __ballot_sync(0xffffffffu, f(lo + h * (lane + 1)));
    const int j = hit ? __ffs(hit) - 1 : 32;   // first point where f holds
    const double nlo = lo + h * j;
    if (j < 32) hi = lo + h * (j + 1);
    lo = nlo;
  }
}

// Smallest (which = 1) or largest (which = k) eigenvalue of the tridiagonal:
// Gershgorin bracket, then Sturm counts by warp multisection (12 rounds take
// the bracket down by 33^12, below a double's resolution).  Called by a whole
// warp.
__device__ double tridiag_eig(const double* a, const double* b, int k, int which) {
  double lo = a[0], hi = a[0];
  for (int i = 0; i < k; ++i) {
    const double r = (i > 0 ? fabs(b[i - 1]) : 0.0) + (i + 1 < k ? fabs(b[i]) : 0.0);
    lo = fmin(lo, a[i] - r);
    hi = fmax(hi, a[i] + r);
  }
  warp_multisect(lo, hi, 12, [&](double x) { return sturm_count(a, b, k, x) >= which; });
  return 0.5 * (lo + hi);
}

// One CTA per matrix: kLanczos Lanczos steps on the valid corner of M0
// (float64 vectors, the float32 statistic as the operator; no
// reorthogonalisation: only the extreme Ritz values are used),
// their extreme eigenvalues by Sturm multisection, and the schedule s_k (both on warp 0).
__global__ void __launch_bounds__(512) newton_lanczos_kernel(const NewtonMat* __restrict__ mats, int S,
                                                             NewtonWork w) {
  __shared__ double v[1024], vp[1024], wv[1024];
  __shared__ double al[kLanczos], be[kLanczos];
  __shared__ double red[16];
  __shared__ double bcast;
  const int m = blockIdx.x;
  const NewtonMat mt = mats[m];
  const int n = mt.size, p = mt.p;
  const float* A32 = reinterpret_cast<const float*>(w.T4 + (size_t)m * S * S);   // written by newton_init
  const double rd = w.ridge[m], inv_cp = 1.0 / w.T2[m];                       // T2 holds c^p until step A
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // start vector: a fixed pseudo-random +-1 pattern (hash of the index)
  double ss = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    uint32_t h = (uint32_t)i * 2654435761u;
    h ^= h >> 15;
    const double x = (h & 1u) ? 1.0 : -1.0;
    v[i] = x;
    vp[i] = 0.0;
    ss += x * x;
  }
  ss = block_sum(ss, red);
  if (threadIdx.x == 0) bcast = 1.0 / sqrt(ss);
  __syncthreads();
  const double inv0 = bcast;
  for (int i = threadIdx.x; i < n; i += blockDim.x) v[i] *= inv0;
  const int n4 = (n + 3) >> 2;
  if (threadIdx.x < 4 * n4 - n) v[n + threadIdx.x] = 0.0;   // pad for the 4-wide row loads
  __syncthreads();
  double beta = 0.0;
  int kk = 0;
  for (int j = 0; j < kLanczos && j < n; ++j) {
    // M0 v = ((A + ridge I) v) / c^p with A the float32 statistic (exact
    // values) streamed from memory; every 16-byte load of a warp's two rows is
    // issued before the first is used
    for (int r = 2 * warp; r < n; r += 2 * nw) {
      const bool two = r + 1 < n;
      const float4* row0 = reinterpret_cast<const float4*>(A32 + (size_t)r * S);
      const float4* row1 = reinterpret_cast<const float4*>(A32 + (size_t)(two ? r + 1 : r) * S);
      double d0 = 0.0, d1 = 0.0;
      for (int base = 0; base < n4; base += 128) {   // 512 columns at a time
        float4 x0[4], x1[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c4 = base + lane + 32 * k;
          x0[k] = c4 < n4 ? row0[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
          x1[k] = c4 < n4 ? row1[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c4 = base + lane + 32 * k;
          if (c4 < n4) {
            const int c = 4 * c4;
            d0 = fma((double)x0[k].x, v[c], fma((double)x0[k].y, v[c + 1],
                     fma((double)x0[k].z, v[c + 2], fma((double)x0[k].w, v[c + 3], d0))));
            d1 = fma((double)x1[k].x, v[c], fma((double)x1[k].y, v[c + 1],
                     fma((double)x1[k].z, v[c + 2], fma((double)x1[k].w, v[c + 3], d1))));
          }
        }
      }
      d0 = warp_sum(d0);
      d1 = warp_sum(d1);
      if (lane == 0) {
        wv[r] = (d0 + rd * v[r]) * inv_cp - beta * vp[r];
        if (two) wv[r + 1] = (d1 + rd * v[r + 1]) * inv_cp - beta * vp[r + 1];
      }
    }
    __syncthreads();
    double a = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) a += v[i] * wv[i];
    a = block_sum(a, red);
    if (threadIdx.x == 0) bcast = a;
    __syncthreads();
    a = bcast;
    double b2 = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const double x = wv[i] - a * v[i];
      wv[i] = x;
      b2 += x * x;
    }
    b2 = block_sum(b2, red);
    if (threadIdx.x == 0) bcast = sqrt(b2);
    __syncthreads();
    const double b = bcast;
    if (threadIdx.x == 0) {
      al[j] = a;
      be[j] = b;
    }
    kk = j + 1;
    if (!(b > 1e-13 * fabs(a)) || !(b <= DBL_MAX)) break;   // invariant subspace (or a non-finite value)
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      vp[i] = v[i];
      v[i] = wv[i] / b;
    }
    beta = b;   // the padding v[n .. 4 n4) stays 0
    __syncthreads();
  }
  __syncthreads();
  if (warp != 0) return;
  // interval estimate, kept inside what is guaranteed: [ridge / c^p, 1]; the
  // warp computes it together (the same values in every lane), lane 0 stores
  const double lo_g = w.ridge[m] / w.T2[m];   // T2 holds c^p until the first step
  double l = tridiag_eig(al, be, kk, 1), u = tridiag_eig(al, be, kk, kk);
  int ns = 0;
  double* sch = w.sched + (size_t)m * kSched;
  if (l <= DBL_MAX && u <= DBL_MAX && l > 0.0) {
    u = fmin(1.0, u * 1.02);
    l = fmin(fmax(l, lo_g), u);
    const double cap = 0.98 * (p + 1);
    while (ns < kSched && l < 0.7) {
      // s in [1/u, min((p+1)/u, cap)] with map(s l) = map(s u)
      double a = 1.0 / u, b = fmin((p + 1) / u, cap), s;
      if (newton_map(b * l, p) <= newton_map(b * u, p)) {
        s = b;
      } else {   // 16 rounds: 33^16 > 2^80
        warp_multisect(a, b, 16, [&](double x) { return !(newton_map(x * l, p) < newton_map(x * u, p)); });
        s = 0.5 * (a + b);
      }
      const double x = newton_map(s * l, p), y = newton_map(s * u, p);
      const double nl = fmin(x, y);
      const double nu = (s * l <= 1.0 && s * u >= 1.0) ? 1.0 : fmax(x, y);
      l = nl;
      u = fmax(nu, nl);
      if (lane == 0) sch[ns] = s;
      ++ns;
    }
  }
  if (lane == 0) w.nsched[m] = ns;
}

__device__ __forceinline__ double sched_at(const NewtonWork& w, int m, int k) { return newton_sched(w, m, k); }

// T0 = ((p+1) I - s_0 M0) / p.  grid: x = row, y = matrix.
__global__ void __launch_bounds__(256) newton_t0_kernel(const NewtonMat* __restrict__ mats, int S,
                                                        NewtonWork w) {
  const int m = blockIdx.y, r = blockIdx.x;
  const int p = mats[m].p;
  const double s0 = sched_at(w, m, 0), pinv = 1.0 / p;
  const size_t off = (size_t)m * S * S + (size_t)r * S;
  for (int c = threadIdx.x; c < S; c += blockDim.x)
    w.T[off + c] = ((p + 1) * (r == c ? 1.0 : 0.0) - s0 * w.M[0][off + c]) * pinv;
}

// ---------------------------------------------------------------------------
// One Newton step, three launches:
//   job 0: X_next = X T      job 1: T2 = T T            (launch A)
//   T4 = T2 T2 (p = 4 only)                              (launch B)
//   M_next = T^p M, residual, T <- ((p+1) I - M_next)/p  (launch C)
// grid: x = upper-triangular tile (x 2 jobs in launch A), y = matrix.  The
// two jobs of a tile are neighbours in launch order, so they run side by
// side and read the tile's column panel of T from L2 once between them.
// ---------------------------------------------------------------------------
template <int TT>
__global__ void __launch_bounds__(kNewtonThreads, 4) newton_step_a_kernel(
    const NewtonMat* __restrict__ mats, int S, int it, NewtonWork w) {
  constexpr int FM = TT / 16;
  __shared__ NewtonSmem<TT> sm;
  if ((int)blockIdx.y >= w.count[2]) return;   // the check listed fewer
  const int m = w.live[blockIdx.y];
  const int st = w.state[m];
  const int job = blockIdx.x & 1;
  if (st != kRunning && !(st == kFinal && job == 0)) return;
  const int T = S / TT;
  int ti, tj;
  tri_tile(blockIdx.x >> 1, T, ti, tj);
  const size_t base = (size_t)m * S * S;
  const double* Tm = w.T + base;
  if (job == 0 && it == 0) {
    // X0 = c^{-1} I, so X1 = s_0^{1/p} c^{-1} T0 needs no product: the tile
    // and its mirror (T0 is stored whole) are copied, scaled
    const double sk = sched_at(w, m, 0);
    const double sc = w.cinv[m] * (sk != 1.0 ? pow(sk, 1.0 / mats[m].p) : 1.0);
    double* X1 = w.X[1] + base;
    const int i0 = ti * TT, j0 = tj * TT;
    for (int e = threadIdx.x; e < TT * TT; e += kNewtonThreads) {
      const int a = e / TT, b = e % TT;
      X1[(size_t)(i0 + a) * S + j0 + b] = sc * Tm[(size_t)(i0 + a) * S + j0 + b];
      if (i0 != j0) X1[(size_t)(j0 + a) * S + i0 + b] = sc * Tm[(size_t)(j0 + a) * S + i0 + b];
    }
    return;
  }
  const double* A = job == 0 ? w.X[it & 1] + base : Tm;
  double* C = job == 0 ? w.X[(it + 1) & 1] + base : w.T2 + base;
  double acc[FM][FM][2] = {};
  dmma_tile<TT>(A, Tm, S, ti * TT, tj * TT, acc, sm);
  if (job == 0) {   // X_next = s_k^{1/p} X T
    const double sk = sched_at(w, m, it);
    if (sk != 1.0) {
      const double mu = pow(sk, 1.0 / mats[m].p);
#pragma unroll
      for (int mi = 0; mi < FM; ++mi)
#pragma unroll
        for (int ni = 0; ni < FM; ++ni) {
          acc[mi][ni][0] *= mu;
          acc[mi][ni][1] *= mu;
        }
    }
  }
  store_sym<TT>(C, S, ti * TT, tj * TT, acc);
}

template <int TT>
__global__ void __launch_bounds__(kNewtonThreads, 4) newton_step_b_kernel(
    const NewtonMat* __restrict__ mats, int S, NewtonWork w) {
  constexpr int FM = TT / 16;
  __shared__ NewtonSmem<TT> sm;
  if ((int)blockIdx.y >= w.count[2]) return;   // the check listed fewer
  const int m = w.live[blockIdx.y];
  if (w.state[m] != kRunning || mats[m].p != 4) return;
  const int T = S / TT;
  int ti, tj;
  tri_tile(blockIdx.x, T, ti, tj);
  const size_t base = (size_t)m * S * S;
  double acc[FM][FM][2] = {};
  dmma_tile<TT>(w.T2 + base, w.T2 + base, S, ti * TT, tj * TT, acc, sm);
  store_sym<TT>(w.T4 + base, S, ti * TT, tj * TT, acc);
}

template <int TT>
__global__ void __launch_bounds__(kNewtonThreads, 4) newton_step_c_kernel(
    const NewtonMat* __restrict__ mats, int S, int it, NewtonWork w) {
  constexpr int FM = TT / 16, HALF = TT / 2;
  __shared__ NewtonSmem<TT> sm;
  __shared__ double red[kNewtonThreads / 32];
  if ((int)blockIdx.y >= w.count[2]) return;   // the check listed fewer
  const int m = w.live[blockIdx.y];
  if (w.state[m] != kRunning) return;
  const int p = mats[m].p;
  const int T = S / TT;
  int ti, tj;
  tri_tile(blockIdx.x, T, ti, tj);
  const size_t base = (size_t)m * S * S;
  const double* Tp = (p == 4 ? w.T4 : w.T2) + base;
  double acc[FM][FM][2] = {};
  const int i0 = ti * TT, j0 = tj * TT;
  dmma_tile<TT>(Tp, w.M[it & 1] + base, S, i0, j0, acc, sm);
  // M_next = s_k T^p M
  const double sk = sched_at(w, m, it), sn = sched_at(w, m, it + 1);
#pragma unroll
  for (int mi = 0; mi < FM; ++mi)
#pragma unroll
    for (int ni = 0; ni < FM; ++ni) {
      acc[mi][ni][0] *= sk;
      acc[mi][ni][1] *= sk;
    }
  store_sym<TT>(w.M[(it + 1) & 1] + base, S, i0, j0, acc);
  // residual (valid corner) and the next T = ((p+1) I - s_{k+1} M_next) / p
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int wm = warp >> 1, wn = warp & 1;
  const int n = mats[m].size;
  const double pinv = 1.0 / p;
  const double wgt = warp_weight(i0, j0);   // 0: idle sub-tile, 2: sub-tile and mirror
  double dev = 0.0, f2 = 0.0;
#pragma unroll
  for (int mi = 0; mi < FM; ++mi)
#pragma unroll
    for (int ni = 0; ni < FM; ++ni)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = i0 + wm * HALF + mi * 8 + g;
        const int c = j0 + wn * HALF + ni * 8 + 2 * t + e;
        const double d = (r == c) ? 1.0 : 0.0;
        double x = (wgt > 0 && r < n && c < n) ? fabs(acc[mi][ni][e] - d) : 0.0;
        if (!(x <= DBL_MAX)) x = INFINITY;
        dev = fmax(dev, x);
        f2 += wgt * x * x;                       // mirrored sub-tiles count twice
        acc[mi][ni][e] = ((p + 1) * d - sn * acc[mi][ni][e]) * pinv;
      }
  store_sym<TT>(w.T + base, S, i0, j0, acc);
  dev = block_max(dev, red);
  f2 = block_sum(f2, red);
  if (threadIdx.x == 0) {
    atomicMax(&w.resid[m], dbl_bits(dev));
    atomicAdd(&w.fro2[m], f2);
  }
}

// Convergence test of M_k for every matrix (k = iterations done), in the
// same order as the oracle: non-finite, tolerance, cap, 5 non-decreasing.
// The matrices the next step works on are listed in w.live in index order
// (a ballot and a scan over the warps per 1024 matrices), their number in
// w.count[2] and, for the host, in w.count[k & 1].  One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) newton_check_kernel(int nm, int k, double tol, int max_iters,
                                                            NewtonWork w) {
  __shared__ int wcount[32];
  __shared__ int listed;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) listed = 0;
  __syncthreads();
  for (int m0 = 0; m0 < nm; m0 += blockDim.x) {
    const int m = m0 + threadIdx.x;
    bool keep = false;
    if (m < nm) {
      const int s0 = w.state[m];
      if (s0 == kFinal) {   // its last step computed X alone
        w.state[m] = kConverged;
        w.iters[m] = k;
      } else if (s0 == kRunning) {
        const double r = __longlong_as_double(static_cast<long long>(w.resid[m]));
        const double f = sqrt(w.fro2[m]);
        w.resid[m] = 0ull;
        w.fro2[m] = 0.0;
        w.iters[m] = k;
        // For a PSD A every eigenvalue of M stays in (0, 1], so max|M - I| < 1;
        // a residual above 1.5 means rounding made A + ridge I indefinite.
        int st = kRunning;
        if (!(r <= 1.5)) {
          st = kDiverged;
        } else if (r <= tol) {
          st = kConverged;
        } else if (k >= max_iters) {
          st = kFailed;
        } else if (k >= w.nsched[m] && k > 0 && f <= 0.05 && 0.75 * f * f * (1.0 + f) <= 0.5 * tol) {
          st = kFinal;   // one more step certainly lands below tol: compute X only
        } else if (k >= w.nsched[m]) {   // the scaled steps may raise the residual
          const int wo = (r >= w.prev[m]) ? w.worse[m] + 1 : 0;
          w.worse[m] = wo;
          w.prev[m] = r;
          if (wo >= 5) st = kDiverged;
        }
        w.state[m] = st;
        keep = (st == kRunning || st == kFinal);
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) wcount[warp] = __popc(bal);
    __syncthreads();
    int pos = listed + __popc(bal & ((1u << lane) - 1u));
    for (int q = 0; q < warp; ++q) pos += wcount[q];
    if (keep) w.live[pos] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int q = 0; q < (int)(blockDim.x >> 5); ++q) t += wcount[q];
      listed += t;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    w.count[2] = listed;
    w.count[k & 1] = listed;
  }
}

__global__ void newton_reset_kernel(int nm, NewtonWork w) {
  for (int m = threadIdx.x; m < nm; m += blockDim.x) {
    w.state[m] = kRunning;
    w.resid[m] = 0ull;
    w.fro2[m] = 0.0;
    w.prev[m] = INFINITY;
    w.worse[m] = 0;
    w.iters[m] = 0;
    w.nsched[m] = 0;
  }
}

// grid: x = row, y = matrix.  Converged: X (float32) from the final buffer.
// Failed: keep the old root if there is one, else write c^{-1} I.
__global__ void __launch_bounds__(256) newton_finalize_kernel(
    float* __restrict__ X, int64_t x_stride, int ldx, const NewtonMat* __restrict__ mats, int S,
    NewtonWork w, int* __restrict__ has_root, int32_t* __restrict__ iters_out, int final_pass) {
  const int m = blockIdx.y;
  const NewtonMat mt = mats[m];
  const int st = w.state[m];
  if (st == kDiverged && !final_pass) return;   // retried with a raised ridge
  const int r = blockIdx.x;
  if (r >= ldx) return;
  const bool ok = (st == kConverged);
  if (!ok && has_root && has_root[mt.slot]) return;
  float* x = X + (size_t)mt.slot * x_stride + (size_t)r * ldx;
  const double* src = w.X[w.iters[m] & 1] + (size_t)m * S * S + (size_t)r * S;
  const double ci = w.cinv[m];
  for (int c = threadIdx.x; c < ldx; c += blockDim.x) {
    double v = 0.0;
    if (r < mt.size && c < mt.size) v = ok ? src[c] : (r == c ? ci : 0.0);
    x[c] = (float)v;
  }
  __syncthreads();
  if (r == 0 && threadIdx.x == 0) {
    if (ok && has_root) has_root[mt.slot] = 1;
    if (iters_out) iters_out[mt.slot] = ok ? w.iters[m] : -1 - w.iters[m];
  }
}

}  // namespace

void launch_newton_reset(int nm, NewtonWork w, cudaStream_t s) {
  newton_reset_kernel<<<1, 1024, 0, s>>>(nm, w);
}

// c^p goes to the first nm doubles of T2, and the row sums to the first
// nm * S doubles of T: no step reads either before step A / T0 overwrite them.
void launch_newton_bound_partial(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                                 int nm, int S, float eps, NewtonWork w, cudaStream_t s) {
  cudaMemsetAsync(w.T, 0, (size_t)nm * S * sizeof(double), s);
  newton_bound_partial_kernel<<<dim3((S + 31) / 32, nm), 256, 0, s>>>(A, a_stride, lda, upper, mats, S, eps,
                                                                      w.fro2, w.T);
}

void launch_newton_bound_final(const NewtonMat* mats, int nm, int S, float eps, int attempt, NewtonWork w,
                               cudaStream_t s) {
  newton_bound_final_kernel<<<(nm + 7) / 8, 256, 0, s>>>(mats, nm, S, eps, attempt, w, w.T, w.T2);
}

void launch_newton_bound(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                         int nm, int S, float eps, int attempt, NewtonWork w, cudaStream_t s) {
  launch_newton_bound_partial(A, a_stride, lda, upper, mats, nm, S, eps, w, s);
  launch_newton_bound_final(mats, nm, S, eps, attempt, w, s);
}

void launch_newton_init(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                        int nm, int S, NewtonWork w, cudaStream_t s) {
  newton_init_kernel<<<dim3(S, nm), 256, 0, s>>>(A, a_stride, lda, upper, mats, S, w, w.T2);
}

void launch_newton_lanczos(const NewtonMat* mats, int nm, int S, NewtonWork w, cudaStream_t s) {
  // Each warp streams two rows of the statistic at a time, so a matvec takes
  // n / (2 x warps) dependent passes: small sides use fewer warps per matrix
  // to fit more matrices on the GPU, unless there are few matrices, where
  // every pass is latency and more warps per matrix shorten the chain.
  const int threads = (S <= 128 && nm > 296) ? 128 : ((S <= 256 && nm > 296) ? 256 : 512);
  newton_lanczos_kernel<<<nm, threads, 0, s>>>(mats, S, w);
}

void launch_newton_t0(const NewtonMat* mats, int nm, int S, NewtonWork w, cudaStream_t s) {
  newton_t0_kernel<<<dim3(S, nm), 256, 0, s>>>(mats, S, w);
}

static int num_tri(int S, int tile) {
  const int T = S / tile;
  return T * (T + 1) / 2;
}

void launch_newton_step_a(const NewtonMat* mats, int rows, int S, int it, int tile, NewtonWork w, cudaStream_t s) {
  if (rows < 1) return;
  if (tile == 32)
    newton_step_a_kernel<32><<<dim3(2 * num_tri(S, 32), rows), kNewtonThreads, 0, s>>>(mats, S, it, w);
  else
    newton_step_a_kernel<64><<<dim3(2 * num_tri(S, 64), rows), kNewtonThreads, 0, s>>>(mats, S, it, w);
}

void launch_newton_step_b(const NewtonMat* mats, int rows, int S, int tile, NewtonWork w, cudaStream_t s) {
  if (rows < 1) return;
  if (tile == 32)
    newton_step_b_kernel<32><<<dim3(num_tri(S, 32), rows), kNewtonThreads, 0, s>>>(mats, S, w);
  else
    newton_step_b_kernel<64><<<dim3(num_tri(S, 64), rows), kNewtonThreads, 0, s>>>(mats, S, w);
}

void launch_newton_step_c(const NewtonMat* mats, int rows, int S, int it, int tile, NewtonWork w, cudaStream_t s) {
  if (rows < 1) return;
  if (tile == 32)
    newton_step_c_kernel<32><<<dim3(num_tri(S, 32), rows), kNewtonThreads, 0, s>>>(mats, S, it, w);
  else
    newton_step_c_kernel<64><<<dim3(num_tri(S, 64), rows), kNewtonThreads, 0, s>>>(mats, S, it, w);
}

void launch_newton_check(int nm, int k, double tol, int max_iters, NewtonWork w, cudaStream_t s) {
  newton_check_kernel<<<1, 1024, 0, s>>>(nm, k, tol, max_iters, w);
}

void launch_newton_finalize(float* X, int64_t x_stride, int ldx, const NewtonMat* mats, int nm,
                            int S, NewtonWork w, int* has_root, int32_t* iters_out, int final_pass,
                            cudaStream_t s) {
  newton_finalize_kernel<<<dim3(ldx, nm), 256, 0, s>>>(X, x_stride, ldx, mats, S, w, has_root,
                                                       iters_out, final_pass);
}

}  // namespace shampoo
