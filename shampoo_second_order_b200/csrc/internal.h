// Internal declarations shared by the host planner and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace shampoo {

// One 2-D block of a parameter (a <= b x b tile of the row-major grid).
struct BlockDesc {
  int param;     // parameter index
  int m, n;      // valid rows / cols of the block
  int side;      // factors kept: 0 both, 1 L only, 2 R only (one-sided, Lemma 1)
  int64_t r0, c0;  // top-left element in the parameter
  int64_t ld;    // the parameter's row length (cols)
};

// One segment of a 1-D parameter.
struct SegDesc {
  int param;
  int len;
  int64_t s0;
};

// A contiguous run of one parameter's elements, the unit of the elementwise
// kernels (Adagrad accumulator, graft norms, weight update).
struct ChunkDesc {
  int param;
  int len;
  int64_t start;   // element offset inside the parameter
};

struct ParamDesc {
  int64_t numel;
  int64_t offset;  // element offset into the flat parameter-shaped buffers
};

constexpr int kChunk = 16384;   // elements per elementwise chunk
constexpr int kSched = 32;      // longest Newton scaling schedule
constexpr int kTile = 64;       // tile side of every matrix kernel
// Newton runs per matrix: the first with the ridge eps, then up to three more
// with the ridge raised after a divergence (both batched-root entry points
// and the optimizer's root step).
constexpr int kNewtonAttempts = 4;

// Per-matrix bookkeeping of the Newton root iteration.
struct NewtonMat {
  int slot;        // statistic slot (stats / roots arrays)
  int size;        // valid side
  int p;           // root order
  int pad;
};

// TMA descriptors of the library's bf16 operand planes (128-byte swizzle):
//  gk   gathered gradient blocks [planes*nblk][S][S], box 64 x 128 (K-major)
//  gmn  the same tensor, box 64 x 64 (MN-major loads of G^T)
//  rk   root planes [2*nmat][S][S] (hi then lo), box 64 x 128
//  ymn  Y = G R^{-1/p} planes [2*nblk][S][S], box 64 x 64 (MN-major)
//  ck   statistics fp32 [nmat][S][S], box 32 x 128 (the update's read-modify-write)
struct TcMaps {
  CUtensorMap gk, gmn, rk, ymn, ck;
  // the gradient planes as [plane][block][row][col], for boxes that carry
  // both planes of a panel (the statistics)
  CUtensorMap gk4, gmn4;
};

// ---------------- tensor-core kernels (k_tc.cu) ----------------
// also flags (atomically) a parameter whose gradient holds NaN or Inf
cudaError_t launch_gather(const BlockDesc* blocks, int nblk, const void* const* gptr, int bf16,
                          int* flags, int S, uint16_t* out, cudaStream_t s);
cudaError_t launch_split(const float* x, int64_t n, uint16_t* out, cudaStream_t s);
// a wait that runs out: sets *err to the timeout code after about a second
cudaError_t launch_stalled_wait(int* err, cudaStream_t s);
// stall != 0 (failure-path test only): the MMA issuer first waits on a
// barrier phase that nothing completes, runs out and aborts the launch
cudaError_t launch_stats_tc(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk,
                            int nmat, int S, int planes_g, float beta2, float* stats, int* err,
                            cudaStream_t s, int stall = 0);
cudaError_t launch_apply_y_tc(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk,
                              int nmat, int S, int planes_g, uint16_t* y, int* err, cudaStream_t s,
                              int stall = 0);
cudaError_t launch_apply_p_tc(const TcMaps& maps, const BlockDesc* blocks, const ParamDesc* params,
                              const int* flags, int nblk, int nmat, int S, float* P, double* p2,
                              int* err, cudaStream_t s);

// ---------------- the GEMMs on CTA pairs (k_tc2.cu) ----------------
bool pair_gemm_supported(int S);   // S a multiple of 256
// the apply GEMMs on 256 x 256 pair tiles
// stall != 0 (failure-path test only): as for launch_stats_tc
cudaError_t launch_apply_y_pair(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk, int nmat,
                                int S, int planes_g, uint16_t* y, int* err, cudaStream_t s, int stall = 0);
cudaError_t launch_apply_p_pair(const TcMaps& maps, const BlockDesc* blocks, const ParamDesc* params,
                                const int* flags, int nblk, int nmat, int S, float* P, double* p2, int* err,
                                cudaStream_t s);

// ---------------- stats (k_stats.cu) ----------------
void launch_check_finite(const ChunkDesc* chunks, int nchunks, const void* const* gptr,
                         int bf16, int* flags, cudaStream_t s);
// a <- beta2 a + g*g, and d2[param] += sum (g / sqrt(a + eps))^2
void launch_diag_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                        const void* const* gptr, int bf16, const int* flags, float beta2, float eps,
                        float* a, double* d2, cudaStream_t s);
void launch_stats_segments(const SegDesc* segs, int nseg, int mat0, const void* const* gptr,
                           int bf16, const int* flags, float beta2, float* stats, int S,
                           cudaStream_t s);

// ---------------- roots (k_roots.cu) ----------------
struct NewtonWork {
  double* X[2];
  double* M[2];
  double* T;
  double* T2;
  double* T4;
  double* cinv;                 // [nmat] c^{-1}
  double* ridge;                // [nmat] ridge added to A (eps, raised on a retry)
  double* sched;                // [nmat][kSched] scaling s_k of the first steps
  int* nsched;                  // [nmat] number of scaled steps
  unsigned long long* resid;    // [nmat] max|M-I| as ordered bits
  double* fro2;                 // [nmat] ||M-I||_F^2 of the valid corner
  double* prev;                 // [nmat] previous residual
  int* worse;                   // [nmat]
  int* live;                    // [nmat] the matrices the next step works on (running or
                                //        X-only), in index order, listed by each check
  int* iters;                   // [nmat] iterations done
  int* state;                   // [nmat] 0 running, 1 converged, 2 failed, 3 diverged,
                                //        4 one X-only step left
  int* count;                   // [3] matrices still active after check k: [k & 1] for the
                                //     host to read back, [2] the length of `live`
  // int8 slices of the iterates for the emulated-float64 products (k_ozaki.cu):
  //   q   int8 [kOzSets][qs][qcap][S][S], slice k of set z for matrix m at
  //       plane (z * qs + k) * qcap + m
  //   qe  int32 [kOzSets][qcap][S], the row exponents
  int8_t* q;
  int* qe;
  int qs;                       // slices per value
  int qcap;                     // matrices the slice planes hold
};

// Matrix sets sliced for the emulated products.
enum : int { kOzX = 0, kOzT = 1, kOzT2 = 2, kOzT4 = 3, kOzM = 4, kOzSets = 5 };
constexpr int kOzMaxSlices = 6;   // accumulators of 64 TMEM columns, rotating over 8 slots
// TMA descriptors over the int8 slice planes [kOzSets * qs * qcap][S][S]
// (64-byte swizzle, K-major): a  box 64 (K) x 128 rows, b  box 64 x 64 rows.
struct OzakiMaps {
  CUtensorMap a, b;
};
// Set up X0, M0, T0 for `nm` matrices read from `A` (float32, slot-strided
// `a_stride` elements apart, row stride `lda`, valid side mats[i].size).
void launch_newton_reset(int nm, NewtonWork w, cudaStream_t s);
// attempt 0 uses the ridge eps; attempt k > 0 raises it to
// eps + 8^k 2^-24 c^p (the fp32 resolution of the statistic).
// upper: A holds only its upper-triangular 128 x 128 tiles; element (r, c)
// of a lower tile is read from (c, r).
void launch_newton_bound(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                         int nm, int S, float eps, int attempt, NewtonWork w, cudaStream_t s);
// the two kernels of launch_newton_bound: partial sums over row bands, then c^p
void launch_newton_bound_partial(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                                 int nm, int S, float eps, NewtonWork w, cudaStream_t s);
void launch_newton_bound_final(const NewtonMat* mats, int nm, int S, float eps, int attempt, NewtonWork w,
                               cudaStream_t s);
void launch_newton_init(const float* A, int64_t a_stride, int lda, int upper, const NewtonMat* mats,
                        int nm, int S, NewtonWork w, cudaStream_t s);
// Lanczos estimate of M0's spectrum and the scaling schedule, then T0.
void launch_newton_lanczos(const NewtonMat* mats, int nm, int S, NewtonWork w, cudaStream_t s);
void launch_newton_t0(const NewtonMat* mats, int nm, int S, NewtonWork w, cudaStream_t s);
// one Newton step: A (X T and T T), B (T2 T2, p = 4 only), C (T^p M,
// residual, next T) on tiles of side `tile` (64, or 32 when few matrices are
// left); check k: convergence test of M_k
// One Newton step over the matrices the last check listed in w.live; `rows`
// (the grid's matrix extent) is any upper bound on their number, e.g. the
// count a previous check reported.
void launch_newton_step_a(const NewtonMat* mats, int rows, int S, int it, int tile, NewtonWork w, cudaStream_t s);
void launch_newton_step_b(const NewtonMat* mats, int rows, int S, int tile, NewtonWork w, cudaStream_t s);
void launch_newton_step_c(const NewtonMat* mats, int rows, int S, int it, int tile, NewtonWork w, cudaStream_t s);
void launch_newton_check(int nm, int k, double tol, int max_iters, NewtonWork w, cudaStream_t s);

// ---------------- emulated float64 Newton products (k_ozaki.cu) ----------------
// Slice the listed sets (bit z of `sets` = set z) of every running matrix:
// per row an exponent e with max|v| < 2^e and qs signed 7-bit slices of the
// truncated fixed-point value v 2^-e.
cudaError_t launch_ozaki_split(const NewtonMat* mats, int nm, int S, int it, unsigned sets, NewtonWork w,
                               cudaStream_t s);
// The products of one Newton step on the int8 tensor cores; step = 0 (A:
// X T and T T), 1 (B: T2 T2, p = 4), 2 (C: T^p M with the residual and next T).
cudaError_t launch_ozaki_step(const OzakiMaps& maps, int step, const NewtonMat* mats, int nm, int S, int it,
                              NewtonWork w, int* err, cudaStream_t s);
// Write the roots back as float32.  keep_old: leave a failed matrix's slot
// untouched if has_root[slot] is set; else write c^{-1} I.
// A diverged matrix is skipped unless final_pass (it will be retried).
void launch_newton_finalize(float* X, int64_t x_stride, int ldx, const NewtonMat* mats, int nm,
                            int S, NewtonWork w, int* has_root, int32_t* iters_out, int final_pass,
                            cudaStream_t s);

// ---------------- apply (k_apply.cu) ----------------
void launch_dnorm(const ChunkDesc* chunks, int nchunks, const ParamDesc* params,
                  const void* const* gptr, int bf16, const int* flags, const float* a, float eps,
                  double* d2, cudaStream_t s);
void launch_precondition_segments(const SegDesc* segs, int nseg, int mat0, const ParamDesc* params,
                                  const void* const* gptr, int bf16, const int* flags,
                                  const float* roots, int S, float* P, double* p2,
                                  cudaStream_t s);
void launch_update(const ChunkDesc* chunks, int nchunks, const ParamDesc* params, float* const* wptr,
                   const int* flags, const float* P, const double* d2, const double* p2, int graft,
                   float mu, float lr, float* mom, cudaStream_t s);

}  // namespace shampoo
