// C-ABI of the library (include/shampoo.h): the host-side planner that builds
// the block table, owns the device state and sequences the kernels of one
// optimizer step on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <condition_variable>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "../../include/shampoo.h"
#include "internal.h"

using namespace shampoo;

namespace {

// Per-kernel launch counts and, when enabled, CUDA-event times taken on the
// launching stream around each launch.  The asynchronous root thread launches
// through the same profiler, hence the lock.
struct Profiler {
  struct Entry {
    std::string name;
    int64_t launches = 0;
    double ms = 0.0;
  };
  struct Pending {
    int entry;
    cudaEvent_t a, b;
  };
  bool on = false;
  std::vector<Entry> entries;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  mutable std::mutex mu;

  int find(const char* name) {
    for (size_t i = 0; i < entries.size(); ++i)
      if (entries[i].name == name) return (int)i;
    entries.push_back(Entry{name, 0, 0.0});
    return (int)entries.size() - 1;
  }
  cudaEvent_t event() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  template <class F>
  void launch(const char* name, cudaStream_t s, F&& f) {
    std::lock_guard<std::mutex> lock(mu);
    const int e = find(name);
    ++entries[e].launches;
    if (!on) {
      f();
      return;
    }
    cudaEvent_t a = event(), b = event();
    cudaEventRecord(a, s);
    f();
    cudaEventRecord(b, s);
    pending.push_back(Pending{e, a, b});
  }
  cudaError_t flush() {
    std::lock_guard<std::mutex> lock(mu);
    return flush_locked();
  }
  cudaError_t flush_locked() {
    cudaError_t err = cudaSuccess;
    for (auto& p : pending) {
      float ms = 0.f;
      cudaError_t e = cudaEventSynchronize(p.b);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.a, p.b);
      if (e != cudaSuccess) err = e;
      entries[p.entry].ms += ms;
      pool.push_back(p.a);
      pool.push_back(p.b);
    }
    pending.clear();
    return err;
  }
  void reset(bool timing) {
    std::lock_guard<std::mutex> lock(mu);
    flush_locked();
    entries.clear();
    on = timing;
  }
  int count() const {
    std::lock_guard<std::mutex> lock(mu);
    return (int)entries.size();
  }
  bool entry(int index, Entry* out) {
    std::lock_guard<std::mutex> lock(mu);
    if (index < 0 || index >= (int)entries.size()) return false;
    *out = entries[index];
    return true;
  }
  ~Profiler() {
    flush();
    for (auto e : pool) cudaEventDestroy(e);
  }
};

// Launch through the profiler when there is one.
template <class F>
void run(Profiler* pr, const char* name, cudaStream_t s, F&& f) {
  if (pr) pr->launch(name, s, f);
  else f();
}

}  // namespace

struct shampoo_ctx {
  cudaStream_t stream = nullptr;
  // the accumulator and the small 1-D kernels run beside the tensor-core
  // GEMMs on this stream (same priority as `stream`), forked and joined with
  // events
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_mid = nullptr, ev_join = nullptr;
  int nparams = 0, b = 0, S = 0, p = 4, graft = 1, bf16 = 0;
  float beta2 = 1.f, eps = 1e-6f, mu = 0.f;
  double tol = 1e-6;
  int max_iters = 100;

  std::vector<ParamDesc> params;
  std::vector<int> ndim;
  std::vector<BlockDesc> blocks;
  std::vector<SegDesc> segs;
  std::vector<ChunkDesc> chunks;
  std::vector<ChunkDesc> chunks1d;   // chunks of the 1-D parameters only
  std::vector<NewtonMat> mats;       // per statistic slot (p = 0: a dropped one-sided factor)
  std::vector<NewtonMat> run_mats;   // the slots the root computation runs on
  std::vector<int> param_side;       // per parameter: 0 both factors, 1 L only, 2 R only
  int64_t total = 0;
  int nmat = 0;

  // device
  ParamDesc* d_params = nullptr;
  BlockDesc* d_blocks = nullptr;
  SegDesc* d_segs = nullptr;
  ChunkDesc* d_chunks = nullptr;
  ChunkDesc* d_chunks1d = nullptr;
  NewtonMat* d_mats = nullptr;       // device copy of run_mats
  const void** d_gptr = nullptr;
  float** d_wptr = nullptr;
  float* stats = nullptr;
  float* roots = nullptr;
  float* a = nullptr;
  float* mom = nullptr;
  float* P = nullptr;
  uint16_t* gblk = nullptr;     // gathered gradient planes [planes_g*nblk][S][S] (h, m)
  uint16_t* rplanes = nullptr;  // root planes [2*nmat][S][S]
  uint16_t* yplanes = nullptr;  // Y planes [2*nblk][S][S]
  TcMaps maps{};
  int planes_g = 1;
  int* d_err = nullptr;
  // pointer tables as last uploaded to d_gptr / d_wptr
  std::vector<const void*> sent_gptr;
  std::vector<float*> sent_wptr;
  std::vector<const void*> gathered_from;   // gradient pointers of the last gather
  std::vector<const void*> stats_from;      // gradient pointers of the last update_stats
  double* d2 = nullptr;   // [nparams] ||D||^2 of the graft target
  double* p2 = nullptr;   // [nparams] ||P||^2
  int* flags = nullptr;
  int* has_root = nullptr;
  NewtonWork nw{};
  NewtonMat* d_retry = nullptr;
  int newton_chunk = 0;
  int root_method = SHAMPOO_ROOTS_FP64;   // or SHAMPOO_ROOTS_INT8_EMULATED
  int oz_slices = 6;
  OzakiMaps oz{};                          // over nw.q, once allocated
  int* h_count = nullptr;   // pinned [3]: Newton counts [0..1], a copy of the error word [2]
  int stall_next_stats = 0;  // failure-path test: the next statistics GEMM stalls and aborts
  int stall_next_apply = 0;  // failure-path test: the next apply's first GEMM stalls and aborts
  int pair_tiles = 1;        // 256 x 256 CTA-pair tiles for the apply GEMMs where the block side allows
  cudaEvent_t ev[2] = {nullptr, nullptr};
  std::vector<void*> allocs;

  bool stats_done = false, roots_done = false;
  int last_not_converged = 0, last_max_iters = 0;
  int64_t generation = 0;            // root sets put in use so far
  // the batched root call allocates from this stream-ordered pool (not owned)
  cudaMemPool_t pool = nullptr;
  cudaStream_t pool_stream = nullptr;
  std::vector<int32_t> root_iters;   // per matrix, last compute_roots (-1-k: gave up at k)
  Profiler prof;
  std::string err;
  int device = 0;

  // Asynchronous root pipeline: a host thread runs the Newton iteration on a
  // copy of the statistics, on its own low-priority stream, into the second
  // set of roots; an install swaps the two sets.  `job` and the job_* results
  // are guarded by mu; the buffers below belong to the job while it runs.
  enum Job { kIdle, kQueued, kRunning, kDone };
  cudaStream_t side = nullptr;
  cudaEvent_t ev_submit = nullptr;   // recorded on `stream` after the statistics copy
  float* stats_snap = nullptr;
  float* roots_back = nullptr;
  uint16_t* rplanes_back = nullptr;
  std::thread worker;
  std::mutex job_mu;
  std::condition_variable cv;
  Job job = kIdle;
  bool quit = false;
  shampoo_status job_status = SHAMPOO_OK;
  std::string job_err;
  int job_nf = 0, job_mi = 0;
  std::vector<int32_t> job_iters;
  double job_tol = 1e-6;   // stopping rule and product method captured when the job was queued
  int job_max_iters = 100;
  bool job_oz = false;
};

namespace {

thread_local std::string g_create_err;

shampoo_status fail(shampoo_ctx* c, shampoo_status st, const std::string& msg) {
  if (c) c->err = msg; else g_create_err = msg;
  return st;
}

shampoo_status cuda_fail(shampoo_ctx* c, cudaError_t e, const char* what) {
  return fail(c, SHAMPOO_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define CK(call)                                               \
  do {                                                         \
    cudaError_t e_ = (call);                                   \
    if (e_ != cudaSuccess) return cuda_fail(ctx, e_, #call);   \
  } while (0)

template <class T>
cudaError_t dalloc(shampoo_ctx* ctx, T** p, size_t count) {
  *p = nullptr;
  if (count == 0) return cudaSuccess;
  void* q = nullptr;
  cudaError_t e = ctx->pool ? cudaMallocFromPoolAsync(&q, count * sizeof(T), ctx->pool, ctx->pool_stream)
                            : cudaMalloc(&q, count * sizeof(T));
  if (e == cudaSuccess) {
    ctx->allocs.push_back(q);
    *p = static_cast<T*>(q);
  }
  return e;
}

template <class T>
shampoo_status upload(shampoo_ctx* ctx, T** dst, const std::vector<T>& v) {
  cudaError_t e = dalloc(ctx, dst, v.size());
  if (e != cudaSuccess) return fail(ctx, SHAMPOO_ENOMEM, "cudaMalloc of the block table failed");
  if (v.empty()) return SHAMPOO_OK;
  if (ctx->pool)   // stream-ordered memory: copy in the allocation's stream (pageable source: staged before return)
    CK(cudaMemcpyAsync(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice, ctx->pool_stream));
  else
    CK(cudaMemcpy(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice));
  return SHAMPOO_OK;
}

// Newton work space for `chunk` matrices of side S.
cudaError_t alloc_newton(shampoo_ctx* ctx, NewtonWork& w, int chunk, int S) {
  const size_t mat = (size_t)chunk * S * S;
  cudaError_t e = cudaSuccess;
  double** bufs[7] = {&w.X[0], &w.X[1], &w.M[0], &w.M[1], &w.T, &w.T2, &w.T4};
  for (auto b : bufs)
    if ((e = dalloc(ctx, b, mat)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.cinv, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.ridge, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.sched, (size_t)chunk * kSched)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.nsched, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.resid, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.fro2, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.prev, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.worse, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.iters, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.state, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.live, chunk)) != cudaSuccess) return e;
  if ((e = dalloc(ctx, &w.count, 3)) != cudaSuccess) return e;
  return e;
}

// Run the Newton iteration over the matrices hm (device copy dm) in chunks of
// `chunk`.  A matrix whose iteration diverges (rounding left A + eps I
// indefinite) is run again with the ridge raised, up to kNewtonAttempts times.
// Reports the number of matrices that gave up, the largest iteration count
// and, per matrix slot, the iterations (-1-k when it gave up at k).
shampoo_status run_newton(shampoo_ctx* ctx, Profiler* pr, const std::vector<NewtonMat>& hm,
                          const NewtonMat* dm, NewtonMat* d_retry, const float* A,
                          int64_t a_stride, int lda, int upper, float* X, int64_t x_stride, int ldx, int S,
                          float eps, double tol, int max_iters, int chunk, NewtonWork& w,
                          int* has_root, int32_t* iters_out, int* h_count, cudaEvent_t* ev,
                          cudaStream_t st, int* n_failed, int* max_it,
                          std::vector<int32_t>* per_slot, const OzakiMaps* oz = nullptr,
                          int* oz_err = nullptr) {
  *n_failed = 0;
  *max_it = 0;
  const int nm_all = (int)hm.size();
  int max_slot = 0;
  for (const auto& m : hm) max_slot = std::max(max_slot, m.slot + 1);
  if (per_slot) per_slot->assign(max_slot, 0);
  std::vector<int> hstate(chunk), hiters(chunk);
  for (int c0 = 0; c0 < nm_all; c0 += chunk) {
    std::vector<NewtonMat> list(hm.begin() + c0, hm.begin() + std::min(nm_all, c0 + chunk));
    const NewtonMat* d = dm + c0;
    std::vector<int> done_iters(list.size(), 0);
    for (int attempt = 0; attempt < kNewtonAttempts && !list.empty(); ++attempt) {
      const int nm = (int)list.size();
      int has_p4 = 0;
      for (const auto& m : list) has_p4 |= (m.p == 4);
      run(pr, "newton_reset", st, [&] { launch_newton_reset(nm, w, st); });
      run(pr, "newton_bound", st, [&] {
        launch_newton_bound_partial(A, a_stride, lda, upper, d, nm, S, eps, w, st);
      });
      run(pr, "newton_bound_final", st, [&] { launch_newton_bound_final(d, nm, S, eps, attempt, w, st); });
      run(pr, "newton_init", st, [&] { launch_newton_init(A, a_stride, lda, upper, d, nm, S, w, st); });
      run(pr, "newton_lanczos", st, [&] { launch_newton_lanczos(d, nm, S, w, st); });
      run(pr, "newton_t0", st, [&] { launch_newton_t0(d, nm, S, w, st); });
      cudaError_t oe = cudaSuccess;
      if (oz)
        run(pr, "ozaki_split", st, [&] {
          oe = launch_ozaki_split(d, nm, S, 0, (1u << kOzX) | (1u << kOzT) | (1u << kOzM), w, st);
        });
      run(pr, "newton_check", st, [&] { launch_newton_check(nm, 0, tol, max_iters, w, st); });
      CK(cudaMemcpyAsync(&h_count[0], &w.count[0], sizeof(int), cudaMemcpyDeviceToHost, st));
      CK(cudaEventRecord(ev[0], st));
      int known = nm;   // matrices iterating, as last read back (an upper bound)
      for (int it = 0; it < max_iters; ++it) {
        // the check of M_it is in flight; queue step it+1 before waiting for it
        if (oz) {   // the same step with emulated float64 products on the int8 tensor cores
          run(pr, "ozaki_step_a", st, [&] { oe = launch_ozaki_step(*oz, 0, d, nm, S, it, w, oz_err, st); });
          run(pr, "ozaki_split", st, [&] {
            oe = launch_ozaki_split(d, nm, S, it + 1, (1u << kOzX) | (1u << kOzT2), w, st);
          });
          if (has_p4) {
            run(pr, "ozaki_step_b", st, [&] { oe = launch_ozaki_step(*oz, 1, d, nm, S, it, w, oz_err, st); });
            run(pr, "ozaki_split", st, [&] { oe = launch_ozaki_split(d, nm, S, it + 1, 1u << kOzT4, w, st); });
          }
          run(pr, "ozaki_step_c", st, [&] { oe = launch_ozaki_step(*oz, 2, d, nm, S, it, w, oz_err, st); });
          run(pr, "ozaki_split", st, [&] {
            oe = launch_ozaki_split(d, nm, S, it + 1, (1u << kOzM) | (1u << kOzT), w, st);
          });
          if (oe != cudaSuccess) return cuda_fail(ctx, oe, "emulated Newton step");
        } else {
          // 32 x 32 tiles once so few matrices are left (the count known on
          // the host bounds the running ones) that 64 x 64 tiles would fill
          // under two CTAs per SM
          const int t64 = (S / 64) * (S / 64 + 1) / 2;
          const int tile = (int64_t)known * t64 * 2 <= 2 * 148 ? 32 : 64;
          // the grid covers `known` matrices; the check before this step
          // listed the running ones (at most that many) in w.live
          run(pr, "newton_step_a", st, [&] { launch_newton_step_a(d, known, S, it, tile, w, st); });
          if (has_p4) run(pr, "newton_step_b", st, [&] { launch_newton_step_b(d, known, S, tile, w, st); });
          run(pr, "newton_step_c", st, [&] { launch_newton_step_c(d, known, S, it, tile, w, st); });
        }
        run(pr, "newton_check", st, [&] { launch_newton_check(nm, it + 1, tol, max_iters, w, st); });
        const int nx = (it + 1) & 1;
        CK(cudaGetLastError());
        CK(cudaMemcpyAsync(&h_count[nx], &w.count[nx], sizeof(int), cudaMemcpyDeviceToHost, st));
        CK(cudaEventRecord(ev[nx], st));
        CK(cudaEventSynchronize(ev[it & 1]));
        if (h_count[it & 1] == 0) break;
        known = h_count[it & 1];
      }
      CK(cudaMemcpyAsync(hstate.data(), w.state, nm * sizeof(int), cudaMemcpyDeviceToHost, st));
      CK(cudaMemcpyAsync(hiters.data(), w.iters, nm * sizeof(int), cudaMemcpyDeviceToHost, st));
      CK(cudaStreamSynchronize(st));
      std::vector<NewtonMat> again;
      for (int i = 0; i < nm; ++i)
        if (hstate[i] == 3) again.push_back(list[i]);
      const int final_pass = (attempt == kNewtonAttempts - 1) || again.empty();
      run(pr, "newton_finalize", st, [&] {
        launch_newton_finalize(X, x_stride, ldx, d, nm, S, w, has_root, iters_out, final_pass, st);
      });
      CK(cudaGetLastError());
      for (int i = 0; i < nm; ++i) {
        const int slot = list[i].slot;
        const int k = hiters[i];
        if (hstate[i] == 1 || hstate[i] == 2 || final_pass) {
          if (hstate[i] != 1) ++*n_failed;
          *max_it = std::max(*max_it, k);
          if (per_slot) (*per_slot)[slot] = hstate[i] == 1 ? k : -1 - k;
        }
      }
      if (final_pass) break;
      list.swap(again);
      CK(cudaMemcpyAsync(d_retry, list.data(), list.size() * sizeof(NewtonMat),
                         cudaMemcpyHostToDevice, st));
      CK(cudaStreamSynchronize(st));   // list is pageable host memory reused below
      d = d_retry;
    }
  }
  return SHAMPOO_OK;
}

shampoo_status set_pointers(shampoo_ctx* ctx, const void* const* grads, float* const* params) {
  if (!grads) return fail(ctx, SHAMPOO_EINVAL, "grads is NULL");
  for (int i = 0; i < ctx->nparams; ++i)
    if (!grads[i]) return fail(ctx, SHAMPOO_EINVAL, "grads[" + std::to_string(i) + "] is NULL");
  // pageable source: staged by the driver before the call returns; tables
  // that equal the last ones uploaded are not sent again
  if (!std::equal(grads, grads + ctx->nparams, ctx->sent_gptr.begin(), ctx->sent_gptr.end())) {
    CK(cudaMemcpyAsync(ctx->d_gptr, grads, ctx->nparams * sizeof(void*), cudaMemcpyHostToDevice,
                       ctx->stream));
    ctx->sent_gptr.assign(grads, grads + ctx->nparams);
  }
  if (params) {
    for (int i = 0; i < ctx->nparams; ++i)
      if (!params[i]) return fail(ctx, SHAMPOO_EINVAL, "params[" + std::to_string(i) + "] is NULL");
    if (!std::equal(params, params + ctx->nparams, ctx->sent_wptr.begin(), ctx->sent_wptr.end())) {
      CK(cudaMemcpyAsync(ctx->d_wptr, params, ctx->nparams * sizeof(float*), cudaMemcpyHostToDevice,
                         ctx->stream));
      ctx->sent_wptr.assign(params, params + ctx->nparams);
    }
  }
  return SHAMPOO_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D tensor [depth][S][S] of bf16 (or fp32) with a box of box_x (inner) x
// box_y rows, 128-byte swizzle.
bool encode_planes(CUtensorMap* m, void* base, int S, int64_t depth, int box_x, int box_y,
                   bool fp32 = false) {
  auto fn = encode_fn();
  if (!fn || depth < 1) return false;
  const cuuint64_t esz = fp32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)S, (cuuint64_t)S, (cuuint64_t)depth};
  cuuint64_t strides[2] = {(cuuint64_t)S * esz, (cuuint64_t)S * S * esz};
  cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The gradient planes [planes][nblk][S][S] bf16 as a 4-D tensor (col, row,
// block, plane) whose boxes hold `planes` planes of one block's panel.
bool encode_planes4(CUtensorMap* m, void* base, int S, int64_t nblk, int planes, int box_x, int box_y) {
  auto fn = encode_fn();
  if (!fn || nblk < 1) return false;
  cuuint64_t dims[4] = {(cuuint64_t)S, (cuuint64_t)S, (cuuint64_t)nblk, (cuuint64_t)planes};
  cuuint64_t strides[3] = {(cuuint64_t)S * 2, (cuuint64_t)S * S * 2, (cuuint64_t)nblk * S * S * 2};
  cuuint32_t box[4] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1, (cuuint32_t)planes};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr const char* kTimeoutMsg =
    "a tensor-core kernel timed out waiting on its pipeline and aborted; the optimizer state of this "
    "context is no longer valid (destroy it and start a new one)";

// A kernel that gave up on a wait leaves a code in the error word; the word
// is never cleared, so once set every later check reports it.
shampoo_status check_kernel_error(shampoo_ctx* ctx) {
  int e = 0;
  CK(cudaMemcpyAsync(&e, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  if (e) {
    if (ctx->h_count) ctx->h_count[2] = e;   // later polls refuse at once
    return fail(ctx, SHAMPOO_ECUDA, kTimeoutMsg);
  }
  return SHAMPOO_OK;
}

// Non-blocking check at the start of a step call: every apply leaves a copy of
// the error word in pinned host memory (copied in stream order after its
// kernels), so a time-out of an earlier step is seen without waiting.
shampoo_status poll_kernel_error(shampoo_ctx* ctx) {
  if (ctx->h_count && *reinterpret_cast<volatile int*>(&ctx->h_count[2]))
    return fail(ctx, SHAMPOO_ECUDA, kTimeoutMsg);
  return SHAMPOO_OK;
}

// Gather the 2-D gradients into the blocked bf16 planes unless the planes
// already hold these very gradient pointers from this step's update_stats.
shampoo_status gather(shampoo_ctx* ctx, const void* const* grads, bool force) {
  const int nblk = (int)ctx->blocks.size();
  if (!nblk) return SHAMPOO_OK;
  bool same = !force && ctx->gathered_from.size() == (size_t)ctx->nparams;
  for (int i = 0; same && i < ctx->nparams; ++i) same = ctx->gathered_from[i] == grads[i];
  if (same) return SHAMPOO_OK;
  cudaError_t e = cudaSuccess;
  run(&ctx->prof, "gather", ctx->stream, [&] {
    e = launch_gather(ctx->d_blocks, nblk, ctx->d_gptr, ctx->bf16, ctx->flags, ctx->S, ctx->gblk,
                      ctx->stream);
  });
  if (e != cudaSuccess) return cuda_fail(ctx, e, "gather");
  ctx->gathered_from.assign(grads, grads + ctx->nparams);
  return SHAMPOO_OK;
}

// Slice planes of the emulated products, allocated on first use: room for
// kOzMaxSlices slices of kOzSets iterates of every matrix of a Newton chunk.
shampoo_status ensure_ozaki(shampoo_ctx* ctx) {
  if (ctx->nw.q) return SHAMPOO_OK;
  const int S = ctx->S, cap = ctx->newton_chunk;
  const int64_t planes = (int64_t)kOzSets * kOzMaxSlices * cap;
  int8_t* q = nullptr;
  int* qe = nullptr;
  cudaError_t e = dalloc(ctx, &q, (size_t)planes * S * S);
  if (e == cudaSuccess) e = dalloc(ctx, &qe, (size_t)kOzSets * cap * S);
  if (e != cudaSuccess) return fail(ctx, SHAMPOO_ENOMEM, std::string("int8 slice planes: ") + cudaGetErrorString(e));
  auto fn = encode_fn();
  cuuint64_t dims[3] = {(cuuint64_t)S, (cuuint64_t)S, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)S, (cuuint64_t)S * S};
  cuuint32_t box_a[3] = {64, 128, 1}, box_b[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  if (!fn ||
      fn(&ctx->oz.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box_a, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      fn(&ctx->oz.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box_b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(ctx, SHAMPOO_ECUDA, "cuTensorMapEncodeTiled failed for the slice planes");
  ctx->nw.q = q;
  ctx->nw.qe = qe;
  ctx->nw.qcap = cap;
  return SHAMPOO_OK;
}

// A stream-ordered memory pool per device for shampoo_batched_inverse_root:
// it keeps the memory its allocations return (release threshold: unlimited),
// so a call after the first one allocates and frees its work space without
// going back to the driver.
cudaError_t batched_pool(cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if ((e = cudaMemPoolCreate(&p, &props)) != cudaSuccess) return e;
    uint64_t keep = UINT64_MAX;
    if ((e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) return e;
    pools[dev] = p;
  }
  *out = pools[dev];
  return cudaSuccess;
}

// The pinned counters and the two events a batched root call polls with, per
// host thread and device, made on the thread's first call there and kept:
// pinning host memory and freeing it (which synchronises the device) on
// every call cost more than the call's own host work.  Each call checks that
// they still belong to a live context (a device reset frees both) and makes
// them again if not.
cudaError_t batched_host_state(int** h_count, cudaEvent_t* ev) {
  struct State {
    int* h = nullptr;
    cudaEvent_t ev[2] = {nullptr, nullptr};
  };
  thread_local State st[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  State& x = st[dev];
  if (x.h) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, x.h) != cudaSuccess || at.type != cudaMemoryTypeHost) {
      cudaGetLastError();   // clear the lookup's error
      x.h = nullptr;        // released with its context
    }
  }
  for (auto& v : x.ev) {
    if (!v) continue;
    const cudaError_t q = cudaEventQuery(v);
    if (q != cudaSuccess && q != cudaErrorNotReady) {
      cudaGetLastError();
      v = nullptr;          // destroyed with its context
    }
  }
  if (!x.h && (e = cudaMallocHost(&x.h, 3 * sizeof(int))) != cudaSuccess) return e;
  for (auto& v : x.ev)
    if (!v && (e = cudaEventCreateWithFlags(&v, cudaEventDisableTiming)) != cudaSuccess) return e;
  x.h[0] = x.h[1] = x.h[2] = 0;
  *h_count = x.h;
  ev[0] = x.ev[0];
  ev[1] = x.ev[1];
  return cudaSuccess;
}

// ---------------- asynchronous root pipeline ----------------

// One root job, on the root thread: Newton on the statistics copy into the
// second set of roots, then its bf16 planes.  Errors land in `ctx`, a scratch
// context that carries only the error text (the owner's text belongs to the
// caller's thread).
shampoo_status run_root_job(shampoo_ctx* o, shampoo_ctx* ctx, double tol, int max_iters, bool use_oz,
                            int* nf, int* mi, std::vector<int32_t>* iters) {
  const int64_t slot = (int64_t)o->S * o->S;
  cudaStream_t st = o->side;
  CK(cudaStreamWaitEvent(st, o->ev_submit, 0));
  // a matrix that does not converge keeps the root in use
  CK(cudaMemcpyAsync(o->roots_back, o->roots, (size_t)o->nmat * slot * sizeof(float),
                     cudaMemcpyDeviceToDevice, st));
  shampoo_status r = run_newton(ctx, &o->prof, o->run_mats, o->d_mats, o->d_retry, o->stats_snap, slot, o->S, 1,
                                o->roots_back, slot, o->S, o->S, o->eps, tol, max_iters,
                                o->newton_chunk, o->nw, o->has_root, nullptr, o->h_count, o->ev, st, nf,
                                mi, iters, use_oz ? &o->oz : nullptr, o->d_err);
  if (r != SHAMPOO_OK) {
    cudaStreamSynchronize(st);
    return r;
  }
  cudaError_t e = cudaSuccess;
  run(&o->prof, "split_roots", st, [&] {
    e = launch_split(o->roots_back, (int64_t)o->nmat * slot, o->rplanes_back, st);
  });
  if (e != cudaSuccess) return cuda_fail(ctx, e, "split_roots");
  CK(cudaStreamSynchronize(st));
  return SHAMPOO_OK;
}

// The root thread: takes queued jobs one at a time until the context goes.
void root_thread(shampoo_ctx* o) {
  cudaSetDevice(o->device);
  std::unique_lock<std::mutex> lock(o->job_mu);
  for (;;) {
    o->cv.wait(lock, [&] { return o->quit || o->job == shampoo_ctx::kQueued; });
    if (o->quit) break;
    o->job = shampoo_ctx::kRunning;
    const double tol = o->job_tol;
    const int max_iters = o->job_max_iters;
    const bool use_oz = o->job_oz;
    lock.unlock();
    shampoo_ctx sink;
    int nf = 0, mi = 0;
    std::vector<int32_t> it;
    shampoo_status r = run_root_job(o, &sink, tol, max_iters, use_oz, &nf, &mi, &it);
    if (r == SHAMPOO_OK && nf) r = SHAMPOO_ENOTCONVERGED;
    lock.lock();
    o->job_status = r;
    o->job_err = r == SHAMPOO_ENOTCONVERGED ? std::to_string(nf) + " roots did not converge" : sink.err;
    o->job_nf = nf;
    o->job_mi = mi;
    o->job_iters.swap(it);
    o->job = shampoo_ctx::kDone;
    o->cv.notify_all();
  }
}

// Swap in the roots of a finished job; with `wait`, first block until the
// job in flight (if any) finishes.
shampoo_status install_roots(shampoo_ctx* ctx, bool wait, int* installed) {
  if (installed) *installed = 0;
  std::unique_lock<std::mutex> lock(ctx->job_mu);
  if (wait)
    ctx->cv.wait(lock, [&] { return ctx->job != shampoo_ctx::kQueued && ctx->job != shampoo_ctx::kRunning; });
  if (wait) {   // a waiting install synchronises anyway: read the error word itself
    const shampoo_status ks = check_kernel_error(ctx);
    if (ks != SHAMPOO_OK) return ks;
  }
  if (ctx->job != shampoo_ctx::kDone) return SHAMPOO_OK;
  ctx->job = shampoo_ctx::kIdle;
  const shampoo_status r = ctx->job_status;
  if (r != SHAMPOO_OK && r != SHAMPOO_ENOTCONVERGED)
    return fail(ctx, r, "asynchronous root job failed: " + ctx->job_err);
  std::swap(ctx->roots, ctx->roots_back);
  std::swap(ctx->rplanes, ctx->rplanes_back);
  if (!ctx->blocks.empty() &&
      !encode_planes(&ctx->maps.rk, ctx->rplanes, ctx->S, 2 * (int64_t)ctx->nmat, 64, 128))
    return fail(ctx, SHAMPOO_ECUDA, "cuTensorMapEncodeTiled failed");
  ctx->roots_done = true;
  ctx->last_not_converged = ctx->job_nf;
  ctx->last_max_iters = ctx->job_mi;
  ctx->root_iters = ctx->job_iters;
  ++ctx->generation;
  if (installed) *installed = 1;
  if (r == SHAMPOO_ENOTCONVERGED) return fail(ctx, r, ctx->job_err);
  return SHAMPOO_OK;
}

bool job_in_flight(shampoo_ctx* ctx) {
  std::lock_guard<std::mutex> lock(ctx->job_mu);
  return ctx->job == shampoo_ctx::kQueued || ctx->job == shampoo_ctx::kRunning;
}

// First asynchronous call: the second set of buffers, the low-priority
// stream and the root thread.
shampoo_status start_pipeline(shampoo_ctx* ctx) {
  const size_t n = (size_t)ctx->nmat * ctx->S * ctx->S;
  cudaError_t e = cudaSuccess;
  float *snap = nullptr, *back = nullptr;
  uint16_t* planes = nullptr;
  if ((e = dalloc(ctx, &snap, n)) != cudaSuccess || (e = dalloc(ctx, &back, n)) != cudaSuccess ||
      (e = dalloc(ctx, &planes, 2 * n)) != cudaSuccess)
    return fail(ctx, SHAMPOO_ENOMEM, std::string("asynchronous root buffers: ") + cudaGetErrorString(e));
  int least = 0, greatest = 0;
  CK(cudaDeviceGetStreamPriorityRange(&least, &greatest));
  CK(cudaStreamCreateWithPriority(&ctx->side, cudaStreamNonBlocking, least));
  CK(cudaEventCreateWithFlags(&ctx->ev_submit, cudaEventDisableTiming));
  ctx->stats_snap = snap;
  ctx->roots_back = back;
  ctx->rplanes_back = planes;
  ctx->worker = std::thread(root_thread, ctx);
  return SHAMPOO_OK;
}

}  // namespace

namespace shampoo {
// The error text shampoo_last_error(NULL) returns, for entry points without a
// context that live in other files.
void set_global_error(const std::string& msg) { g_create_err = msg; }
}  // namespace shampoo

extern "C" {

const char* shampoo_version(void) { return "0.1.0"; }

const char* shampoo_last_error(const shampoo_ctx* ctx) {
  return ctx ? ctx->err.c_str() : g_create_err.c_str();
}

void shampoo_destroy(shampoo_ctx* ctx) {
  if (!ctx) return;
  if (ctx->worker.joinable()) {   // a running root job finishes first; a queued one is dropped
    {
      std::lock_guard<std::mutex> lock(ctx->job_mu);
      ctx->quit = true;
    }
    ctx->cv.notify_all();
    ctx->worker.join();
  }
  if (ctx->side) {
    cudaStreamSynchronize(ctx->side);
    cudaStreamDestroy(ctx->side);
  }
  if (ctx->ev_submit) cudaEventDestroy(ctx->ev_submit);
  if (ctx->aux) {
    cudaStreamSynchronize(ctx->aux);
    cudaStreamDestroy(ctx->aux);
  }
  if (ctx->ev_fork) cudaEventDestroy(ctx->ev_fork);
  if (ctx->ev_mid) cudaEventDestroy(ctx->ev_mid);
  if (ctx->ev_join) cudaEventDestroy(ctx->ev_join);
  cudaStreamSynchronize(ctx->stream);
  for (void* q : ctx->allocs) cudaFree(q);
  if (ctx->h_count) cudaFreeHost(ctx->h_count);
  for (auto& e : ctx->ev)
    if (e) cudaEventDestroy(e);
  delete ctx;
}

shampoo_status shampoo_create(shampoo_ctx** out, int nparams, const int64_t* shapes,
                              const int32_t* ndims, int block_size, float beta2, float epsilon,
                              int p, shampoo_graft graft, float momentum, shampoo_dtype grad_dtype,
                              void* cuda_stream) {
  if (!out) return fail(nullptr, SHAMPOO_EINVAL, "out is NULL");
  *out = nullptr;
  if (nparams < 1 || !shapes) return fail(nullptr, SHAMPOO_EINVAL, "need nparams >= 1 and shapes");
  if (block_size < 64 || block_size > 1024 || block_size % 64)
    return fail(nullptr, SHAMPOO_EINVAL, "block_size must be a multiple of 64 in [64, 1024]");
  if (!(beta2 > 0.f && beta2 <= 1.f)) return fail(nullptr, SHAMPOO_EINVAL, "beta2 must be in (0, 1]");
  if (!(epsilon > 0.f) || !std::isfinite(epsilon)) return fail(nullptr, SHAMPOO_EINVAL, "epsilon must be > 0");
  if (p != 2 && p != 4) return fail(nullptr, SHAMPOO_EINVAL, "p must be 2 or 4");
  if (graft != SHAMPOO_GRAFT_NONE && graft != SHAMPOO_GRAFT_ADAGRAD)
    return fail(nullptr, SHAMPOO_EINVAL, "unknown graft");
  if (!(momentum >= 0.f && momentum < 1.f)) return fail(nullptr, SHAMPOO_EINVAL, "momentum must be in [0, 1)");
  if (grad_dtype != SHAMPOO_F32 && grad_dtype != SHAMPOO_BF16)
    return fail(nullptr, SHAMPOO_EINVAL, "unknown grad dtype");

  shampoo_ctx* ctx = new shampoo_ctx();
  ctx->stream = static_cast<cudaStream_t>(cuda_stream);
  cudaGetDevice(&ctx->device);
  ctx->nparams = nparams;
  ctx->b = ctx->S = block_size;
  ctx->p = p;
  ctx->beta2 = beta2;
  ctx->eps = epsilon;
  ctx->mu = momentum;
  ctx->graft = graft;
  ctx->bf16 = grad_dtype == SHAMPOO_BF16;
  ctx->planes_g = ctx->bf16 ? 1 : 2;
  const int b = block_size;

  for (int i = 0; i < nparams; ++i) {
    const int64_t r = shapes[2 * i], c = shapes[2 * i + 1];
    const int nd = ndims ? ndims[i] : 2;
    if (r < 1 || c < 1 || (nd != 1 && nd != 2) || (nd == 1 && r != 1) || r > (1ll << 31) ||
        c > (1ll << 31)) {
      delete ctx;
      return fail(nullptr, SHAMPOO_EINVAL, "bad shape or ndim for parameter " + std::to_string(i));
    }
    ParamDesc pd;
    pd.numel = r * c;
    pd.offset = ctx->total;
    ctx->total += (pd.numel + 3) & ~int64_t(3);   // 16-byte aligned parameter starts
    ctx->params.push_back(pd);
    ctx->ndim.push_back(nd);
    if (nd == 2) {
      for (int64_t r0 = 0; r0 < r; r0 += b)
        for (int64_t c0 = 0; c0 < c; c0 += b) {
          BlockDesc bd{};
          bd.param = i;
          bd.r0 = r0;
          bd.c0 = c0;
          bd.m = (int)std::min<int64_t>(b, r - r0);
          bd.n = (int)std::min<int64_t>(b, c - c0);
          bd.ld = c;
          ctx->blocks.push_back(bd);
        }
    }
    for (int64_t s0 = 0; s0 < pd.numel; s0 += kChunk) {
      ChunkDesc ch;
      ch.param = i;
      ch.start = s0;
      ch.len = (int)std::min<int64_t>(kChunk, pd.numel - s0);
      ctx->chunks.push_back(ch);
      if (nd == 1) ctx->chunks1d.push_back(ch);
    }
  }
  for (int i = 0; i < nparams; ++i) {
    if (ctx->ndim[i] != 1) continue;
    for (int64_t s0 = 0; s0 < ctx->params[i].numel; s0 += b) {
      SegDesc sd;
      sd.param = i;
      sd.s0 = s0;
      sd.len = (int)std::min<int64_t>(b, ctx->params[i].numel - s0);
      ctx->segs.push_back(sd);
    }
  }
  for (size_t k = 0; k < ctx->blocks.size(); ++k) {
    ctx->mats.push_back({(int)(2 * k), ctx->blocks[k].m, p, 0});
    ctx->mats.push_back({(int)(2 * k + 1), ctx->blocks[k].n, p, 0});
  }
  const int mat0 = 2 * (int)ctx->blocks.size();
  for (size_t k = 0; k < ctx->segs.size(); ++k)
    ctx->mats.push_back({mat0 + (int)k, ctx->segs[k].len, p / 2, 0});
  ctx->nmat = (int)ctx->mats.size();
  ctx->run_mats = ctx->mats;
  ctx->param_side.assign(nparams, 0);

  shampoo_status st;
  if ((st = upload(ctx, &ctx->d_params, ctx->params)) != SHAMPOO_OK ||
      (st = upload(ctx, &ctx->d_blocks, ctx->blocks)) != SHAMPOO_OK ||
      (st = upload(ctx, &ctx->d_segs, ctx->segs)) != SHAMPOO_OK ||
      (st = upload(ctx, &ctx->d_chunks, ctx->chunks)) != SHAMPOO_OK ||
      (st = upload(ctx, &ctx->d_chunks1d, ctx->chunks1d)) != SHAMPOO_OK ||
      (st = upload(ctx, &ctx->d_mats, ctx->run_mats)) != SHAMPOO_OK) {
    g_create_err = ctx->err;
    shampoo_destroy(ctx);
    return st;
  }
  const size_t slot = (size_t)b * b;
  const int64_t nblk64 = (int64_t)ctx->blocks.size();
  // Newton work space: at most ~4 GiB of float64 in flight.
  const size_t per = 7 * slot * sizeof(double);
  ctx->newton_chunk = (int)std::max<size_t>(1, std::min<size_t>(ctx->nmat, (size_t(4) << 30) / per));
  cudaError_t e = cudaSuccess;
  bool okm = (e = dalloc(ctx, &ctx->d_gptr, nparams)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->d_wptr, nparams)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->stats, ctx->nmat * slot)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->roots, ctx->nmat * slot)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->a, (size_t)ctx->total)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->P, (size_t)ctx->total)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->d2, (size_t)nparams)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->p2, (size_t)nparams)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->flags, (size_t)nparams)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->has_root, (size_t)ctx->nmat)) == cudaSuccess &&
             (momentum == 0.f || (e = dalloc(ctx, &ctx->mom, (size_t)ctx->total)) == cudaSuccess) &&
             (e = alloc_newton(ctx, ctx->nw, ctx->newton_chunk, b)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->d_retry, (size_t)ctx->newton_chunk)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->d_err, 1)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->gblk, (size_t)ctx->planes_g * ctx->blocks.size() * slot)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->rplanes, 2 * (size_t)ctx->nmat * slot)) == cudaSuccess &&
             (e = dalloc(ctx, &ctx->yplanes, 2 * ctx->blocks.size() * slot)) == cudaSuccess;
  if (!okm) {
    shampoo_destroy(ctx);
    return fail(nullptr, SHAMPOO_ENOMEM, std::string("device allocation failed: ") + cudaGetErrorString(e));
  }
  e = cudaMallocHost(&ctx->h_count, 3 * sizeof(int));
  if (e == cudaSuccess) ctx->h_count[2] = 0;
  int prio = 0;
  if (e == cudaSuccess) e = cudaStreamGetPriority(ctx->stream, &prio);
  if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&ctx->aux, cudaStreamNonBlocking, prio);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_mid, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_join, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev[0], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev[1], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->stats, 0, ctx->nmat * slot * sizeof(float), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->roots, 0, ctx->nmat * slot * sizeof(float), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->a, 0, ctx->total * sizeof(float), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->P, 0, ctx->total * sizeof(float), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->flags, 0, nparams * sizeof(int), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->has_root, 0, ctx->nmat * sizeof(int), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->d_err, 0, sizeof(int), ctx->stream);
  if (e == cudaSuccess && nblk64)
    e = cudaMemsetAsync(ctx->gblk, 0, ctx->planes_g * nblk64 * slot * 2, ctx->stream);
  if (e == cudaSuccess && nblk64) e = cudaMemsetAsync(ctx->yplanes, 0, 2 * nblk64 * slot * 2, ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->rplanes, 0, 2 * (size_t)ctx->nmat * slot * 2, ctx->stream);
  if (e == cudaSuccess && ctx->mom) e = cudaMemsetAsync(ctx->mom, 0, ctx->total * sizeof(float), ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  if (e != cudaSuccess) {
    shampoo_destroy(ctx);
    return fail(nullptr, SHAMPOO_ECUDA, std::string("state set-up failed: ") + cudaGetErrorString(e));
  }
  if (nblk64 &&
      !(encode_planes(&ctx->maps.gk, ctx->gblk, b, ctx->planes_g * nblk64, 64, 128) &&
        encode_planes(&ctx->maps.gmn, ctx->gblk, b, ctx->planes_g * nblk64, 64, 64) &&
        encode_planes4(&ctx->maps.gk4, ctx->gblk, b, nblk64, ctx->planes_g, 64, 128) &&
        encode_planes4(&ctx->maps.gmn4, ctx->gblk, b, nblk64, ctx->planes_g, 64, 64) &&
        encode_planes(&ctx->maps.rk, ctx->rplanes, b, 2 * (int64_t)ctx->nmat, 64, 128) &&
        encode_planes(&ctx->maps.ymn, ctx->yplanes, b, 2 * nblk64, 64, 64) &&
        encode_planes(&ctx->maps.ck, ctx->stats, b, ctx->nmat, 32, 128, true))) {
    shampoo_destroy(ctx);
    return fail(nullptr, SHAMPOO_ECUDA, "cuTensorMapEncodeTiled failed");
  }
  *out = ctx;
  return SHAMPOO_OK;
}

shampoo_status shampoo_update_stats(shampoo_ctx* ctx, const void* const* grads) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  shampoo_status st = poll_kernel_error(ctx);
  if (st != SHAMPOO_OK) return st;
  st = set_pointers(ctx, grads, nullptr);
  if (st != SHAMPOO_OK) return st;
  cudaStream_t s = ctx->stream, x = ctx->aux;
  const int nch = (int)ctx->chunks.size();
  const int nblk = (int)ctx->blocks.size(), nseg = (int)ctx->segs.size();
  Profiler* pr = &ctx->prof;
  CK(cudaMemsetAsync(ctx->flags, 0, ctx->nparams * sizeof(int), s));
  // Two streams: the gather and the block statistics on `stream`; the 1-D
  // non-finite check, the Adagrad accumulator and the 1-D statistics on the
  // auxiliary stream beside them.  The accumulator waits for the gather,
  // which flags non-finite 2-D gradients.
  CK(cudaEventRecord(ctx->ev_fork, s));
  CK(cudaStreamWaitEvent(x, ctx->ev_fork, 0));
  const int nch1 = (int)ctx->chunks1d.size();
  if (nch1)
    run(pr, "check_finite", x, [&] {
      launch_check_finite(ctx->d_chunks1d, nch1, ctx->d_gptr, ctx->bf16, ctx->flags, x);
    });
  if (nblk) {
    shampoo_status gs = gather(ctx, grads, true);
    if (gs != SHAMPOO_OK) return gs;
  }
  CK(cudaEventRecord(ctx->ev_mid, s));
  CK(cudaStreamWaitEvent(x, ctx->ev_mid, 0));
  if (ctx->graft) {
    CK(cudaMemsetAsync(ctx->d2, 0, ctx->nparams * sizeof(double), x));
    run(pr, "diag_update", x, [&] {
      launch_diag_update(ctx->d_chunks, nch, ctx->d_params, ctx->d_gptr, ctx->bf16, ctx->flags,
                         ctx->beta2, ctx->eps, ctx->a, ctx->d2, x);
    });
  }
  if (nseg)   // the 1-D statistics: slots disjoint from the blocks'
    run(pr, "stats_segments", x, [&] {
      launch_stats_segments(ctx->d_segs, nseg, 2 * nblk, ctx->d_gptr, ctx->bf16, ctx->flags,
                            ctx->beta2, ctx->stats, ctx->S, x);
    });
  CK(cudaEventRecord(ctx->ev_join, x));
  ctx->stats_from.assign(grads, grads + ctx->nparams);
  if (nblk) {
    cudaError_t e = cudaSuccess;
    run(pr, "stats_tc", s, [&] {
      e = launch_stats_tc(ctx->maps, ctx->d_blocks, ctx->flags, nblk, ctx->nmat, ctx->S, ctx->planes_g,
                          ctx->beta2, ctx->stats, ctx->d_err, s, ctx->stall_next_stats);
    });
    ctx->stall_next_stats = 0;
    if (e != cudaSuccess) return cuda_fail(ctx, e, "stats_tc");
  }
  CK(cudaStreamWaitEvent(s, ctx->ev_join, 0));
  CK(cudaGetLastError());
  ctx->stats_done = true;
  return SHAMPOO_OK;
}

shampoo_status shampoo_compute_roots(shampoo_ctx* ctx) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  int nf = 0, mi = 0;
  if (!ctx->stats_done) return fail(ctx, SHAMPOO_ESTATE, "compute_roots before update_stats");
  if (job_in_flight(ctx)) return fail(ctx, SHAMPOO_EBUSY, "an asynchronous root job is in flight");
  {   // statistics left by an aborted GEMM are not rooted: this call synchronises anyway
    const shampoo_status ks = check_kernel_error(ctx);
    if (ks != SHAMPOO_OK) return ks;
  }
  {   // a finished job's roots are older than these: install, then overwrite
    const shampoo_status ir = install_roots(ctx, false, nullptr);
    if (ir != SHAMPOO_OK && ir != SHAMPOO_ENOTCONVERGED) return ir;
  }
  const int64_t slot = (int64_t)ctx->S * ctx->S;
  const bool use_oz = ctx->root_method == SHAMPOO_ROOTS_INT8_EMULATED;
  if (use_oz) {
    const shampoo_status os = ensure_ozaki(ctx);
    if (os != SHAMPOO_OK) return os;
    ctx->nw.qs = ctx->oz_slices;
  }
  shampoo_status st = run_newton(ctx, &ctx->prof, ctx->run_mats, ctx->d_mats, ctx->d_retry, ctx->stats,
                                 slot, ctx->S, 1,
                                 ctx->roots, slot, ctx->S, ctx->S, ctx->eps, ctx->tol,
                                 ctx->max_iters, ctx->newton_chunk, ctx->nw, ctx->has_root, nullptr,
                                 ctx->h_count, ctx->ev, ctx->stream, &nf, &mi, &ctx->root_iters,
                                 use_oz ? &ctx->oz : nullptr, ctx->d_err);
  if (st != SHAMPOO_OK) return st;
  cudaError_t e = cudaSuccess;
  run(&ctx->prof, "split_roots", ctx->stream, [&] {
    e = launch_split(ctx->roots, (int64_t)ctx->nmat * slot, ctx->rplanes, ctx->stream);
  });
  if (e != cudaSuccess) return cuda_fail(ctx, e, "split_roots");
  {   // the emulated products' tensor-core kernels report time-outs here too
    const shampoo_status ks = check_kernel_error(ctx);
    if (ks != SHAMPOO_OK) return ks;
  }
  ctx->roots_done = true;
  ++ctx->generation;
  ctx->last_not_converged = nf;
  ctx->last_max_iters = mi;
  if (nf) return fail(ctx, SHAMPOO_ENOTCONVERGED, std::to_string(nf) + " roots did not converge");
  return SHAMPOO_OK;
}

shampoo_status shampoo_compute_roots_async(shampoo_ctx* ctx) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (!ctx->stats_done) return fail(ctx, SHAMPOO_ESTATE, "compute_roots_async before update_stats");
  {
    const shampoo_status ks = poll_kernel_error(ctx);
    if (ks != SHAMPOO_OK) return ks;
  }
  if (job_in_flight(ctx)) return fail(ctx, SHAMPOO_EBUSY, "the previous asynchronous root job is still running");
  const shampoo_status ir = install_roots(ctx, false, nullptr);
  if (ir != SHAMPOO_OK && ir != SHAMPOO_ENOTCONVERGED) return ir;
  if (!ctx->worker.joinable()) {
    const shampoo_status ps = start_pipeline(ctx);
    if (ps != SHAMPOO_OK) return ps;
  }
  const bool use_oz = ctx->root_method == SHAMPOO_ROOTS_INT8_EMULATED;
  if (use_oz) {
    const shampoo_status os = ensure_ozaki(ctx);
    if (os != SHAMPOO_OK) return os;
    ctx->nw.qs = ctx->oz_slices;
  }
  // the statistics as they stand after every call so far
  const size_t n = (size_t)ctx->nmat * ctx->S * ctx->S;
  CK(cudaMemcpyAsync(ctx->stats_snap, ctx->stats, n * sizeof(float), cudaMemcpyDeviceToDevice, ctx->stream));
  CK(cudaEventRecord(ctx->ev_submit, ctx->stream));
  {
    std::lock_guard<std::mutex> lock(ctx->job_mu);
    ctx->job_tol = ctx->tol;
    ctx->job_max_iters = ctx->max_iters;
    ctx->job_oz = use_oz;
    ctx->job = shampoo_ctx::kQueued;
  }
  ctx->cv.notify_all();
  return SHAMPOO_OK;
}

shampoo_status shampoo_install_roots(shampoo_ctx* ctx, int wait, int* installed) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  return install_roots(ctx, wait != 0, installed);
}

int64_t shampoo_roots_generation(const shampoo_ctx* ctx) { return ctx ? ctx->generation : -1; }

shampoo_status shampoo_apply(shampoo_ctx* ctx, float* const* params, const void* const* grads,
                             float lr) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  {
    const shampoo_status ks = poll_kernel_error(ctx);
    if (ks != SHAMPOO_OK) return ks;
  }
  {
    const shampoo_status ir = install_roots(ctx, false, nullptr);
    if (ir != SHAMPOO_OK && ir != SHAMPOO_ENOTCONVERGED) return ir;
  }
  if (!ctx->roots_done) return fail(ctx, SHAMPOO_ESTATE, "apply before compute_roots");
  if (!params) return fail(ctx, SHAMPOO_EINVAL, "params is NULL");
  shampoo_status st = set_pointers(ctx, grads, params);
  if (st != SHAMPOO_OK) return st;
  cudaStream_t s = ctx->stream;
  const int nch = (int)ctx->chunks.size();
  const int nblk = (int)ctx->blocks.size();
  const int nseg = (int)ctx->segs.size();
  Profiler* pr = &ctx->prof;
  CK(cudaMemsetAsync(ctx->p2, 0, ctx->nparams * sizeof(double), s));
  if (nseg) {   // the 1-D preconditioning beside the block GEMMs (disjoint parameters)
    CK(cudaEventRecord(ctx->ev_fork, s));
    CK(cudaStreamWaitEvent(ctx->aux, ctx->ev_fork, 0));
    run(pr, "precond_seg", ctx->aux, [&] {
      launch_precondition_segments(ctx->d_segs, nseg, 2 * nblk, ctx->d_params, ctx->d_gptr,
                                   ctx->bf16, ctx->flags, ctx->roots, ctx->S, ctx->P, ctx->p2,
                                   ctx->aux);
    });
    CK(cudaEventRecord(ctx->ev_join, ctx->aux));
  }
  bool same = ctx->stats_from.size() == (size_t)ctx->nparams;
  for (int i = 0; same && i < ctx->nparams; ++i) same = ctx->stats_from[i] == grads[i];
  if (ctx->graft && !same) {   // ||D||^2 of these gradients against the current a
    CK(cudaMemsetAsync(ctx->d2, 0, ctx->nparams * sizeof(double), s));
    run(pr, "dnorm", s, [&] {
      launch_dnorm(ctx->d_chunks, nch, ctx->d_params, ctx->d_gptr, ctx->bf16, ctx->flags, ctx->a,
                   ctx->eps, ctx->d2, s);
    });
  }
  if (nblk) {
    shampoo_status gs = gather(ctx, grads, false);
    if (gs != SHAMPOO_OK) return gs;
    cudaError_t e = cudaSuccess;
    const bool pair = ctx->pair_tiles && pair_gemm_supported(ctx->S);
    run(pr, "apply_y_tc", s, [&] {
      e = pair ? launch_apply_y_pair(ctx->maps, ctx->d_blocks, ctx->flags, nblk, ctx->nmat, ctx->S, ctx->planes_g,
                                     ctx->yplanes, ctx->d_err, s, ctx->stall_next_apply)
               : launch_apply_y_tc(ctx->maps, ctx->d_blocks, ctx->flags, nblk, ctx->nmat, ctx->S,
                                   ctx->planes_g, ctx->yplanes, ctx->d_err, s, ctx->stall_next_apply);
    });
    ctx->stall_next_apply = 0;
    if (e != cudaSuccess) return cuda_fail(ctx, e, "apply_y_tc");
    run(pr, "apply_p_tc", s, [&] {
      e = pair ? launch_apply_p_pair(ctx->maps, ctx->d_blocks, ctx->d_params, ctx->flags, nblk, ctx->nmat, ctx->S,
                                     ctx->P, ctx->p2, ctx->d_err, s)
               : launch_apply_p_tc(ctx->maps, ctx->d_blocks, ctx->d_params, ctx->flags, nblk, ctx->nmat,
                                   ctx->S, ctx->P, ctx->p2, ctx->d_err, s);
    });
    if (e != cudaSuccess) return cuda_fail(ctx, e, "apply_p_tc");
  }
  if (nseg) CK(cudaStreamWaitEvent(s, ctx->ev_join, 0));
  run(pr, "update", s, [&] {
    launch_update(ctx->d_chunks, nch, ctx->d_params, ctx->d_wptr, ctx->flags, ctx->P, ctx->d2,
                  ctx->p2, ctx->graft, ctx->mu, lr, ctx->mom, s);
  });
  CK(cudaGetLastError());
  // the error word as it stands after this step, for the next call's poll
  CK(cudaMemcpyAsync(&ctx->h_count[2], ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost, s));
  return SHAMPOO_OK;
}

shampoo_status shampoo_root_status(shampoo_ctx* ctx, int* n_not_converged, int* max_iters) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  shampoo_status ks = check_kernel_error(ctx);
  if (ks != SHAMPOO_OK) return ks;
  if (n_not_converged) *n_not_converged = ctx->last_not_converged;
  if (max_iters) *max_iters = ctx->last_max_iters;
  return SHAMPOO_OK;
}

shampoo_status shampoo_nonfinite_status(shampoo_ctx* ctx, int* n_params_skipped) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (!n_params_skipped) return fail(ctx, SHAMPOO_EINVAL, "n_params_skipped is NULL");
  std::vector<int> f(ctx->nparams);
  CK(cudaMemcpyAsync(f.data(), ctx->flags, ctx->nparams * sizeof(int), cudaMemcpyDeviceToHost,
                     ctx->stream));
  shampoo_status ks = check_kernel_error(ctx);
  if (ks != SHAMPOO_OK) return ks;
  int n = 0;
  for (int v : f) n += v != 0;
  *n_params_skipped = n;
  return SHAMPOO_OK;
}

shampoo_status shampoo_set_root_options(shampoo_ctx* ctx, double tol, int max_iters) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (!(tol > 0.0) || max_iters < 1 || max_iters > 1000)
    return fail(ctx, SHAMPOO_EINVAL, "need tol > 0 and 1 <= max_iters <= 1000");
  ctx->tol = tol;
  ctx->max_iters = max_iters;
  return SHAMPOO_OK;
}

shampoo_status shampoo_set_root_method(shampoo_ctx* ctx, int method, int slices) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (method != SHAMPOO_ROOTS_FP64 && method != SHAMPOO_ROOTS_INT8_EMULATED)
    return fail(ctx, SHAMPOO_EINVAL, "unknown root method");
  if (method == SHAMPOO_ROOTS_INT8_EMULATED && (slices < 4 || slices > kOzMaxSlices))
    return fail(ctx, SHAMPOO_EINVAL, "slices must be in [4, 6]");
  if (job_in_flight(ctx)) return fail(ctx, SHAMPOO_EBUSY, "an asynchronous root job is in flight");
  ctx->root_method = method;
  if (method == SHAMPOO_ROOTS_INT8_EMULATED) ctx->oz_slices = slices;
  return SHAMPOO_OK;
}

shampoo_status shampoo_set_one_sided(shampoo_ctx* ctx, int param, int side) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (param < 0 || param >= ctx->nparams || side < SHAMPOO_SIDES_BOTH || side > SHAMPOO_SIDE_RIGHT)
    return fail(ctx, SHAMPOO_EINVAL, "bad parameter index or side");
  if (ctx->ndim[param] != 2) return fail(ctx, SHAMPOO_EINVAL, "a 1-D parameter has a single factor already");
  if (ctx->p != 4) return fail(ctx, SHAMPOO_EINVAL, "one-sided blocks need p = 4 (the kept factor is rooted at p/2)");
  if (ctx->stats_done) return fail(ctx, SHAMPOO_ESTATE, "set_one_sided after the first update_stats");
  const int S = ctx->S, p = ctx->p;
  ctx->param_side[param] = side;
  std::vector<float> eye;
  for (size_t k = 0; k < ctx->blocks.size(); ++k) {
    BlockDesc& bd = ctx->blocks[k];
    if (bd.param != param) continue;
    bd.side = side;
    ctx->mats[2 * k].p = side == SHAMPOO_SIDE_RIGHT ? 0 : (side == SHAMPOO_SIDE_LEFT ? p / 2 : p);
    ctx->mats[2 * k + 1].p = side == SHAMPOO_SIDE_LEFT ? 0 : (side == SHAMPOO_SIDE_RIGHT ? p / 2 : p);
    // the dropped factor's root is the identity on its valid corner
    for (int h = 0; h < 2; ++h) {
      if (ctx->mats[2 * k + h].p != 0) continue;
      const int n = ctx->mats[2 * k + h].size;
      eye.assign((size_t)S * S, 0.f);
      for (int d = 0; d < n; ++d) eye[(size_t)d * S + d] = 1.f;
      CK(cudaMemcpy(ctx->roots + (size_t)(2 * k + h) * S * S, eye.data(), eye.size() * sizeof(float),
                    cudaMemcpyHostToDevice));
    }
  }
  ctx->run_mats.clear();
  for (const auto& m : ctx->mats)
    if (m.p > 0) ctx->run_mats.push_back(m);
  if (!ctx->blocks.empty())
    CK(cudaMemcpy(ctx->d_blocks, ctx->blocks.data(), ctx->blocks.size() * sizeof(BlockDesc), cudaMemcpyHostToDevice));
  if (!ctx->run_mats.empty())
    CK(cudaMemcpy(ctx->d_mats, ctx->run_mats.data(), ctx->run_mats.size() * sizeof(NewtonMat),
                  cudaMemcpyHostToDevice));
  CK(launch_split(ctx->roots, (int64_t)ctx->nmat * S * S, ctx->rplanes, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  return SHAMPOO_OK;
}

shampoo_status shampoo_set_gemm_tiles(shampoo_ctx* ctx, int pair) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if (pair != 0 && pair != 1) return fail(ctx, SHAMPOO_EINVAL, "pair must be 0 or 1");
  ctx->pair_tiles = pair;
  return SHAMPOO_OK;
}

shampoo_status shampoo_selftest_stall_next_stats(shampoo_ctx* ctx) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  ctx->stall_next_stats = 1;
  return SHAMPOO_OK;
}

shampoo_status shampoo_selftest_stall_next_apply(shampoo_ctx* ctx) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  ctx->stall_next_apply = 1;
  return SHAMPOO_OK;
}

shampoo_status shampoo_selftest_stalled_wait(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* d = nullptr;
  int h = 0;
  cudaError_t e = cudaMalloc(&d, sizeof(int));
  if (e == cudaSuccess) e = cudaMemsetAsync(d, 0, sizeof(int), st);
  if (e == cudaSuccess) e = launch_stalled_wait(d, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, d, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (d) cudaFree(d);
  if (e != cudaSuccess) return fail(nullptr, SHAMPOO_ECUDA, std::string("stalled-wait self-test: ") + cudaGetErrorString(e));
  if (h) return fail(nullptr, SHAMPOO_ECUDA, "a tensor-core kernel timed out waiting on its pipeline");
  return SHAMPOO_OK;
}

int shampoo_num_matrices(const shampoo_ctx* ctx) { return ctx ? ctx->nmat : 0; }

shampoo_status shampoo_matrix_info(const shampoo_ctx* ctx, int index, int* size, int* root_p) {
  if (!ctx || index < 0 || index >= ctx->nmat) return SHAMPOO_EINVAL;
  if (size) *size = ctx->mats[index].size;
  if (root_p) *root_p = ctx->mats[index].p;
  return SHAMPOO_OK;
}

shampoo_status shampoo_read_matrix(shampoo_ctx* ctx, int which, int index, float* dst) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  if ((which != 0 && which != 1) || index < 0 || index >= ctx->nmat || !dst)
    return fail(ctx, SHAMPOO_EINVAL, "bad which / index / dst");
  const size_t slot = (size_t)ctx->S * ctx->S;
  const float* src = (which == 0 ? ctx->stats : ctx->roots) + slot * index;
  std::vector<float> h(slot);
  CK(cudaMemcpyAsync(h.data(), src, slot * sizeof(float), cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  // block statistics keep only their upper 128 x 128 tiles: mirror the rest
  if (which == 0 && index < 2 * (int)ctx->blocks.size()) {
    const int S = ctx->S;
    for (int r = 0; r < S; ++r)
      for (int c = 0; c < S; ++c)
        if ((r >> 7) > (c >> 7)) h[(size_t)r * S + c] = h[(size_t)c * S + r];
  }
  CK(cudaMemcpy(dst, h.data(), slot * sizeof(float), cudaMemcpyDefault));
  return SHAMPOO_OK;
}

shampoo_status shampoo_root_iterations(shampoo_ctx* ctx, int32_t* out) {
  if (!ctx || !out) return fail(ctx, SHAMPOO_EINVAL, "ctx or out is NULL");
  if (ctx->root_iters.empty()) return fail(ctx, SHAMPOO_ESTATE, "no roots computed yet");
  // slots past the last one iterated (dropped one-sided factors) report 0
  std::memset(out, 0, ctx->nmat * sizeof(int32_t));
  std::memcpy(out, ctx->root_iters.data(), std::min<size_t>(ctx->root_iters.size(), ctx->nmat) * sizeof(int32_t));
  return SHAMPOO_OK;
}

shampoo_status shampoo_profile_enable(shampoo_ctx* ctx, int on) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  ctx->prof.reset(on != 0);
  return SHAMPOO_OK;
}

int shampoo_profile_count(const shampoo_ctx* ctx) { return ctx ? ctx->prof.count() : 0; }

shampoo_status shampoo_profile_entry(shampoo_ctx* ctx, int index, char* name, int name_len,
                                     int64_t* launches, double* ms) {
  if (!ctx) return fail(nullptr, SHAMPOO_EINVAL, "ctx is NULL");
  CK(ctx->prof.flush());
  Profiler::Entry e;
  if (!ctx->prof.entry(index, &e)) return fail(ctx, SHAMPOO_EINVAL, "profile index out of range");
  if (name && name_len > 0) {
    std::strncpy(name, e.name.c_str(), name_len - 1);
    name[name_len - 1] = 0;
  }
  if (launches) *launches = e.launches;
  if (ms) *ms = e.ms;
  return SHAMPOO_OK;
}

shampoo_status shampoo_batched_inverse_root(const float* A, float* X, int batch, int n, int p,
                                            float eps, double tol, int max_iters, int32_t* iters,
                                            void* stream) {
  return shampoo_batched_inverse_root_ex(A, X, batch, n, p, eps, tol, max_iters, iters, stream,
                                         SHAMPOO_ROOTS_FP64, 0);
}

shampoo_status shampoo_batched_inverse_root_ex(const float* A, float* X, int batch, int n, int p,
                                               float eps, double tol, int max_iters, int32_t* iters,
                                               void* stream, int method, int slices) {
  if (!A || !X || batch < 1 || n < 1 || n > 1024 || (p != 2 && p != 4) || !(eps > 0.f) ||
      !(tol > 0.0) || max_iters < 1 || max_iters > 1000 ||
      (method != SHAMPOO_ROOTS_FP64 && method != SHAMPOO_ROOTS_INT8_EMULATED) ||
      (method == SHAMPOO_ROOTS_INT8_EMULATED && (slices < 4 || slices > kOzMaxSlices)))
    return fail(nullptr, SHAMPOO_EINVAL, "bad argument to shampoo_batched_inverse_root");
  shampoo_ctx tmp;   // carries the allocations and the error text only
  shampoo_ctx* ctx = &tmp;
  const bool use_oz = method == SHAMPOO_ROOTS_INT8_EMULATED;
  int kerr = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    const cudaError_t pe = batched_pool(&ctx->pool);
    if (pe != cudaSuccess) return fail(nullptr, SHAMPOO_ECUDA, std::string("memory pool: ") + cudaGetErrorString(pe));
    ctx->pool_stream = st;
  }
  const int S = (n + kTile - 1) / kTile * kTile;
  const size_t per = 7 * (size_t)S * S * sizeof(double);
  const int chunk = (int)std::max<size_t>(1, std::min<size_t>(batch, (size_t(2) << 30) / per));
  std::vector<NewtonMat> hm(batch);
  for (int i = 0; i < batch; ++i) hm[i] = {i, n, p, 0};
  NewtonMat* dm = nullptr;
  NewtonMat* dr = nullptr;
  NewtonWork w{};
  shampoo_status res = SHAMPOO_OK;
  int nf = 0, mi = 0;
  cudaError_t e = cudaSuccess;
  if ((res = upload(ctx, &dm, hm)) != SHAMPOO_OK) goto done;
  if ((e = dalloc(ctx, &dr, (size_t)chunk)) != cudaSuccess) {
    res = fail(ctx, SHAMPOO_ENOMEM, std::string("retry list: ") + cudaGetErrorString(e));
    goto done;
  }
  if ((e = alloc_newton(ctx, w, chunk, S)) != cudaSuccess) {
    res = fail(ctx, SHAMPOO_ENOMEM, std::string("work space: ") + cudaGetErrorString(e));
    goto done;
  }
  if ((e = batched_host_state(&ctx->h_count, ctx->ev)) != cudaSuccess ||
      (e = dalloc(ctx, &ctx->d_err, 1)) != cudaSuccess ||
      (e = cudaMemsetAsync(ctx->d_err, 0, sizeof(int), st)) != cudaSuccess) {
    res = cuda_fail(ctx, e, "set-up");
    goto done;
  }
  if (use_oz) {
    ctx->S = S;
    ctx->newton_chunk = chunk;
    if ((res = ensure_ozaki(ctx)) != SHAMPOO_OK) goto done;
    w.q = ctx->nw.q;
    w.qe = ctx->nw.qe;
    w.qcap = ctx->nw.qcap;
    w.qs = slices;
  }
  res = run_newton(ctx, nullptr, hm, dm, dr, A, (int64_t)n * n, n, 0, X, (int64_t)n * n, n, S, eps, tol,
                   max_iters, chunk, w, nullptr, iters, ctx->h_count, ctx->ev, st, &nf, &mi, nullptr,
                   use_oz ? &ctx->oz : nullptr, ctx->d_err);
  if (res == SHAMPOO_OK && use_oz) {
    if ((e = cudaMemcpyAsync(&kerr, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
      res = cuda_fail(ctx, e, "error word");
    else if (kerr)
      res = fail(ctx, SHAMPOO_ECUDA, "a tensor-core kernel timed out waiting on its pipeline");
  }
  if (res == SHAMPOO_OK && nf) res = fail(ctx, SHAMPOO_ENOTCONVERGED, std::to_string(nf) + " roots did not converge");
done:
  for (void* q : ctx->allocs) cudaFreeAsync(q, st);   // back to the pool, in stream order
  ctx->allocs.clear();
  cudaStreamSynchronize(st);
  ctx->h_count = nullptr;   // this thread's, kept for its next call
  ctx->ev[0] = ctx->ev[1] = nullptr;
  if (res != SHAMPOO_OK) g_create_err = ctx->err;
  return res;
}

}  // extern "C"
