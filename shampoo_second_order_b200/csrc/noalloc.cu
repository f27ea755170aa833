// shampoo_batched_inverse_root_noalloc: the batched inverse-root computation
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need roots: code
// running under a framework that owns all device memory through its own pool
// (where a raw cudaMalloc would fragment the pool or fail once the pool has
// reserved the GPU), callers inside a region where allocation would
// synchronise the device, and embedded or real-time hosts that forbid
// allocation after start-up.  This entry point runs the same coupled Newton
// kernels as shampoo_batched_inverse_root but keeps its float64 work space in
// one file-scope device array, so a call allocates nothing: no cudaMalloc,
// cudaFree, pinned host memory, events or library allocator.
//
// Limits and sharing rules (stated for the user in include/shampoo.h):
//  * the array is kNoAllocBytes = 64 MiB and lives on every GPU that loads the
//    library, until the process exits;
//  * matrices are processed in chunks that fit the array: 7 n' x n' float64
//    buffers per matrix, n' = n rounded up to 64, so n <= 1024;
//  * every call shares the array; calls that overlap on the GPU (other streams,
//    other host threads) race and must be serialised by the caller;
//  * every call looks up the array's device address on the current device
//    (cudaGetSymbolAddress with that device current) instead of keeping it:
//    after a device reset, or under another driver context, the array can sit
//    at another address, and a kept one would point at freed memory.  The
//    first lookup in a process may load the library's device code.
#include <string>

#include "../../include/shampoo.h"
#include "internal.h"

namespace shampoo {

void set_global_error(const std::string& msg);   // api.cu

namespace {

constexpr size_t kNoAllocBytes = size_t(64) << 20;

// The work space.  In host code this name is only a stand-in for the symbol:
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// The scratch array's device address on the current device, looked up anew
// on every call (a lookup allocates nothing).
cudaError_t scratch_address(void** out) {
  *out = nullptr;
  return cudaGetSymbolAddress(out, g_noalloc_scratch);
}

// Carve the work space for `chunk` matrices of side S out of the array.
struct Carve {
  unsigned char* base;
  size_t used = 0;
  template <class T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + used);
    used += count * sizeof(T);
    return p;
  }
};

size_t carve(unsigned char* base, int chunk, int S, NewtonWork* w, NewtonMat** mats, NewtonMat** retry,
             int** nretry) {
  Carve c{base};
  const size_t mat = (size_t)chunk * S * S;
  w->X[0] = c.take<double>(mat);
  w->X[1] = c.take<double>(mat);
  w->M[0] = c.take<double>(mat);
  w->M[1] = c.take<double>(mat);
  w->T = c.take<double>(mat);
  w->T2 = c.take<double>(mat);
  w->T4 = c.take<double>(mat);
  w->cinv = c.take<double>(chunk);
  w->ridge = c.take<double>(chunk);
  w->sched = c.take<double>((size_t)chunk * kSched);
  w->nsched = c.take<int>(chunk);
  w->resid = c.take<unsigned long long>(chunk);
  w->fro2 = c.take<double>(chunk);
  w->prev = c.take<double>(chunk);
  w->worse = c.take<int>(chunk);
  w->live = c.take<int>(chunk);
  w->iters = c.take<int>(chunk);
  w->state = c.take<int>(chunk);
  w->count = c.take<int>(3);
  *mats = c.take<NewtonMat>(chunk);
  *retry = c.take<NewtonMat>(chunk);
  *nretry = c.take<int>(1);
  return c.used;
}

// mats[i] = matrix c0 + i of the batch.
__global__ void fill_mats_kernel(NewtonMat* mats, int nm, int c0, int n, int p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < nm) mats[i] = NewtonMat{c0 + i, n, p, 0};
}

// Move the matrices whose iteration diverged (state 3) to the front of
// `retry` and count them; one thread keeps the order of the batch.
__global__ void compact_diverged_kernel(const NewtonMat* mats, int nm, NewtonWork w, NewtonMat* retry,
                                        int* nretry) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int k = 0;
  for (int i = 0; i < nm; ++i)
    if (w.state[i] == 3) retry[k++] = mats[i];
  *nretry = k;
}

__global__ void copy_mats_kernel(const NewtonMat* src, NewtonMat* dst, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i];
}

// Add to *failed the matrices that end this pass unconverged: those that hit
// the iteration cap (state 2) and, on the last pass, those that diverged.
__global__ void count_failed_kernel(int nm, NewtonWork w, int final_pass, int* failed) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int k = 0;
  for (int i = 0; i < nm; ++i) k += (w.state[i] == 2) || (final_pass && w.state[i] == 3);
  *failed += k;
}

// A device int read back through pageable host memory: the copy returns once
// it has completed, so no event or pinned buffer is needed.
cudaError_t read_int(const int* d, int* h, cudaStream_t s) {
  return cudaMemcpyAsync(h, d, sizeof(int), cudaMemcpyDeviceToHost, s);
}

shampoo_status fail_na(shampoo_status st, const std::string& msg) {
  set_global_error(msg);
  return st;
}

}  // namespace
}  // namespace shampoo

using namespace shampoo;

extern "C" shampoo_status shampoo_batched_inverse_root_noalloc(const float* A, float* X, int batch,
                                                               int n, int p, float eps, double tol,
                                                               int max_iters, int32_t* iters,
                                                               void* stream) {
  if (!A || !X || batch < 1 || n < 1 || (p != 2 && p != 4) || !(eps > 0.f) || !(tol > 0.0) ||
      max_iters < 1 || max_iters > 1000)
    return fail_na(SHAMPOO_EINVAL, "bad argument to shampoo_batched_inverse_root_noalloc");
  if (n > 1024)
    return fail_na(SHAMPOO_EINVAL,
                   "shampoo_batched_inverse_root_noalloc: n = " + std::to_string(n) +
                       " exceeds the maximum of 1024 that its 64 MiB work space holds");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess)
    return fail_na(SHAMPOO_ECUDA,
                   std::string("cudaGetSymbolAddress of the work space: ") + cudaGetErrorString(e));
  unsigned char* b = static_cast<unsigned char*>(base);
  const int S = (n + kTile - 1) / kTile * kTile;
  // the largest chunk of matrices whose work space fits the array (plus one int)
  NewtonWork w{};
  NewtonMat *mats = nullptr, *retry = nullptr;
  int* nretry = nullptr;
  int chunk = 1;
  while (chunk < batch && carve(b, chunk + 1, S, &w, &mats, &retry, &nretry) + 256 <= kNoAllocBytes)
    ++chunk;
  const size_t used = carve(b, chunk, S, &w, &mats, &retry, &nretry);
  int* failed = reinterpret_cast<int*>(b + ((used + 255) & ~size_t(255)));
  if (used + 512 > kNoAllocBytes)
    return fail_na(SHAMPOO_EINVAL, "shampoo_batched_inverse_root_noalloc: work space too small");
  // the failure counter is the only state that must start at zero
  e = cudaMemsetAsync(failed, 0, sizeof(int), st);

  for (int c0 = 0; c0 < batch && e == cudaSuccess; c0 += chunk) {
    int nm = batch - c0 < chunk ? batch - c0 : chunk;
    fill_mats_kernel<<<(nm + 127) / 128, 128, 0, st>>>(mats, nm, c0, n, p);
    for (int attempt = 0; attempt < kNewtonAttempts && nm > 0 && e == cudaSuccess; ++attempt) {
      launch_newton_reset(nm, w, st);
      launch_newton_bound(A, (int64_t)n * n, n, 0, mats, nm, S, eps, attempt, w, st);
      launch_newton_init(A, (int64_t)n * n, n, 0, mats, nm, S, w, st);
      launch_newton_lanczos(mats, nm, S, w, st);
      launch_newton_t0(mats, nm, S, w, st);
      launch_newton_check(nm, 0, tol, max_iters, w, st);
      int alive = 0;
      e = read_int(&w.count[0], &alive, st);
      for (int it = 0; it < max_iters && alive && e == cudaSuccess; ++it) {
        launch_newton_step_a(mats, alive, S, it, 64, w, st);   // `alive`: the last check's count
        if (p == 4) launch_newton_step_b(mats, alive, S, 64, w, st);
        launch_newton_step_c(mats, alive, S, it, 64, w, st);
        launch_newton_check(nm, it + 1, tol, max_iters, w, st);
        e = read_int(&w.count[(it + 1) & 1], &alive, st);
      }
      if (e != cudaSuccess) break;
      compact_diverged_kernel<<<1, 32, 0, st>>>(mats, nm, w, retry, nretry);
      int nr = 0;
      if ((e = read_int(nretry, &nr, st)) != cudaSuccess) break;
      const int final_pass = (attempt == kNewtonAttempts - 1) || nr == 0;
      launch_newton_finalize(X, (int64_t)n * n, n, mats, nm, S, w, nullptr, iters, final_pass, st);
      count_failed_kernel<<<1, 32, 0, st>>>(nm, w, final_pass, failed);
      if (final_pass) break;
      // the diverged matrices run again with a raised ridge
      copy_mats_kernel<<<(nr + 127) / 128, 128, 0, st>>>(retry, mats, nr);
      nm = nr;
    }
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  int n_failed = 0;
  if (e == cudaSuccess) e = read_int(failed, &n_failed, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess)
    return fail_na(SHAMPOO_ECUDA, std::string("shampoo_batched_inverse_root_noalloc: ") + cudaGetErrorString(e));
  if (n_failed) return fail_na(SHAMPOO_ENOTCONVERGED, std::to_string(n_failed) + " roots did not converge");
  return SHAMPOO_OK;
}
