// Float64-accurate products of the Newton iteration on the int8 tensor
// cores: the Ozaki scheme (Ozaki, Ogita, Oishi, Rump 2012) in its integer
// form (Ootomo, Ozaki, Yokota 2024), for the coupled Newton iteration of
// k_roots.cu (podcast transcript, segment 12: the roots need double
// precision).  tcgen05 has no float64 kind; its int8 kind multiplies exactly.
//
// Each row r of an iterate Z is written as
//   Z[r][:] ~ 2^{e_r} sum_{k=1..qs} q_k[r][:] 2^{-7k},   q_k in [-127, 127],
// the qs 7-bit digits of the fixed-point value |Z[r][:]| 2^{-e_r}, truncated
// toward zero and signed like Z, with e_r the smallest exponent such that
// max|Z[r][:]| < 2^{e_r}.  A product C = A B of two such iterates (B is
// symmetric: every iterate is a polynomial in the statistic, so B's columns
// are its rows) becomes
//   C[i][j] ~ 2^{e_i + f_j} sum_{a + b <= qs + 1} 2^{-7(a+b)} (q^A_a (q^B_b)^T)[i][j],
// where each q_a q_b^T is an exact int8 x int8 -> int32 product on the
// tensor cores (|entry| <= S 127^2 < 2^24 for S <= 1024).  Pairs with the
// same a + b share one int32 accumulator (at most qs pairs, still exact), so
// a tile keeps qs accumulators in TMEM and turns them into float64 once.
// Truncating each value and dropping the pairs with a + b > qs + 1 leaves an
// error of order S 2^{-7 qs} 2^{e_i + f_j} per entry: 2^-42 S relative to the
// row and column scales for the default qs = 6, against 2^-53 per rounding
// of a float64 product.
//
// Kernels:
//   ozaki_split  per row: exponent and qs int8 slice planes of a float64 iterate
//                (T's slices come from M, T = ((p+1) I - s M) / p, in the same pass)
//   ozaki_gemm   persistent, warp-specialised: lane 0 of warp 0 loads the
//                slice planes by TMA (a stage = one slice of A's 128-row
//                tile and of B's 64-row tile over 64 K), lane 0 of warp 1
//                issues the int8 MMAs of every pair as soon as its slices
//                are in, warps 2-5 combine the accumulators in float64, scale
//                them and run the step's epilogue.
// Output tiles are 128 x 64 over the upper triangle; every entry with
// r <= c is written by its tile and mirrored to (c, r), as in k_roots.cu.
#include <float.h>

#include "common.cuh"
#include "tc.cuh"

namespace shampoo {

namespace {

enum : int { kRunning = 0, kFinal = 4 };    // NewtonWork.state values read here
constexpr int kBadExp = 1 << 20;             // exponent of a row holding NaN or Inf
// A stage holds one slice of the 128-row A tile and of the 64-row B tile
// over 64 K (64-byte swizzled rows): 12 KB.  A K chunk needs its QS stages
// at once (slice 0 pairs with every other), so 18 stages keep two chunks of
// look-ahead in flight.
constexpr int kTileM = 128, kTileN = 64, kKBytes = 64;
constexpr int kABytes = kTileM * kKBytes;    // 8 KB
constexpr int kBBytes = kTileN * kKBytes;    // 4 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kStages = 18;
constexpr int kSlots = 8;                    // TMEM accumulator slots of 64 columns (all 512)
constexpr uint32_t kIdesc = tc::idesc_s8(kTileM, kTileN);

// ---------------------------------------------------------------------------
// split
// ---------------------------------------------------------------------------
struct SplitJobs {
  const double* src[2];   // float64 [qcap][S][S]
  int set[2];
  int with_t[2];          // 1: src is M; also slice T = ((p+1) I - s_it M) / p into set kOzT
  int it;                 // schedule index of that T
};

// Exponent and slices of one row held as 4 NCH values per lane (columns
// 128 i + 4 lane .. + 3); `val` maps a stored value to the one to slice.
template <int NCH, class F>
__device__ __forceinline__ void slice_row(const double (&v)[4 * NCH], int S, int c0, int lane, int qs,
                                          int8_t* q0, size_t plane, int* exp_out, F val) {
  double mx = 0.0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NCH; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 128 * i + 4 * lane + j;
      if (c < S) {
        const double x = val(v[4 * i + j], c);
        bad |= !(fabs(x) <= DBL_MAX);
        mx = fmax(mx, fabs(x));
      }
    }
  mx = warp_max(mx);
  bad = __any_sync(0xffffffffu, bad);
  int e = 0;
  if (!bad && mx > 0.0) frexp(mx, &e);        // mx = f 2^e, f in [0.5, 1): every |x| < 2^e
  // a row far below the float64 range of its neighbours counts as zero
  const bool zero = bad || mx == 0.0 || e < -900;
  const double scale = zero ? 0.0 : ldexp(1.0, 7 * qs - e);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 128 * i + 4 * lane;
    if (c >= S) continue;
    unsigned long long f[4];
    bool neg[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double x = val(v[4 * i + j], c + j);
      f[j] = (unsigned long long)(fabs(x) * scale);   // < 2^{7 qs}: exact scaling, truncated
      neg[j] = x < 0.0;
    }
    for (int k = 0; k < qs; ++k) {
      const int sh = 7 * (qs - 1 - k);
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int d = (int)((f[j] >> sh) & 127ull);
        if (neg[j]) d = -d;
        word |= (uint32_t)(uint8_t)(int8_t)d << (8 * j);
      }
      *reinterpret_cast<uint32_t*>(q0 + k * plane + c) = word;
    }
  }
  if (lane == 0) *exp_out = bad ? kBadExp : (zero ? 0 : e);
}

// grid: x = group of 8 rows, y = matrix, z = job.  One warp per row, S <= 128 NCH.
template <int NCH>
__global__ void __launch_bounds__(256, NCH <= 4 ? 3 : 1) ozaki_split_kernel(const NewtonMat* __restrict__ mats, int S,
                                                          SplitJobs jobs, NewtonWork w) {
  const int m = blockIdx.y;
  if (w.state[m] != kRunning) return;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= S) return;
  const int z = blockIdx.z, set = jobs.set[z];
  const double* row = jobs.src[z] + (size_t)m * S * S + (size_t)r * S;
  const int qs = w.qs;
  double v[4 * NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = 128 * i + 4 * lane;
    if (c < S) {
      const double2 a = *reinterpret_cast<const double2*>(row + c);
      const double2 b = *reinterpret_cast<const double2*>(row + c + 2);
      v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = b.x; v[4 * i + 3] = b.y;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * i + j] = 0.0;
    }
  }
  const size_t plane = (size_t)w.qcap * S * S;
  int8_t* q0 = w.q + ((size_t)set * qs * w.qcap + m) * S * S + (size_t)r * S;
  slice_row<NCH>(v, S, 0, lane, qs, q0, plane, &w.qe[((size_t)set * w.qcap + m) * S + r],
                 [](double x, int) { return x; });
  if (jobs.with_t[z]) {   // T from M: its digits in set kOzT, without a float64 copy of T
    const int p = mats[m].p;
    const double sn = newton_sched(w, m, jobs.it), pinv = 1.0 / p;
    int8_t* qt = w.q + ((size_t)kOzT * qs * w.qcap + m) * S * S + (size_t)r * S;
    slice_row<NCH>(v, S, 0, lane, qs, qt, plane, &w.qe[((size_t)kOzT * w.qcap + m) * S + r],
                   [&](double x, int c) { return ((p + 1) * (r == c ? 1.0 : 0.0) - sn * x) * pinv; });
  }
}

// ---------------------------------------------------------------------------
// products
// ---------------------------------------------------------------------------
struct OzArgs {
  const NewtonMat* mats;
  NewtonWork w;
  int S, it, step, ntri;
  int* err;
};

// Tile idx of a matrix's upper triangle, row-major: row tile ti covers rows
// 128 ti .., column tile tj columns 64 tj ..; tj runs from 2 ti.
__host__ __device__ inline void oz_tile(int idx, int S, int& ti, int& tj) {
  const int tc = S / kTileN;
  ti = 0;
  while (idx >= tc - 2 * ti) {
    idx -= tc - 2 * ti;
    ++ti;
  }
  tj = 2 * ti + idx;
}

int oz_ntri(int S) {
  const int tc = S / kTileN, tr = (S + kTileM - 1) / kTileM;
  int n = 0;
  for (int ti = 0; ti < tr; ++ti) n += tc - 2 * ti > 0 ? tc - 2 * ti : 0;
  return n;
}

struct OzTile {
  int m, job, i0, j0, setA, setB;
  bool skip;
};

__device__ __forceinline__ OzTile oz_decode(int t, const OzArgs& a) {
  const int njobs = a.step == 0 ? 2 : 1;
  OzTile x{};
  x.m = t / (njobs * a.ntri);
  const int r = t % (njobs * a.ntri);
  x.job = r / a.ntri;
  int ti, tj;
  oz_tile(r % a.ntri, a.S, ti, tj);
  x.i0 = ti * kTileM;
  x.j0 = tj * kTileN;
  const int st = a.w.state[x.m];
  const int p = a.mats[x.m].p;
  if (a.step == 0) {
    x.skip = x.job == 0 ? !(st == kRunning || st == kFinal) : st != kRunning;
    x.setA = x.job == 0 ? kOzX : kOzT;
    x.setB = kOzT;
  } else if (a.step == 1) {
    x.skip = st != kRunning || p != 4;
    x.setA = x.setB = kOzT2;
  } else {
    x.skip = st != kRunning;
    x.setA = p == 4 ? kOzT4 : kOzT2;
    x.setB = kOzM;
  }
  return x;
}

// Power of two 2^e as a float64 (|e| well inside the normal range).
__device__ __forceinline__ double pow2(int e) {
  return __longlong_as_double(static_cast<long long>(1023 + e) << 52);
}

template <int QS>
__global__ void __launch_bounds__(192, 1) ozaki_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                                            const __grid_constant__ CUtensorMap map_b,
                                                            OzArgs args, int ntiles) {
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = args.S, qcap = args.w.qcap;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;    // [2] a tile's accumulators complete
  uint64_t* sfree = tfull + 2;          // [kSlots] TMEM slot read out by the epilogue
  uint64_t* drain = sfree + kSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(&tfull[0], 1);
    tc::mbar_init(&tfull[1], 1);
    for (int s = 0; s < kSlots; ++s) tc::mbar_init(&sfree[s], 128);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nk = (S + kKBytes - 1) / kKBytes;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int s = 0;
    uint32_t ph = 0;      // phase of the ring's current lap
    bool first = true;    // the first lap needs no free stage
    for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
      const OzTile x = oz_decode(t, args);
      if (x.skip) continue;
      bool ok = true;
      for (int kc = 0; kc < nk && ok; ++kc)
        for (int k = 0; k < QS; ++k) {
          if (!first && !tc::mbar_wait(&empty[s], ph ^ 1)) {
            *abort_flag = 1;
            atomicExch(args.err, tc::kErrTimeout);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          tc::mbar_expect_tx(&full[s], kStageBytes);
          tc::tma_load_3d(st, &map_a, &full[s], kc * kKBytes, x.i0, (x.setA * QS + k) * qcap + x.m);
          tc::tma_load_3d(st + kABytes, &map_b, &full[s], kc * kKBytes, x.j0, (x.setB * QS + k) * qcap + x.m);
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
            first = false;
          }
        }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    // Accumulator d of the i-th tile lives in TMEM slot (i QS + d) mod kSlots:
    // the next tile starts in the slots its predecessor left free and waits
    // for each other slot only when it first writes it.
    int s = 0, i = 0;
    uint32_t ph = 0;
    const uint64_t desc0 = tc::smem_desc(0, 16, 512, 4);   // 64-byte swizzle; + (address >> 4)
    const uint32_t ring = tc::smem_u32(smem);
    for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
      const OzTile x = oz_decode(t, args);
      if (x.skip) continue;
      const int g0 = i * QS;
      bool ok = true;
      for (int kc = 0; kc < nk && ok; ++kc) {
        int idx[QS];          // ring stage of each slice of this K chunk
#pragma unroll
        for (int k = 0; k < QS; ++k) {
          if (!tc::mbar_wait(&full[s], ph)) {
            ok = false;
            break;
          }
          idx[k] = s;
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
          }
          if (kc == 0) {   // first writes of accumulators 2k - 1 and 2k: their slots must be read out
#pragma unroll
            for (int d = 2 * k - 1; d <= 2 * k; ++d) {
              if (d < 0 || d >= QS) continue;
              const int gd = g0 + d;
              if (gd >= kSlots && !tc::mbar_wait(&sfree[gd % kSlots], ((gd / kSlots) - 1) & 1)) ok = false;
            }
            if (!ok) break;
          }
          tc::fence_after_sync();
          // every pair (a, b), a + b <= QS - 1 (0-based), whose later slice is
          // k: (k, o) and (o, k).  The pair with o = k or o = k - 1 is the
          // first to reach its accumulator a + b in a tile.
#pragma unroll
          for (int o = 0; o <= k; ++o) {
            if (o + k > QS - 1) continue;
#pragma unroll
            for (int sw = 0; sw < 2; ++sw) {
              if (sw == 1 && o == k) continue;
              const int ia = sw ? o : k, ib = sw ? k : o;
              const uint32_t dt = tmem + ((g0 + ia + ib) % kSlots) * kTileN;
              const uint64_t da = desc0 + ((ring + idx[ia] * kStageBytes) >> 4);
              const uint64_t db = desc0 + ((ring + idx[ib] * kStageBytes + kABytes) >> 4);
              const bool lead = sw == 0 && (o == k || o == k - 1);
#pragma unroll
              for (int kk = 0; kk < kKBytes / 32; ++kk)
                tc::mma_i8(dt, da + 2 * kk, db + 2 * kk, kIdesc, (kc > 0 || kk > 0 || !lead) ? 1u : 0u);
            }
          }
        }
        if (!ok) break;
        // this chunk's stages are free once its MMAs have read them
#pragma unroll
        for (int k = 0; k < QS; ++k) tc::mma_commit(&empty[idx[k]]);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicExch(args.err, tc::kErrTimeout);
        break;
      }
      tc::mma_commit(&tfull[i & 1]);
      ++i;
    }
    tc::mma_commit(drain);
    tc::mbar_wait(drain, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    int i = 0;
    const NewtonWork& w = args.w;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      const OzTile x = oz_decode(t, args);
      if (x.skip) continue;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&tfull[i & 1], (i >> 1) & 1) && !*abort_flag);
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicExch(args.err, tc::kErrTimeout);
        }
        break;
      }
      tc::fence_after_sync();
      const int m = x.m, rl = q * 32 + lane, r = x.i0 + rl;
      const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
      // Accumulator d weighs 2^{-7(d+2)}: the value is 2^{-7(QS+1)} times the
      // exact int64 sum of acc_d 2^{7(QS-1-d)} (below 2^60 for S <= 1024).
      // Each slot is released as soon as it is read.
      long long tot[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) tot[j] = 0;
#pragma unroll
      for (int d = 0; d < QS; ++d) {
        const int slot = (i * QS + d) % kSlots;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          tc::tmem_ld32(trow + slot * kTileN + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) tot[c * 32 + j] += (long long)__float_as_int(v[j]) << (7 * (QS - 1 - d));
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&sfree[slot]);
      }
      ++i;

      const size_t base = (size_t)m * S * S;
      const int ea = r < S ? w.qe[((size_t)x.setA * qcap + m) * S + r] : 0;
      const int* eb = w.qe + ((size_t)x.setB * qcap + m) * S;
      const int p = args.mats[m].p;
      double mul = 1.0;
      double* C;
      if (args.step == 0 && x.job == 0) {            // X_next = s_k^{1/p} X T
        const double sk = newton_sched(w, m, args.it);
        if (sk != 1.0) mul = pow(sk, 1.0 / p);
        C = w.X[(args.it + 1) & 1] + base;
      } else if (args.step == 0) {
        C = w.T2 + base;                             // T2 = T T
      } else if (args.step == 1) {
        C = w.T4 + base;                             // T4 = T2 T2
      } else {
        mul = newton_sched(w, m, args.it);           // M_next = s_k T^p M
        C = w.M[(args.it + 1) & 1] + base;
      }
      const bool resid = args.step == 2;
      const double sn = resid ? newton_sched(w, m, args.it + 1) : 0.0, pinv = 1.0 / p;
      const int n = args.mats[m].size;
      // whole tile strictly above the diagonal: every entry is stored and mirrored
      const bool above = x.j0 >= x.i0 + kTileM;
      double dev = 0.0, f2 = 0.0;
      const double sc = mul * pow2(ea - 7 * (QS + 1));
      // one entry (r, col) of the upper triangle: stored, mirrored and, for
      // step C, folded into the residual and turned into the next T
      auto emit = [&](int col, double v, bool stored) {
        if (r >= S || col >= S || r > col) return;
        if (!stored) {
          C[(size_t)r * S + col] = v;
          if (r < col) C[(size_t)col * S + r] = v;
        }
        if (resid) {
          const double dl = (r == col) ? 1.0 : 0.0;
          if (r < n && col < n) {
            double xd = fabs(v - dl);
            if (!(xd <= DBL_MAX)) xd = INFINITY;
            dev = fmax(dev, xd);
            f2 += (r == col ? 1.0 : 2.0) * xd * xd;   // an entry above the diagonal counts for its mirror too
          }
        }
      };
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const int col = x.j0 + j;
        const int e0 = eb[col], e1 = eb[col + 1];
        const bool bad0 = ea == kBadExp || e0 == kBadExp, bad1 = ea == kBadExp || e1 == kBadExp;
        const double nan = __longlong_as_double(0x7ff8000000000000ll);
        const double v0 = bad0 ? nan : (double)tot[j] * (sc * pow2(e0));
        const double v1 = bad1 ? nan : (double)tot[j + 1] * (sc * pow2(e1));
        if (above && r < S) {
          *reinterpret_cast<double2*>(C + (size_t)r * S + col) = make_double2(v0, v1);
          C[(size_t)col * S + r] = v0;
          C[(size_t)(col + 1) * S + r] = v1;
        }
        emit(col, v0, above);
        emit(col + 1, v1, above);
      }
      if (resid) {
        dev = warp_max(dev);
        f2 = warp_sum(f2);
        if (lane == 0) {
          atomicMax(&w.resid[m], static_cast<unsigned long long>(__double_as_longlong(dev)));
          atomicAdd(&w.fro2[m], f2);
        }
      }
    }
  }
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

int sm_count_oz() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int QS>
cudaError_t launch_gemm(const OzakiMaps& maps, const OzArgs& a, int ntiles, int grid, int smem, cudaStream_t s) {
  static bool configured = false;   // the attribute is per instantiation
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(ozaki_gemm_kernel<QS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  ozaki_gemm_kernel<QS><<<grid, 192, smem, s>>>(maps.a, maps.b, a, ntiles);
  return cudaGetLastError();
}

}  // namespace

template <int NCH>
void launch_split_jobs(const NewtonMat* mats, int nm, int S, const SplitJobs& jobs, int nj, NewtonWork w,
                       cudaStream_t s) {
  ozaki_split_kernel<NCH><<<dim3((S + 7) / 8, nm, nj), 256, 0, s>>>(mats, S, jobs, w);
}

cudaError_t launch_ozaki_split(const NewtonMat* mats, int nm, int S, int it, unsigned sets, NewtonWork w,
                               cudaStream_t s) {
  // the float64 source of each set at step `it` (X and M: the buffers step it
  // wrote); T, when asked together with M, comes from M in the same pass
  const double* src[kOzSets] = {w.X[it & 1], w.T, w.T2, w.T4, w.M[it & 1]};
  const bool t_from_m = (sets >> kOzM & 1u) && (sets >> kOzT & 1u);
  if (t_from_m) sets &= ~(1u << kOzT);
  SplitJobs jobs{};
  jobs.it = it;
  int nj = 0;
  auto flush = [&] {
    if (!nj) return;
    if (S <= 128) launch_split_jobs<1>(mats, nm, S, jobs, nj, w, s);
    else if (S <= 256) launch_split_jobs<2>(mats, nm, S, jobs, nj, w, s);
    else if (S <= 512) launch_split_jobs<4>(mats, nm, S, jobs, nj, w, s);
    else launch_split_jobs<8>(mats, nm, S, jobs, nj, w, s);
    nj = 0;
  };
  for (int z = 0; z < kOzSets; ++z) {
    if (!(sets >> z & 1u)) continue;
    if (nj == 2) flush();
    jobs.src[nj] = src[z];
    jobs.set[nj] = z;
    jobs.with_t[nj] = (z == kOzM && t_from_m) ? 1 : 0;
    ++nj;
  }
  flush();
  return cudaGetLastError();
}

cudaError_t launch_ozaki_step(const OzakiMaps& maps, int step, const NewtonMat* mats, int nm, int S, int it,
                              NewtonWork w, int* err, cudaStream_t s) {
  const int smem = kStages * kStageBytes + 1024 + 512;   // ring, alignment slack, barriers
  OzArgs a{};
  a.mats = mats; a.w = w; a.S = S; a.it = it; a.step = step; a.ntri = oz_ntri(S); a.err = err;
  const int ntiles = nm * (step == 0 ? 2 : 1) * a.ntri;
  const int grid = ntiles < sm_count_oz() ? ntiles : sm_count_oz();
  switch (w.qs) {
    case 4: return launch_gemm<4>(maps, a, ntiles, grid, smem, s);
    case 5: return launch_gemm<5>(maps, a, ntiles, grid, smem, s);
    case 6: return launch_gemm<6>(maps, a, ntiles, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace shampoo
