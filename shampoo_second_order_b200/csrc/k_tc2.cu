// The apply GEMMs on CTA pairs (tcgen05 cta_group::2), for block sides S that
// are multiples of 256: Y = G R^{-1/p} and P = L^{-1/p} Y.
//
// The single-CTA kernels (k_tc.cu) compute 128 x 128 output tiles: every
// tensor-core instruction then reads its whole A and B slices from one SM's
// shared memory, which holds the MMA to about half its rate at b = 1024.  A
// pair of CTAs on neighbouring SMs computes a 256 x 256 tile instead: each
// CTA loads 128 rows of A and 128 rows (the N/2 half) of B, and one thread of
// the even CTA issues MMAs that read both CTAs' shared memory and leave rows
// 0..127 of D in the even CTA's TMEM and rows 128..255 in the odd CTA's.
// Per output element each SM then reads half the operand bytes, and each
// stage carries twice the MMA work, so the ring hides twice the latency.
//
// Roles (192 threads per CTA):
//   warp 0 lane 0   TMA producer, in both CTAs, into its own ring; a stage's
//                   loads complete on the CTA's own `loaded` barrier
//   warp 1 lane 0   even CTA: MMA issuer.  Odd CTA: relay -- it waits for its
//                   own stage to land and arrives on the even CTA's
//                   `peer_ready` barrier, so each CTA can always tell that
//                   its own loads have landed (the teardown needs that)
//   warps 2-5       epilogue, in both CTAs, on their own 128 rows of D
// The MMA issuer's commits arrive on `empty` and `tfull` of both CTAs; the
// epilogue warps of both CTAs arrive on the even CTA's `tempty`.
//
// (The statistics stay on the single-CTA kernel: their two-level
// accumulation keeps a running sum of 128 columns per thread in registers,
// which 256-column pair tiles cannot hold.  256 x 128 pair tiles, which can,
// measured 7-13% slower than single-CTA 128 x 128 tiles at b = 1024: pairing
// the upper-triangle tiles of a column panel computes 11% extra tiles there,
// more than the pair saves.)  Every wait is bounded; a give-up
// sets the error word and both CTAs' abort flags, each producer lets its own
// loads land, the MMA issuer lets its MMAs land, and the pair meets at a
// cluster barrier before freeing TMEM and returning.
#include "common.cuh"
#include "tc.cuh"

namespace shampoo {

namespace {

constexpr int kTM = 128;                    // rows of A (and of B) per CTA
constexpr int kBKe = 64;                    // K elements per stage
constexpr int kBox = kTM * kBKe * 2;        // 16 KB: one operand plane of one CTA
constexpr int kTP = 256;                    // output tile side of the pair
constexpr int kThreads = 192;

enum : int { kApplyY = 1, kApplyP = 2 };

struct PairArgs {
  const BlockDesc* blocks;
  const ParamDesc* params;
  const int* flags;
  int nblk, nmat, S;
  int planes_g;
  uint16_t* y;
  float* P;
  double* p2;
  int* err;
  int stall;
};

struct PairTile {
  int blk, I, J, K;
  bool skip;
};

// Pair tile t over (block, 256-tile); skipped by every role of both CTAs alike.
__device__ __forceinline__ PairTile decode(int t, int mode, const PairArgs& a) {
  const int T = a.S / kTP;
  PairTile x{};
  x.blk = t / (T * T);
  const int r = t % (T * T);
  x.I = r / T;
  x.J = r % T;
  const BlockDesc bd = a.blocks[x.blk];
  x.skip = x.I * kTP >= bd.m || x.J * kTP >= bd.n || a.flags[bd.param] != 0;
  x.K = (mode == kApplyY) ? bd.n : bd.m;
  return x;
}

__host__ __device__ constexpr int pair_stages(int stage_bytes) {
  return (200 * 1024) / stage_bytes < 2 ? 2 : ((200 * 1024) / stage_bytes > 8 ? 8 : (200 * 1024) / stage_bytes);
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_pair_kernel(const __grid_constant__ CUtensorMap map_gk, const __grid_constant__ CUtensorMap map_rk,
                   const __grid_constant__ CUtensorMap map_ymn, PairArgs args, int ntiles) {
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = args.S;
  const uint32_t rank = tc::cluster_ctarank();     // 0: the even CTA (issues the MMAs)
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const bool g1 = args.planes_g == 1;
  const int nA = (MODE == kApplyP) ? 2 : (g1 ? 1 : 2);
  const int nB = 2;
  int npass;
  uint32_t pas, pbs;
  if (MODE == kApplyY && g1) {
    npass = 2; pas = 0; pbs = (1u << 2);                  // g R_h, g R_l
  } else {
    npass = 3; pas = (1u << 4); pbs = (1u << 2);          // h h, h l, l h
  }
  const int stage_bytes = (nA + nB) * kBox;
  const int ST = pair_stages(stage_bytes);

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* loaded = reinterpret_cast<uint64_t*>(smem + ST * stage_bytes);
  uint64_t* peer_ready = loaded + ST;   // even CTA: the odd CTA's stage has landed
  uint64_t* empty = peer_ready + ST;
  uint64_t* tfull = empty + ST;         // [2]
  uint64_t* tempty = tfull + 2;         // [2] even CTA: 4 epilogue warps x 2 CTAs
  uint64_t* drain = tempty + 2;
  uint64_t* never = drain + 1;          // no thread ever arrives here (the failure-path test)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(&loaded[s], 1);
      tc::mbar_init(&peer_ready[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 8);
    }
    tc::mbar_init(drain, 1);
    tc::mbar_init(never, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(tmem_slot, 512);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  tc::cluster_sync();   // both CTAs' barriers exist before any remote arrive or commit
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t peer_abort = tc::cluster_addr(const_cast<int*>(abort_flag), rank ^ 1u);
  auto give_up = [&]() {
    *abort_flag = 1;
    tc::st_cluster_u32(peer_abort, 1u);
    atomicExch(args.err, tc::kErrTimeout);
  };

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    int g = 0;
    for (int t = pair; t < ntiles && !*abort_flag; t += npairs) {
      const PairTile x = decode(t, MODE, args);
      if (x.skip) continue;
      const int i0 = x.I * kTP + (int)rank * kTM;     // this CTA's A rows
      const int j0 = x.J * kTP + (int)rank * kTM;     // this CTA's half of B
      const int blk = x.blk;
      const CUtensorMap* mA = (MODE == kApplyP) ? &map_rk : &map_gk;
      const CUtensorMap* mB = (MODE == kApplyY) ? &map_rk : &map_ymn;
      const int nk = (x.K + kBKe - 1) / kBKe;
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt, ++g) {
        const int s = g % ST;
        if (g >= ST && !tc::mbar_wait(&empty[s], ((g / ST) - 1) & 1)) {
          give_up();
          ok = false;
          break;
        }
        uint8_t* st = smem + s * stage_bytes;
        tc::mbar_expect_tx(&loaded[s], stage_bytes);
        const int k0 = kt * kBKe;
        for (int pa = 0; pa < nA; ++pa) {
          uint8_t* dst = st + pa * kBox;
          if (MODE == kApplyP)                  // A = L^{-1/p} planes
            tc::tma_load_3d(dst, mA, &loaded[s], k0, i0, pa * args.nmat + 2 * blk);
          else                                  // A = G rows
            tc::tma_load_3d(dst, mA, &loaded[s], k0, i0, pa * args.nblk + blk);
        }
        for (int pb = 0; pb < nB; ++pb) {
          uint8_t* dst = st + (nA + pb) * kBox;
          if (MODE == kApplyY) {                // B(k, j) = R^{-1/p}[j][k] (symmetric)
            tc::tma_load_3d(dst, mB, &loaded[s], k0, j0, pb * args.nmat + 2 * blk + 1);
          } else {                              // B(k, j) = Y[k][j], MN-major
            tc::tma_load_3d(dst, mB, &loaded[s], j0, k0, pb * args.nblk + blk);
            tc::tma_load_3d(dst + kBox / 2, mB, &loaded[s], j0 + 64, k0, pb * args.nblk + blk);
          }
        }
      }
      if (!ok) break;
    }
    // every load this CTA issued lands before the pair retires
    for (int q = g > ST ? g - ST : 0; q < g; ++q) tc::mbar_wait(&loaded[q % ST], (q / ST) & 1);
  } else if (warp == 1 && lane == 0 && rank == 1) {
    // ---------------- relay (odd CTA) ----------------
    const uint32_t ready_base = tc::cluster_addr(peer_ready, 0);
    int g = 0;
    for (int t = pair; t < ntiles && !*abort_flag; t += npairs) {
      const PairTile x = decode(t, MODE, args);
      if (x.skip) continue;
      const int nk = (x.K + kBKe - 1) / kBKe;
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt, ++g) {
        const int s = g % ST;
        if (!tc::mbar_wait(&loaded[s], (g / ST) & 1)) {
          give_up();
          ok = false;
          break;
        }
        tc::mbar_arrive_remote(ready_base + s * (uint32_t)sizeof(uint64_t));
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer (even CTA) ----------------
    // failure-path test: a bounded wait on a phase that nothing completes
    // runs out exactly like a stalled pipeline and takes the abort path
    if (args.stall && !tc::mbar_wait(never, 0)) give_up();
    const uint32_t idesc = tc::idesc_bf16(2 * kTM, kTP, 0, MODE == kApplyP);
    int g = 0, i = 0;
    for (int t = pair; t < ntiles && !*abort_flag; t += npairs) {
      const PairTile x = decode(t, MODE, args);
      if (x.skip) continue;
      const int acc = i & 1;
      if (i >= 2 && !tc::mbar_wait_cluster(&tempty[acc], ((i >> 1) - 1) & 1)) {
        give_up();
        break;
      }
      tc::fence_after_sync();
      const uint32_t dt = tmem + acc * kTP;
      const int nk = (x.K + kBKe - 1) / kBKe;
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt, ++g) {
        const int s = g % ST;
        if (!tc::mbar_wait(&loaded[s], (g / ST) & 1) || !tc::mbar_wait_cluster(&peer_ready[s], (g / ST) & 1)) {
          give_up();
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t st = tc::smem_u32(smem + s * stage_bytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          for (int q = 0; q < npass; ++q) {
            const uint32_t sa = st + ((pas >> (2 * q)) & 3) * kBox;
            const uint32_t sb = st + (nA + ((pbs >> (2 * q)) & 3)) * kBox;
            const uint64_t da = tc::smem_desc(sa + kk * 32, 16, 1024);
            const uint64_t db = (MODE == kApplyP) ? tc::smem_desc(sb + kk * 2048, 8192, 1024)
                                                  : tc::smem_desc(sb + kk * 32, 16, 1024);
            tc::mma_bf16_pair(dt, da, db, idesc, (kt | kk | q) != 0);
          }
        }
        tc::mma_commit_pair(&empty[s], 3);
      }
      if (!ok) break;
      tc::mma_commit_pair(&tfull[acc], 3);
      ++i;
    }
    // every MMA issued has landed before the pair retires
    tc::mma_commit_pair(drain, 1);
    tc::mbar_wait(drain, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs): TMEM -> registers -> global ----------------
    const int q = warp & 3;                      // TMEM lanes 32q .. 32q + 31
    const uint32_t tempty0 = tc::cluster_addr(tempty, 0);
    int i = 0;
    for (int t = pair; t < ntiles; t += npairs) {
      const PairTile x = decode(t, MODE, args);
      if (x.skip) continue;
      const int acc = i & 1;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait_sleepy(&tfull[acc], (i >> 1) & 1) && !*abort_flag);
      if (!ok) {
        if (lane == 0) give_up();
        break;
      }
      tc::fence_after_sync();
      const int blk = x.blk;
      const int i0 = x.I * kTP + (int)rank * kTM;
      const int j0 = x.J * kTP;
      const BlockDesc bd = args.blocks[blk];
      const int r = i0 + q * 32 + lane;          // output row owned by this thread
      const uint32_t trow = tmem + acc * kTP + ((uint32_t)(q * 32) << 16);
      if (MODE == kApplyY) {
        uint16_t* yh = args.y + (size_t)blk * S * S;
        uint16_t* yl = args.y + (size_t)(args.nblk + blk) * S * S;
        for (int c = 0; c < 8; ++c) {
          float v[32];
          tc::tmem_ld32(trow + c * 32, v);
          const int cb = j0 + c * 32;
          if (r < S && cb < S) {
            uint32_t hw[16], lw[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const uint16_t h0 = tc::bf16_bits_rn(v[2 * u]), h1 = tc::bf16_bits_rn(v[2 * u + 1]);
              const uint16_t l0 = tc::bf16_bits_rn(v[2 * u] - tc::bf16_to_f(h0));
              const uint16_t l1 = tc::bf16_bits_rn(v[2 * u + 1] - tc::bf16_to_f(h1));
              hw[u] = (uint32_t)h0 | ((uint32_t)h1 << 16);
              lw[u] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            uint4* dh = reinterpret_cast<uint4*>(yh + (size_t)r * S + cb);
            uint4* dl = reinterpret_cast<uint4*>(yl + (size_t)r * S + cb);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              dh[u] = make_uint4(hw[4 * u], hw[4 * u + 1], hw[4 * u + 2], hw[4 * u + 3]);
              dl[u] = make_uint4(lw[4 * u], lw[4 * u + 1], lw[4 * u + 2], lw[4 * u + 3]);
            }
          }
        }
      } else {
        double ss = 0.0;
        float* Pp = args.P + args.params[bd.param].offset;
        for (int c = 0; c < 8; ++c) {
          float v[32];
          tc::tmem_ld32(trow + c * 32, v);
          const int cb = j0 + c * 32;
          if (r < bd.m) {
            float* dst = Pp + (bd.r0 + r) * bd.ld + bd.c0 + cb;
            if (cb + 32 <= bd.n && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
              for (int u = 0; u < 8; ++u)
                reinterpret_cast<float4*>(dst)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
#pragma unroll
              for (int e = 0; e < 32; ++e) ss += (double)v[e] * v[e];
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (cb + e < bd.n) {
                  dst[e] = v[e];
                  ss += (double)v[e] * v[e];
                }
              }
            }
          }
        }
        ss = warp_sum(ss);
        if (lane == 0 && ss != 0.0) atomicAdd(&args.p2[bd.param], ss);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_remote_tmem(tempty0 + acc * (uint32_t)sizeof(uint64_t));
      ++i;
    }
  }
  __syncwarp();
  tc::fence_before_sync();
  tc::cluster_sync();   // no MMA, load or remote arrive of either CTA is left in flight
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc_pair(tmem, 512);
}

int sm_count_pair() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int MODE>
cudaError_t launch_pair(int ntiles, int stage_bytes, const TcMaps& maps, const PairArgs& a, cudaStream_t s) {
  static bool configured = false;   // per process; the attribute is per function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(tc_pair_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const size_t smem = (size_t)pair_stages(stage_bytes) * stage_bytes + 1024 + 256;
  const int npairs = ntiles < sm_count_pair() / 2 ? ntiles : sm_count_pair() / 2;
  tc_pair_kernel<MODE><<<2 * npairs, kThreads, smem, s>>>(maps.gk, maps.rk, maps.ymn, a, ntiles);
  return cudaGetLastError();
}

}  // namespace

bool pair_gemm_supported(int S) { return S >= 256 && S % 256 == 0; }

cudaError_t launch_apply_y_pair(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk, int nmat,
                                int S, int planes_g, uint16_t* y, int* err, cudaStream_t s, int stall) {
  if (nblk <= 0) return cudaSuccess;
  PairArgs a{};
  a.blocks = blocks; a.flags = flags; a.nblk = nblk; a.nmat = nmat; a.S = S;
  a.planes_g = planes_g; a.y = y; a.err = err; a.stall = stall;
  const int T = S / kTP;
  return launch_pair<kApplyY>(nblk * T * T, ((planes_g == 1 ? 1 : 2) + 2) * kBox, maps, a, s);
}

cudaError_t launch_apply_p_pair(const TcMaps& maps, const BlockDesc* blocks, const ParamDesc* params,
                                const int* flags, int nblk, int nmat, int S, float* P, double* p2, int* err,
                                cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  PairArgs a{};
  a.blocks = blocks; a.params = params; a.flags = flags; a.nblk = nblk; a.nmat = nmat; a.S = S;
  a.planes_g = 2; a.P = P; a.p2 = p2; a.err = err;
  const int T = S / kTP;
  return launch_pair<kApplyP>(nblk * T * T, 4 * kBox, maps, a, s);
}

}  // namespace shampoo
