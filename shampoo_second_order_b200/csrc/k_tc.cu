// Tensor-core (tcgen05) kernels of the step:
//   gather   K1: partition each 2-D gradient into zero-padded S x S blocks as
//                bf16 planes (fp32 gradients: h = bf16(g), m = bf16(g - h))
//   stats    K2: L <- beta2 L + G G^T, R <- beta2 R + G^T G (transcript
//                segment 10, first piece), upper-triangular 128 x 128 tiles
//   apply    K4: Y = G R^{-1/p}, then P = L^{-1/p} Y (segment 10, third piece)
//   split        roots (fp32) -> bf16 hi/lo planes for the apply GEMMs
//
// Every product runs as bf16 x bf16 -> fp32 on tcgen05 with the accumulator
// in TMEM; fp32 operands enter as sums of bf16 terms.  bf16 gradients are
// exact in one term.  fp32 gradients are split into two terms x = h + m
// (h = bf16(x), m = bf16(x - h): x to 16 significant bits, rounded to
// nearest) and the statistics keep all four products h h, h m, m h, m m, so
// they are (h + m)(h + m)^T exactly up to accumulation.  What is left out,
// h r^T + r h^T with r = x - h - m, is 2^-16 of the statistic and has no
// sign bias (r is a round-to-nearest remainder); a positive semi-definite
// term left out (m m^T in the three-product scheme h h + h m + m h) would
// bias the small eigenvalues down, and an ill-conditioned block's root
// amplifies that bias by its condition number.  The apply products keep
// h*h + h*l + l*h of two-term splits (relative error near 2^-16), well inside
// the step tolerance.
//
// The GEMM kernel is persistent and warp-specialised: one CTA per SM walks
// the 128 x 128 output tiles round-robin with 192 threads.  Lane 0 of warp 0
// issues TMA loads into a ring of shared-memory stages, lane 0 of warp 1
// issues the MMAs into a rotation of TMEM accumulators (two for the apply
// GEMMs, four K chunks for the statistics) and releases stages with
// tcgen05.commit, and warps 2-5 drain the finished accumulators (warp w owns
// TMEM lanes 32 (w % 4) ..), so the epilogue of one tile overlaps the main
// loop of the next.
#include "common.cuh"
#include "tc.cuh"

namespace shampoo {

namespace {

constexpr int kTM = 128;          // output tile side (M = N = 128)
constexpr int kBKe = 64;          // K elements per stage (one 128-byte row)
constexpr int kBoxBytes = kTM * kBKe * 2;   // 16 KB: one operand plane per stage
#ifndef SHAMPOO_STATS_CHUNK_STAGES
#define SHAMPOO_STATS_CHUNK_STAGES 1
#endif
constexpr int kChunkStages = SHAMPOO_STATS_CHUNK_STAGES;   // statistics: K stages per accumulation chunk
// TMEM accumulators of the statistics GEMM (4 x 128 columns): the MMA issuer
// may run three K chunks ahead of the epilogue, which stops draining TMEM
// while it read-modify-writes a finished tile
constexpr int kStatsAcc = 4;

enum : int { kStats = 0, kApplyY = 1, kApplyP = 2 };

struct TcArgs {
  const BlockDesc* blocks;
  const ParamDesc* params;
  const int* flags;
  int nblk, nmat, S;
  int planes_g;      // 1: bf16 gradients, 2: fp32 gradients (h, m)
  float beta2;
  float* stats;      // fp32 [nmat][S][S], upper 128-tiles kept
  uint16_t* y;       // bf16 planes [2][nblk][S][S], row-major Y
  float* P;          // parameter-shaped preconditioned gradient
  double* p2;        // [nparams] sum of P^2
  int* err;
  int stall;         // failure-path test: the MMA issuer first waits on a phase nothing completes
};

__device__ __forceinline__ void tri_tile128(int idx, int T, int& ti, int& tj) {
  ti = 0;
  while (idx >= T - ti) {
    idx -= T - ti;
    ++ti;
  }
  tj = ti + idx;
}

struct TileInfo {
  int blk, isR, i0, j0, K;
  bool skip;
};

// Tile t of the launch: stats tiles run over (block, L/R, upper-triangle
// tile), apply tiles over (block, tile); tiles outside a ragged block's valid
// range, or of a parameter flagged non-finite, are skipped by every role.
template <int MODE>
__device__ __forceinline__ TileInfo decode_tile(int t, const TcArgs& a) {
  const int T = (a.S + kTM - 1) / kTM;
  TileInfo x{};
  int ti, tj;
  if (MODE == kStats) {
    const int ntri = T * (T + 1) / 2;
    x.blk = t / (2 * ntri);
    const int r = t % (2 * ntri);
    x.isR = r / ntri;
    tri_tile128(r % ntri, T, ti, tj);
  } else {
    x.blk = t / (T * T);
    const int r = t % (T * T);
    ti = r / T;
    tj = r % T;
  }
  const BlockDesc bd = a.blocks[x.blk];
  x.i0 = ti * kTM;
  x.j0 = tj * kTM;
  if (MODE == kStats) {
    const int side = x.isR ? bd.n : bd.m;
    x.skip = x.i0 >= side || x.j0 >= side;
    x.K = x.isR ? bd.m : bd.n;
  } else {
    x.skip = x.i0 >= bd.m || x.j0 >= bd.n;
    x.K = (MODE == kApplyY) ? bd.n : bd.m;
  }
  // a one-sided block never accumulates its dropped factor
  if (MODE == kStats) x.skip = x.skip || (bd.side == 1 && x.isR) || (bd.side == 2 && !x.isR);
  x.skip = x.skip || a.flags[bd.param] != 0;
  return x;
}

constexpr int kCTileBytes = 128 * 128 * 4;   // one fp32 statistics tile (4 boxes of 32 columns)

// The statistics tile goes through shared memory (TMA load, update, TMA
// store) where the ring leaves room for it: bf16 gradients (one plane per
// operand) and S <= 128 (the stages hold the A planes only).  Elsewhere the
// epilogue threads update it in place, one row each.
__host__ __device__ constexpr bool stats_cstage(int planes_g, int S) {
  return planes_g == 1 || S <= kTM;
}

// Ring stages that fit beside the 64 KB statistics tile when the update
// stages it in shared memory (cstage), else beside nothing.
__host__ __device__ constexpr int ring_stages(int stage_bytes, bool cstage = false) {
  const int budget = (cstage ? 224 * 1024 : 192 * 1024) - (cstage ? kCTileBytes : 0);
  return budget / stage_bytes < 2 ? 2 : (budget / stage_bytes > 8 ? 8 : budget / stage_bytes);
}

template <int MODE>
__global__ void __launch_bounds__(192, 1) tc_gemm_kernel(const __grid_constant__ CUtensorMap map_gk,
                                                         const __grid_constant__ CUtensorMap map_gmn,
                                                         const __grid_constant__ CUtensorMap map_rk,
                                                         const __grid_constant__ CUtensorMap map_ymn,
                                                         const __grid_constant__ CUtensorMap map_ck,
                                                         TcArgs args, int ntiles) {
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = args.S;
  constexpr int kNAcc = (MODE == kStats) ? kStatsAcc : 2;   // TMEM accumulators
  constexpr uint32_t kTmemCols = kNAcc * kTM <= 256 ? 256 : 512;
  constexpr int kEpiT = 128;   // epilogue threads (warps 2-5)

  // operand planes loaded and the (A plane, B plane) products kept, packed
  // two bits per product
  const bool g1 = args.planes_g == 1;
  const int nA = (MODE == kApplyP) ? 2 : (MODE == kApplyY ? (g1 ? 1 : 2) : args.planes_g);
  const int nB = (MODE == kStats) ? args.planes_g : 2;
  int npass;
  uint32_t pas, pbs;
  if (MODE == kStats && g1) {
    npass = 1; pas = 0; pbs = 0;                          // g g
  } else if (MODE == kStats) {
    npass = 4; pas = 0; pbs = 0;                          // hm mh mm hh, issued explicitly
  } else if (MODE == kApplyY && g1) {
    npass = 2; pas = 0; pbs = (1u << 2);                  // g R_h, g R_l
  } else {
    npass = 3; pas = (1u << 4); pbs = (1u << 2);          // h h, h l, l h
  }
  // at S <= 128 every statistics tile is diagonal (its B operand is the A
  // panel), so a stage holds the A planes only and twice as many fit
  const int stage_bytes = (MODE == kStats && S <= kTM ? nA : nA + nB) * kBoxBytes;
  // staged statistics (stats_cstage): the old statistics tile comes in by TMA
  // during the main loop, is updated in shared memory and goes back out by TMA
  const bool cstage = (MODE == kStats) && stats_cstage(args.planes_g, S);
  const int ST = ring_stages(stage_bytes, cstage);

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cbuf = smem + ST * stage_bytes;     // the 64 KB statistics tile
  uint64_t* full = reinterpret_cast<uint64_t*>(cbuf + (cstage ? kCTileBytes : 0));
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;     // [kNAcc] accumulator ready for the epilogue
  uint64_t* tempty = tfull + 4;     // [kNAcc] accumulator drained by the epilogue
  uint64_t* drain = tempty + 4;
  uint64_t* cfull = drain + 1;      // statistics tile loaded
  uint64_t* cready = cfull + 1;     // all epilogue threads wrote the tile
  uint64_t* never = cready + 1;     // no thread ever arrives here (the failure-path test)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kNAcc; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], kEpiT);
    }
    tc::mbar_init(drain, 1);
    tc::mbar_init(cfull, 1);
    tc::mbar_init(cready, kEpiT);
    tc::mbar_init(never, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int g = 0;   // ring position, counted across tiles
    for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
      const TileInfo x = decode_tile<MODE>(t, args);
      if (x.skip) continue;
      const int blk = x.blk, i0 = x.i0, j0 = x.j0, isR = x.isR;
      const CUtensorMap* mA = (MODE == kApplyP) ? &map_rk : (isR ? &map_gmn : &map_gk);
      const CUtensorMap* mB = (MODE == kStats) ? (isR ? &map_gmn : &map_gk)
                                               : (MODE == kApplyY ? &map_rk : &map_ymn);
      const int nk = (x.K + kBKe - 1) / kBKe;
      for (int kt = 0; kt < nk; ++kt, ++g) {
        const int s = g % ST;
        if (g >= ST && !tc::mbar_wait(&empty[s], ((g / ST) - 1) & 1)) {
          *abort_flag = 1;
          atomicExch(args.err, tc::kErrTimeout);
          break;
        }
        uint8_t* st = smem + s * stage_bytes;
        // a diagonal statistics tile multiplies a panel by itself: its B
        // operand is the A panel already in the stage
        const bool diag = (MODE == kStats) && i0 == j0;
        tc::mbar_expect_tx(&full[s], diag ? nA * kBoxBytes : stage_bytes);
        const int k0 = kt * kBKe;
        if (MODE == kStats) {
          // one 4-D box carries both planes of a panel (h and m of fp32
          // gradients): K-major [plane][128 rows][64 K], or MN-major in two
          // 64-wide halves [half][plane][64 K][64]
          if (isR) {
            const int hb = nA * kBoxBytes / 2;
            tc::tma_load_4d(st, mA, &full[s], i0, k0, blk, 0);
            tc::tma_load_4d(st + hb, mA, &full[s], i0 + 64, k0, blk, 0);
            if (!diag) {
              tc::tma_load_4d(st + nA * kBoxBytes, mB, &full[s], j0, k0, blk, 0);
              tc::tma_load_4d(st + nA * kBoxBytes + hb, mB, &full[s], j0 + 64, k0, blk, 0);
            }
          } else {
            tc::tma_load_4d(st, mA, &full[s], k0, i0, blk, 0);
            if (!diag) tc::tma_load_4d(st + nA * kBoxBytes, mB, &full[s], k0, j0, blk, 0);
          }
          continue;
        }
        for (int pa = 0; pa < nA; ++pa) {
          uint8_t* dst = st + pa * kBoxBytes;
          if (MODE == kApplyP) {                // A = L^{-1/p} planes
            tc::tma_load_3d(dst, mA, &full[s], k0, i0, pa * args.nmat + 2 * blk);
          } else {                              // A = G rows
            tc::tma_load_3d(dst, mA, &full[s], k0, i0, pa * args.nblk + blk);
          }
        }
        for (int pb = 0; pb < nB && !diag; ++pb) {
          uint8_t* dst = st + (nA + pb) * kBoxBytes;
          if (MODE == kApplyY) {                // B(k, j) = R^{-1/p}[j][k] (symmetric)
            tc::tma_load_3d(dst, mB, &full[s], k0, j0, pb * args.nmat + 2 * blk + 1);
          } else {                              // B(k, j) = Y[k][j], MN-major
            tc::tma_load_3d(dst, mB, &full[s], j0, k0, pb * args.nblk + blk);
            tc::tma_load_3d(dst + kBoxBytes / 2, mB, &full[s], j0 + 64, k0, pb * args.nblk + blk);
          }
        }
      }
    }
    // Every load issued lands before the CTA retires: after an abort the MMA
    // issuer no longer consumes the ring, so the last use of each stage may
    // still be in flight.  (On the normal path these phases completed long
    // ago and each wait returns at once.)
    for (int q = g > ST ? g - ST : 0; q < g; ++q) tc::mbar_wait(&full[q % ST], (q / ST) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    // failure-path test: a bounded wait on a phase that nothing completes
    // runs out exactly like a stalled pipeline and takes the abort path
    if (args.stall && !tc::mbar_wait(never, 0)) {
      *abort_flag = 1;
      atomicExch(args.err, tc::kErrTimeout);
    }
    int g = 0, i = 0;   // i counts accumulation items: (tile, K chunk)
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok && !*abort_flag; t += gridDim.x) {
      const TileInfo x = decode_tile<MODE>(t, args);
      if (x.skip) continue;
      const int a_mn = (MODE == kStats) ? x.isR : 0;
      const int b_mn = (MODE == kStats) ? x.isR : (MODE == kApplyP);
      const bool diag = (MODE == kStats) && x.i0 == x.j0;   // B operand = the A panel
      const uint32_t idesc = tc::idesc_bf16(kTM, kTM, a_mn, b_mn);
      const int nk = (x.K + kBKe - 1) / kBKe;
      // stages per accumulation chunk (bf16 gradients: one product per stage, twice as deep)
      const int cs = (MODE == kStats) ? (g1 ? 2 : 1) * kChunkStages : nk;
      for (int c0 = 0; c0 < nk && ok; c0 += cs, ++i) {
        const int acc = i % kNAcc;
        if (i >= kNAcc && !tc::mbar_wait(&tempty[acc], ((i / kNAcc) - 1) & 1)) {
          *abort_flag = 1;
          atomicExch(args.err, tc::kErrTimeout);
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t dt = tmem + acc * kTM;
        const int c1 = c0 + cs < nk ? c0 + cs : nk;
        for (int kt = c0; kt < c1; ++kt, ++g) {
          const int s = g % ST;
          if (!tc::mbar_wait(&full[s], (g / ST) & 1)) {
            *abort_flag = 1;
            atomicExch(args.err, tc::kErrTimeout);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t st = tc::smem_u32(smem + s * stage_bytes);
          // statistics: a stage's small split products (hm mh mm) go into
          // the accumulator before its large h h products, while the running
          // sum is still small, so their truncation costs less
          if (MODE == kStats && npass == 4) {
            // fp32 gradients: the stage's 16 MMAs, h m, m h, m m, then h h,
            // from descriptors made once per stage.  Planes: K-major one box
            // apart; MN-major half a box apart, with the second 64-wide half
            // of both planes one box further
            const uint64_t tmpl = a_mn ? tc::smem_desc(0, kBoxBytes, 1024) : tc::smem_desc(0, 16, 1024);
            const uint32_t step = a_mn ? 128u : 2u;   // one 16-deep slice, in 16-byte units
            const uint32_t po = a_mn ? kBoxBytes / 2 : kBoxBytes;
            const uint64_t ah = tmpl + (st >> 4), am = tmpl + ((st + po) >> 4);
            const uint64_t bh = diag ? ah : tmpl + ((st + 2 * kBoxBytes) >> 4);
            const uint64_t bm = diag ? am : tmpl + ((st + 2 * kBoxBytes + po) >> 4);
            const uint32_t first = (kt - c0) != 0;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(dt, ah + step * kk, bm + step * kk, idesc, first | kk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(dt, am + step * kk, bh + step * kk, idesc, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(dt, am + step * kk, bm + step * kk, idesc, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(dt, ah + step * kk, bh + step * kk, idesc, 1u);
            tc::mma_commit(&empty[s]);
            continue;
          }
          for (int qq = 0; qq < npass; ++qq) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int pa = (pas >> (2 * qq)) & 3;
              const int pb = (pbs >> (2 * qq)) & 3;
              const uint32_t sa = st + pa * kBoxBytes;
              const uint32_t sb = st + (diag ? pb : nA + pb) * kBoxBytes;
              const uint64_t da = a_mn ? tc::smem_desc(sa + kk * 2048, 8192, 1024)
                                       : tc::smem_desc(sa + kk * 32, 16, 1024);
              const uint64_t db = b_mn ? tc::smem_desc(sb + kk * 2048, 8192, 1024)
                                       : tc::smem_desc(sb + kk * 32, 16, 1024);
              tc::mma_bf16(dt, da, db, idesc, ((kt - c0) | kk | qq) != 0);
            }
          }
          tc::mma_commit(&empty[s]);
        }
        if (!ok) break;
        tc::mma_commit(&tfull[acc]);
      }
    }
    // every MMA this thread issued has landed before TMEM is released
    tc::mma_commit(drain);
    tc::mbar_wait(drain, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> global ----------------
    const int q = warp & 3;                      // TMEM lanes 32q .. 32q + 31
    int i = 0;         // accumulation items: (tile, K chunk)
    int nt = 0;        // tiles finished (the phase of the statistics-tile barriers)
    int c_loads = 0;   // statistics-tile loads issued (phase of the next one)
    // staged statistics: lane 0 of warp 2 owns the shared statistics tile; it
    // loads the first tile's old statistics now and each next tile's right
    // after storing the previous one, while that tile's main loop runs
    auto load_c = [&](int from) {
      for (int t = from; t < ntiles; t += gridDim.x) {
        const TileInfo y = decode_tile<MODE>(t, args);
        if (y.skip) continue;
        const int nbox = (S - y.j0 + 31) / 32 < 4 ? (S - y.j0 + 31) / 32 : 4;
        tc::mbar_expect_tx(cfull, nbox * (kCTileBytes / 4));
        for (int c = 0; c < nbox; ++c)
          tc::tma_load_3d(cbuf + c * (kCTileBytes / 4), &map_ck, cfull, y.j0 + 32 * c, y.i0,
                          2 * y.blk + y.isR);
        ++c_loads;
        return;
      }
    };
    if (cstage && warp == 2 && lane == 0) load_c(blockIdx.x);
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const TileInfo x = decode_tile<MODE>(t, args);
      if (x.skip) continue;
      const int blk = x.blk, i0 = x.i0, j0 = x.j0;
      const BlockDesc bd = args.blocks[blk];
      const int r = i0 + q * 32 + lane;          // output row owned by this thread
      const int nk = (x.K + kBKe - 1) / kBKe;
      const int cs = (MODE == kStats) ? (g1 ? 2 : 1) * kChunkStages : nk;
      float sum[MODE == kStats ? 128 : 1];       // statistics: this row of the tile over the chunks
      for (int c0 = 0; c0 < nk; c0 += cs, ++i) {
        const int acc = i % kNAcc;
        ok = __all_sync(0xffffffffu, tc::mbar_wait_sleepy(&tfull[acc], (i / kNAcc) & 1) && !*abort_flag);
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            atomicExch(args.err, tc::kErrTimeout);
          }
          break;
        }
        tc::fence_after_sync();
        const uint32_t trow = tmem + acc * kTM + ((uint32_t)(q * 32) << 16);
        if (MODE == kStats) {
          const bool first = c0 == 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tc::tmem_ld32(trow + c * 32, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int k = MODE == kStats ? 32 * c + e : 0;
              sum[k] = (first ? 0.f : sum[k]) + v[e];
            }
          }
        } else if (MODE == kApplyY) {
          uint16_t* yh = args.y + (size_t)blk * S * S;
          uint16_t* yl = args.y + (size_t)(args.nblk + blk) * S * S;
          for (int c = 0; c < 4; ++c) {
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
          for (int c = 0; c < 4; ++c) {
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
        tc::mbar_arrive(&tempty[acc]);
      }
      if (!ok) break;
      if (MODE == kStats && cstage) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(cfull, nt & 1))) {
          if (lane == 0) {
            *abort_flag = 1;
            atomicExch(args.err, tc::kErrTimeout);
          }
          break;
        }
        const int rl = q * 32 + lane;            // tile-local row
        const int nbox = (S - j0 + 31) / 32 < 4 ? (S - j0 + 31) / 32 : 4;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c >= nbox) continue;
          // row rl of box c: 8 chunks of 16 B, chunk j stored at j ^ (rl & 7)
          uint8_t* row = cbuf + c * (kCTileBytes / 4) + rl * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int k = MODE == kStats ? 32 * c + 4 * j : 0;
            float4* p4 = reinterpret_cast<float4*>(row + ((j ^ (rl & 7)) << 4));
            float4 o = *p4;
            o.x = fmaf(args.beta2, o.x, sum[k]);
            o.y = fmaf(args.beta2, o.y, sum[k + (MODE == kStats ? 1 : 0)]);
            o.z = fmaf(args.beta2, o.z, sum[k + (MODE == kStats ? 2 : 0)]);
            o.w = fmaf(args.beta2, o.w, sum[k + (MODE == kStats ? 3 : 0)]);
            *p4 = o;
          }
        }
        tc::fence_proxy_async_smem();            // my writes, before the TMA store reads them
        tc::mbar_arrive(cready);
        if (warp == 2 && lane == 0) {
          if (!tc::mbar_wait(cready, nt & 1)) {
            *abort_flag = 1;
            atomicExch(args.err, tc::kErrTimeout);
          } else {
            for (int c = 0; c < nbox; ++c)
              tc::tma_store_3d(&map_ck, cbuf + c * (kCTileBytes / 4), j0 + 32 * c, i0, 2 * blk + x.isR);
            tc::bulk_commit();
            tc::bulk_wait_read0();                 // the tile buffer is free again
            load_c(t + gridDim.x);
          }
        }
      } else if (MODE == kStats) {
        float* C = args.stats + (size_t)(2 * blk + x.isR) * S * S;
        constexpr int NG = 2;   // column groups of 32 whose old values are loaded together
#pragma unroll
        for (int c0 = 0; c0 < 4; c0 += NG) {
          float4 o[8 * NG];
#pragma unroll
          for (int gq = 0; gq < NG; ++gq) {
            const int cb = j0 + (c0 + gq) * 32;
            if (r < S && cb < S) {
              const float4* row = reinterpret_cast<const float4*>(C + (size_t)r * S + cb);
#pragma unroll
              for (int u = 0; u < 8; ++u) o[8 * gq + u] = row[u];
            }
          }
#pragma unroll
          for (int gq = 0; gq < NG; ++gq) {
            const int cb = j0 + (c0 + gq) * 32;
            if (r < S && cb < S) {
              float4* row = reinterpret_cast<float4*>(C + (size_t)r * S + cb);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int k = MODE == kStats ? 32 * (c0 + gq) + 4 * u : 0;
                float4 v = o[8 * gq + u];
                v.x = fmaf(args.beta2, v.x, sum[k]);
                v.y = fmaf(args.beta2, v.y, sum[k + (MODE == kStats ? 1 : 0)]);
                v.z = fmaf(args.beta2, v.z, sum[k + (MODE == kStats ? 2 : 0)]);
                v.w = fmaf(args.beta2, v.w, sum[k + (MODE == kStats ? 3 : 0)]);
                row[u] = v;
              }
            }
          }
        }
      }
      ++nt;
    }
    // after an abort a statistics-tile load may still be in flight: let it land
    if (cstage && warp == 2 && lane == 0 && c_loads > nt) tc::mbar_wait(cfull, (c_loads - 1) & 1);
  }
  if (cstage && warp == 2 && lane == 0) tc::bulk_wait0();   // statistics stores complete
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// K1: gradients -> blocked, zero-padded bf16 planes.  grid: x = 2048-element
// run of the S x S slot, y = block; each thread handles 8 consecutive columns.
__global__ void __launch_bounds__(256) gather_kernel(const BlockDesc* __restrict__ blocks,
                                                     const void* const* __restrict__ gptr, int bf16,
                                                     int* __restrict__ flags, int S, int nblk,
                                                     uint16_t* __restrict__ out) {
  const BlockDesc bd = blocks[blockIdx.y];
  if (flags[bd.param]) return;
  const int64_t e0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (e0 >= (int64_t)S * S) return;
  const int i = (int)(e0 / S), j = (int)(e0 % S);
  uint32_t hw[4] = {0, 0, 0, 0}, mw[4] = {0, 0, 0, 0};
  const void* g = gptr[bd.param];
  const int64_t base = (bd.r0 + i) * bd.ld + bd.c0;
  int bad = 0;
  if (i < bd.m) {
    if (j + 8 <= bd.n) {   // a whole run of 8: vector loads when aligned
      float x[8];
      if (bf16) {
        const uint16_t* src = reinterpret_cast<const uint16_t*>(g) + base + j;
        uint32_t u[4];
        if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
          u[0] = v.x; u[1] = v.y; u[2] = v.z; u[3] = v.w;
        } else {
          for (int q = 0; q < 4; ++q)
            u[q] = (uint32_t)__ldg(src + 2 * q) | ((uint32_t)__ldg(src + 2 * q + 1) << 16);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          hw[q] = u[q];
          bad |= ((u[q] & 0x7F80u) == 0x7F80u) | ((u[q] & 0x7F800000u) == 0x7F800000u);
        }
      } else {
        const float* src = reinterpret_cast<const float*>(g) + base + j;
        if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(src));
          const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
          x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
          x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) x[q] = __ldg(src + q);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          bad |= !isfinite(x[q]);
          const uint16_t h = tc::bf16_bits_rn(x[q]);
          const uint16_t m = tc::bf16_bits_rn(x[q] - tc::bf16_to_f(h));   // the difference is exact
          hw[q >> 1] |= (uint32_t)h << (16 * (q & 1));
          mw[q >> 1] |= (uint32_t)m << (16 * (q & 1));
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int jj = j + q;
        if (jj < bd.n) {
          uint16_t h, m = 0;
          if (bf16) {
            h = __ldg(reinterpret_cast<const uint16_t*>(g) + base + jj);
            bad |= (h & 0x7F80) == 0x7F80;
          } else {
            const float x = __ldg(reinterpret_cast<const float*>(g) + base + jj);
            bad |= !isfinite(x);
            h = tc::bf16_bits_rn(x);
            m = tc::bf16_bits_rn(x - tc::bf16_to_f(h));   // the difference is exact
          }
          hw[q >> 1] |= (uint32_t)h << (16 * (q & 1));
          mw[q >> 1] |= (uint32_t)m << (16 * (q & 1));
        }
      }
    }
  }
  if (bad) atomicOr(&flags[bd.param], 1);
  const size_t slot = (size_t)S * S;
  *reinterpret_cast<uint4*>(out + blockIdx.y * slot + e0) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  if (!bf16) {
    *reinterpret_cast<uint4*>(out + (nblk + blockIdx.y) * slot + e0) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
  }
}

// roots (fp32, [nmat][S][S]) -> bf16 planes hi [nmat] then lo [nmat]
__global__ void split_kernel(const float* __restrict__ x, int64_t n, uint16_t* __restrict__ out) {
  for (int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; e < n;
       e += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + e);
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint16_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      h[q] = tc::bf16_bits_rn(f[q]);
      l[q] = tc::bf16_bits_rn(f[q] - tc::bf16_to_f(h[q]));
    }
    *reinterpret_cast<uint2*>(out + e) =
        make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16), (uint32_t)h[2] | ((uint32_t)h[3] << 16));
    *reinterpret_cast<uint2*>(out + n + e) =
        make_uint2((uint32_t)l[0] | ((uint32_t)l[1] << 16), (uint32_t)l[2] | ((uint32_t)l[3] << 16));
  }
}

size_t smem_bytes(int nA, int nB, bool cstage = false) {
  const int sb = (nA + nB) * kBoxBytes;
  return (size_t)ring_stages(sb, cstage) * sb + (cstage ? kCTileBytes : 0) + 1024 + 256;
}

int sm_count() {
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
cudaError_t launch_mode(int ntiles, size_t smem, const TcMaps& maps, const TcArgs& a, cudaStream_t s) {
  static bool configured = false;   // per process; the attribute is per function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  // the statistics load both gradient planes of a panel in one 4-D box
  tc_gemm_kernel<MODE><<<grid, 192, smem, s>>>(MODE == kStats ? maps.gk4 : maps.gk,
                                               MODE == kStats ? maps.gmn4 : maps.gmn, maps.rk, maps.ymn,
                                               maps.ck, a, ntiles);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather(const BlockDesc* blocks, int nblk, const void* const* gptr, int bf16,
                          int* flags, int S, uint16_t* out, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  dim3 grid((unsigned)(((int64_t)S * S / 8 + 255) / 256), nblk);
  gather_kernel<<<grid, 256, 0, s>>>(blocks, gptr, bf16, flags, S, nblk, out);
  return cudaGetLastError();
}

// One warp waits, through the pipelines' bounded wait, on a barrier phase
// that nothing completes; the give-up lands in *err like a stalled pipeline's.
__global__ void stalled_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0)) atomicExch(err, tc::kErrTimeout);
}

cudaError_t launch_stalled_wait(int* err, cudaStream_t s) {
  stalled_wait_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

cudaError_t launch_split(const float* x, int64_t n, uint16_t* out, cudaStream_t s) {
  split_kernel<<<1184, 256, 0, s>>>(x, n, out);
  return cudaGetLastError();
}

cudaError_t launch_stats_tc(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk,
                            int nmat, int S, int planes_g, float beta2, float* stats, int* err,
                            cudaStream_t s, int stall) {
  if (nblk <= 0) return cudaSuccess;
  TcArgs a{};
  a.blocks = blocks; a.flags = flags; a.nblk = nblk; a.nmat = nmat; a.S = S;
  a.planes_g = planes_g; a.beta2 = beta2; a.stats = stats; a.err = err; a.stall = stall;
  const int T = (S + kTM - 1) / kTM;
  return launch_mode<kStats>(nblk * 2 * (T * (T + 1) / 2),
                             smem_bytes(planes_g, S <= kTM ? 0 : planes_g, stats_cstage(planes_g, S)),
                             maps, a, s);
}

cudaError_t launch_apply_y_tc(const TcMaps& maps, const BlockDesc* blocks, const int* flags, int nblk,
                              int nmat, int S, int planes_g, uint16_t* y, int* err, cudaStream_t s,
                              int stall) {
  if (nblk <= 0) return cudaSuccess;
  TcArgs a{};
  a.blocks = blocks; a.flags = flags; a.nblk = nblk; a.nmat = nmat; a.S = S;
  a.planes_g = planes_g; a.y = y; a.err = err; a.stall = stall;
  const int T = (S + kTM - 1) / kTM;
  return launch_mode<kApplyY>(nblk * T * T, smem_bytes(planes_g == 1 ? 1 : 2, 2), maps, a, s);
}

cudaError_t launch_apply_p_tc(const TcMaps& maps, const BlockDesc* blocks, const ParamDesc* params,
                              const int* flags, int nblk, int nmat, int S, float* P, double* p2,
                              int* err, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  TcArgs a{};
  a.blocks = blocks; a.params = params; a.flags = flags; a.nblk = nblk; a.nmat = nmat; a.S = S;
  a.planes_g = 2; a.P = P; a.p2 = p2; a.err = err;
  const int T = (S + kTM - 1) / kTM;
  return launch_mode<kApplyP>(nblk * T * T, smem_bytes(2, 2), maps, a, s);
}

}  // namespace shampoo
