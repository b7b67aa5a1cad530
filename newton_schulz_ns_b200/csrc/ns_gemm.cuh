// Persistent grouped tensor-core GEMM for the Newton-Schulz iteration (sm_100a).
//
// One launch runs up to MAX_PROBLEMS "problems"; a problem is a batch of
// same-shape slices C[s] = epilogue(opA(A[s]) * opB(B[s])) with
//   opA: M x K, stored K-major ([M][K] row-major) or MN-major ([K][M]);
//   opB: K x N, stored K-major ([N][K], i.e. C = A B^T) or MN-major ([K][N]).
// Output tiles are TILE_M x 256 with 64-wide K blocks.  Two variants share
// the code: CG = 1 runs one CTA per 128 x 256 tile; CG = 2 runs a 2-CTA
// cluster per 256 x 256 tile with the pair MMA (cta_group::2), each CTA
// holding half of A and half of B in its shared memory, which halves the
// operand bytes each SM moves per flop.  Operands are brought into shared
// memory by TMA (128-byte swizzle, zero fill outside the slice), multiplied
// by tcgen05.mma (bf16 or fp16 in, fp32 accumulate in TMEM), and the
// epilogue applies
//   C = f * (alpha * acc + beta * D) + gamma * [row == col]
// where D is an addend with C's shape and f = f0 * s^p per slice, with
// s = 1 / (sqrt(sumsq[slice]) + eps) and p in {0, 1, 2}.
//
// Symmetric problems ("tri") compute only the tiles that touch the lower
// triangle, so A = X X^T and B = b*A + c*A^2 cost about half of a full
// product (the one-triangle products of the Megatron-Core
// layer_sharded_muon docs, use_syrk).  The tiles of each 256 x 256 diagonal
// block are written as computed.  Every tile below them is either written
// twice, as computed and transposed into the upper triangle ("mirror"), or
// once, when every consumer reads the matrix as symmetric: an operand
// flagged a_sym / b_sym takes each 128-wide K stage that lies above the
// 256 x 256 diagonal blocks from the stored lower triangle, transposed
// (S[rows][k] = S[k][rows]: the same tensor map read MN-major), so the
// upper triangle is never written nor read.  (That read uses the pair
// kernel's stage geometry: K stages and row halves of 128.)
//
// The epilogue stages each warp's 32 x 32 piece of the tile in shared
// memory (double-buffered) and writes it with TMA bulk tensor stores, which
// clip at the slice's bounds; the transposed copy of a mirrored tile goes
// straight to global memory (64 contiguous bytes per column and warp).
//
// Roles (320 threads, one CTA per SM, persistent over a static tile stride):
//   warp 0 lane 0 : TMA producer over a STAGES-deep shared-memory ring (in a
//                   pair, both CTAs load their halves; the leader's barrier
//                   counts the bytes of both)
//   warp 1        : TMEM allocation; lane 0 issues the MMAs (the leader only
//                   in a pair; its commits reach both CTAs' barriers)
//   warps 2..9    : epilogue, one TMEM lane (= output row) per thread; in
//                   launches whose tiles have a short main loop (K <= 2048)
//                   or that hold at most one wave of tiles, two warps per
//                   lane quadrant split a tile's 256 columns (its epilogue
//                   then takes half as long), otherwise warps 2..5 take whole
//                   tiles; two 256-column accumulators let the epilogue of
//                   one tile overlap the main loop of the next.
// Every wait is bounded (see mbar_wait_bounded); a role that gives up
// records an error code in *err, raises the CTA's abort flag and leaves;
// in-flight TMA loads and MMAs are waited for (bounded) before TMEM is freed.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx_sm100.cuh"

namespace muon {

constexpr int BM = 128;                          // rows of A (and of the accumulator) per CTA
constexpr int BN = 256;                          // columns of a tile
constexpr int BK = 64;                           // K of one TMA box (one 128-byte swizzled row of bf16)
constexpr uint32_t TMEM_COLS = 2 * BN;           // two accumulators
constexpr int MAX_PROBLEMS = 8;
constexpr int EPI_WARPS = 8;                                // two per TMEM lane quadrant, one per column half
constexpr int GEMM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int EPI_CHUNKS = BN / 32 / 2;                     // 32-column chunks per epilogue warp and tile
constexpr int STG_BYTES = 32 * 32 * 2;                      // one 32 x 32 box of 16-bit values
constexpr int STG_PER_WARP = 2 /*buffers*/ * STG_BYTES;

// A stage holds KB = 64 * KSUB elements of K.  K-major operands are KSUB
// boxes of [rows][64] (one 128-byte swizzled row each); MN-major operands are
// blocks of [KB rows][64 MN].  Several MMAs per stage amortize the stage's
// barrier wait and commit: the pair kernel takes 128-wide K stages.
template <int CG>
struct GemmCfg {
  static constexpr int TILE_M = BM * CG;                    // rows of a tile
  static constexpr int B_ROWS = BN / CG;                    // rows of B this CTA loads
  static constexpr int KSUB = CG == 1 ? 1 : 2;
  static constexpr int KB = BK * KSUB;                      // K per stage
  static constexpr int A_STAGE_BYTES = BM * KB * 2;
  static constexpr int B_STAGE_BYTES = B_ROWS * KB * 2;
  static constexpr int MN_BLOCK_BYTES = 64 * KB * 2;        // one [KB K rows][64 MN] swizzled block
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int STAGES = CG == 1 ? 4 : 3;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_WARPS * STG_PER_WARP + 1024 /*align*/ +
                                    256 /*barriers*/;
  // Bytes the leader's full barrier counts per stage (both CTAs' loads in a pair).
  static constexpr uint32_t TX_BYTES = static_cast<uint32_t>(STAGE_BYTES * CG);
};

enum GemmError : int { kErrNone = 0, kErrProducer = 1, kErrMma = 2, kErrEpilogue = 3 };

struct GemmProblem {
  int M, N, K;
  int slices;
  int mt, nt, kt;           // tile counts along M, N, K
  int tiles_per_slice;
  int tile_begin;           // first linear tile of this problem in the launch
  int group_m;              // non-symmetric problems: row tiles per raster band
  int tri;                  // symmetric output: lower-triangle tiles (+ mirror)
  int mirror;               // tri: also write the transposed tiles into the upper triangle
  int a_mn, b_mn;           // operand majors (1 = MN-major)
  int a_sym, b_sym;         // operand is a symmetric matrix stored as its lower 256-blocks (pair kernel)
  uint32_t idesc;           // tcgen05 instruction descriptor (a_mn, b_mn majors)
  float alpha, beta, gamma, f0;
  int s_pow;                // exponent of the per-slice normalization factor
  float eps;
  const float* sumsq;       // [slices] when s_pow > 0
  const void* addend;       // D (same dtype as C), may be null when beta == 0
  long long add_ld, add_bs;
  void* out;
  long long out_ld, out_bs;
  int out_f16;              // 1: C is fp16, 0: bf16
  int add_f16;              // 1: D is fp16, 0: bf16
  float* row_ss;            // optional [slices][2 nt][M]: per 128-column half of a tile, sum of bf16(C)^2
};

struct __align__(64) GemmParams {
  CUtensorMap mapA[MAX_PROBLEMS];
  CUtensorMap mapB[MAX_PROBLEMS];
  CUtensorMap mapC[MAX_PROBLEMS];     // output, 32 x 32 boxes, 64-byte swizzle
  GemmProblem prob[MAX_PROBLEMS];
  int num_problems;
  int total_tiles;
  int epi_split;                      // 1: two epilogue warps per lane quadrant, one per column half;
                                      // 0: warps 2..5 take whole tiles and warps 6..9 stay idle
  int* err;
  unsigned long long timeout_ns;
};

struct TileCoord {
  int p, slice, tm, tn;
};

// Column j (256 output columns) of a symmetric problem needs the row tiles
// from j * (256 / TILE_M) on.  Other problems are walked in bands of group_m
// row tiles, M fastest within a band, so that the tiles in flight at once
// cover a near-square block of the output and share operand rows and
// columns in L2.
template <int CG>
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& P, int t) {
  constexpr int STEP = BN / GemmCfg<CG>::TILE_M;
  int p = 0;
  while (p + 1 < P.num_problems && t >= P.prob[p + 1].tile_begin) ++p;
  const GemmProblem& pr = P.prob[p];
  const int local = t - pr.tile_begin;
  const int slice = local / pr.tiles_per_slice;
  int r = local - slice * pr.tiles_per_slice;
  int tm, tn;
  if (pr.tri) {
    int j = 0;
    while (r >= pr.mt - STEP * j) {
      r -= pr.mt - STEP * j;
      ++j;
    }
    tn = j;
    tm = STEP * j + r;
  } else {
    const int band = r / (pr.group_m * pr.nt);
    const int rem = r - band * pr.group_m * pr.nt;
    const int rows = min(pr.group_m, pr.mt - band * pr.group_m);
    tn = rem / rows;
    tm = band * pr.group_m + (rem - tn * rows);
  }
  return TileCoord{p, slice, tm, tn};
}

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  *abort_flag = 1;
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float load_elem(const void* base, long long off, int f16) {
  if (f16) return __half2float(reinterpret_cast<const __half*>(base)[off]);
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[off]);
}

// Element j of a chunk packed two per word (low half first).
__device__ __forceinline__ uint16_t half16(const uint32_t (&w32)[16], int j) {
  return static_cast<uint16_t>(w32[j >> 1] >> ((j & 1) * 16));
}

// One 32-column chunk of an epilogue row: x = v * f (+ gamma where the
// column is the row, j == dj), rounded to bf16 or fp16 two at a time into
// w32; with SS, css += (rounded x)^2 over the first ncol columns in column
// order.  (x * 1 == x: a unit factor is not multiplied.)
template <bool F16, bool SS>
__device__ __forceinline__ void round_chunk(float (&v)[32], float f, float gamma, int dj, int ncol,
                                            uint32_t (&w32)[16], float& css) {
  if (f != 1.0f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= f;
  }
  float xr[32];
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float x0 = v[j], x1 = v[j + 1];
    if (dj >= 0) {                                     // only chunks that cross the diagonal
      x0 = (j == dj) ? x0 + gamma : x0;
      x1 = (j + 1 == dj) ? x1 + gamma : x1;
    }
    if constexpr (F16) {
      const __half2 h = __floats2half2_rn(x0, x1);
      w32[j >> 1] = *reinterpret_cast<const uint32_t*>(&h);
      xr[j] = __low2float(h);
      xr[j + 1] = __high2float(h);
    } else {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
      w32[j >> 1] = *reinterpret_cast<const uint32_t*>(&h);
      xr[j] = __low2float(h);
      xr[j + 1] = __high2float(h);
    }
  }
  if constexpr (SS) {
    if (ncol == 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) css += xr[j] * xr[j];
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < ncol) css += xr[j] * xr[j];
    }
  }
}

// Fetches the line holding p into L1 (no register result, nothing waits).
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

template <int CG>
__device__ __forceinline__ void ns_gemm_body(const GemmParams& P) {
  using Cfg = GemmCfg<CG>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_STAGE_BYTES;
  uint8_t* sStg = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + EPI_WARPS * STG_PER_WARP);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = P.timeout_ns;
  // In a pair, rank 0 is the leader (issues the MMAs); tiles are per pair.
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * (P.epi_split ? EPI_WARPS : EPI_WARPS / 2) * CG);   // every working epilogue thread of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < P.num_problems; ++p) {
      tma_prefetch_desc(&P.mapA[p]);
      tma_prefetch_desc(&P.mapB[p]);
      tma_prefetch_desc(&P.mapC[p]);
    }
  }
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();   // the peer signals the leader's barriers only once they exist
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched no global memory; the previous kernel of the
  // stream may still be running (programmatic dependent launch).  Let the
  // next one start its own prologue, then wait for the previous one's results.
  pdl_launch_dependents();
  pdl_wait_prerequisites();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t last_par[STAGES];
      bool used[STAGES];
      for (int s = 0; s < STAGES; ++s) {
        used[s] = false;
        last_par[s] = 0;
      }
      bool ok = true;
      for (int t = unit; t < P.total_tiles && ok; t += units) {
        const TileCoord tc = decode_tile<CG>(P, t);
        const GemmProblem& pr = P.prob[tc.p];
        const int arow = tc.tm * Cfg::TILE_M + static_cast<int>(rank) * BM;      // this CTA's A rows
        const int brow = tc.tn * BN + static_cast<int>(rank) * Cfg::B_ROWS;      // this CTA's B rows
        // First K stage read transposed (above the diagonal 256-blocks), per symmetric operand.
        const int kbA = pr.a_sym ? (((tc.tm * Cfg::TILE_M) >> 8) + 1) * (256 / Cfg::KB) : 0x7FFFFFFF;
        const int kbB = pr.b_sym ? (tc.tn + 1) * (256 / Cfg::KB) : 0x7FFFFFFF;
        const bool a_mn0 = pr.a_mn != 0, b_mn0 = pr.b_mn != 0;
        for (int kb = 0; kb < pr.kt; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, limit)) {
            record_error(P.err, abort_flag, kErrProducer);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], Cfg::TX_BYTES);
          uint8_t* a_dst = sA + stage * Cfg::A_STAGE_BYTES;
          uint8_t* b_dst = sB + stage * Cfg::B_STAGE_BYTES;
          const int k0 = kb * Cfg::KB;
          // K-major: KSUB boxes [rows][64]; MN-major: blocks [KB][64] along M (or N).  A
          // symmetric operand's stages above the diagonal blocks are read transposed (MN-major).
          const bool amn = a_mn0 || kb >= kbA;
          const bool bmn = b_mn0 || kb >= kbB;
#pragma unroll
          for (int j = 0; j < (amn ? BM / 64 : Cfg::KSUB); ++j) {
            const int x = amn ? arow + 64 * j : k0 + 64 * j;
            const int y = amn ? k0 : arow;
            uint8_t* dst = a_dst + j * (amn ? Cfg::MN_BLOCK_BYTES : BM * BK * 2);
            if (CG == 2)
              tma_load_3d_pair(dst, &P.mapA[tc.p], &full[stage], x, y, tc.slice);
            else
              tma_load_3d(dst, &P.mapA[tc.p], &full[stage], x, y, tc.slice);
          }
#pragma unroll
          for (int j = 0; j < (bmn ? Cfg::B_ROWS / 64 : Cfg::KSUB); ++j) {
            const int x = bmn ? brow + 64 * j : k0 + 64 * j;
            const int y = bmn ? k0 : brow;
            uint8_t* dst = b_dst + j * (bmn ? Cfg::MN_BLOCK_BYTES : Cfg::B_ROWS * BK * 2);
            if (CG == 2)
              tma_load_3d_pair(dst, &P.mapB[tc.p], &full[stage], x, y, tc.slice);
            else
              tma_load_3d(dst, &P.mapB[tc.p], &full[stage], x, y, tc.slice);
          }
          used[stage] = true;
          last_par[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // Leave no bulk copy in flight into shared memory (the leader's full
        // barriers count the peer's copies too).
        for (int s = 0; s < STAGES; ++s)
          if (used[s]) {
            volatile int never = 0;
            mbar_wait_bounded(&full[s], last_par[s], &never, limit);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int iter = 0;
      bool ok = true;
      for (int t = unit; t < P.total_tiles && ok; t += units, ++iter) {
        const TileCoord tc = decode_tile<CG>(P, t);
        const GemmProblem& pr = P.prob[tc.p];
        const int acc = iter & 1;
        const uint32_t acc_par = (iter >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], acc_par ^ 1u, abort_flag, limit)) {
          record_error(P.err, abort_flag, kErrMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        // Descriptors of stage 0, advanced by adding to the start-address
        // field (bits 0-13, in 16-byte units; shared memory stays below 256 KB).
        // K-major: the next 16 K elements are 32 bytes along the swizzled row,
        // and every 64 K the next box; MN-major: the next 16 K rows are two
        // 8-row groups, 2048 bytes.
        const uint64_t mn_desc0 = smem_desc_sw128(smem_u32(sA), Cfg::MN_BLOCK_BYTES, 1024);
        const uint64_t k_desc0 = smem_desc_sw128(smem_u32(sA), 16, 1024);
        const uint64_t mn_bdesc0 = smem_desc_sw128(smem_u32(sB), Cfg::MN_BLOCK_BYTES, 1024);
        const uint64_t k_bdesc0 = smem_desc_sw128(smem_u32(sB), 16, 1024);
        const int kbA = pr.a_sym ? (((tc.tm * Cfg::TILE_M) >> 8) + 1) * (256 / Cfg::KB) : 0x7FFFFFFF;
        const int kbB = pr.b_sym ? (tc.tn + 1) * (256 / Cfg::KB) : 0x7FFFFFFF;
        const bool a_mn0 = pr.a_mn != 0, b_mn0 = pr.b_mn != 0;
        const uint32_t idesc0 = pr.idesc;
        const int kt = pr.kt;
        for (int kb = 0; kb < kt; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, limit)) {
            record_error(P.err, abort_flag, kErrMma);
            ok = false;
            break;
          }
          tc_fence_after();
          // The producer's choice of major for this stage (see its loads).
          const bool a_mn = a_mn0 || kb >= kbA;
          const bool b_mn = b_mn0 || kb >= kbB;
          const uint32_t idesc = idesc0 | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
          const uint64_t a_desc0 = a_mn ? mn_desc0 : k_desc0;
          const uint64_t b_desc0 = b_mn ? mn_bdesc0 : k_bdesc0;
          const uint64_t ad = a_desc0 + static_cast<uint64_t>((stage * Cfg::A_STAGE_BYTES) >> 4);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>((stage * Cfg::B_STAGE_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < Cfg::KB / 16; ++k) {
            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
            const uint64_t ak = a_mn ? static_cast<uint64_t>(k * (2048 >> 4))
                                     : static_cast<uint64_t>((k >> 2) * (BM * BK * 2 >> 4) + (k & 3) * 2);
            const uint64_t bk = b_mn ? static_cast<uint64_t>(k * (2048 >> 4))
                                     : static_cast<uint64_t>((k >> 2) * (Cfg::B_ROWS * BK * 2 >> 4) + (k & 3) * 2);
            if (CG == 2)
              tc_mma_f16_pair(d_tmem, ad + ak, bd + bk, idesc, accum);
            else
              tc_mma_f16(d_tmem, ad + ak, bd + bk, idesc, accum);
          }
          if (CG == 2)
            tc_commit_pair_mc(&empty[stage], 0x3);
          else
            tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 2)
          tc_commit_pair_mc(&tfull[acc], 0x3);
        else
          tc_commit(&tfull[acc]);
      }
      // Every MMA this thread issued has finished before TMEM can be freed.
      if (CG == 2)
        tc_commit_pair_mc(drain, 0x1);
      else
        tc_commit(drain);
      volatile int never = 0;
      if (!mbar_wait_bounded(drain, 0, &never, limit)) record_error(P.err, abort_flag, kErrMma);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // Warps 2..9: warp & 3 is the TMEM lane quadrant a warp may access (rows
    // 32q .. 32q + 31 of the CTA's accumulator).  With epi_split the two
    // warps of a quadrant take one 128-column half of the tile each (launches
    // whose main loop per tile is short, where the epilogue would be exposed);
    // otherwise warps 2..5 take whole tiles, which hide behind long main loops.
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;
    const bool split = P.epi_split != 0;
    const int c_begin = split ? ch * EPI_CHUNKS : 0;
    const int c_end = split ? c_begin + EPI_CHUNKS : 2 * EPI_CHUNKS;
    uint8_t* stg = sStg + (warp - 2) * STG_PER_WARP;
    const bool idle = !split && ch == 1;
    int iter = 0;
    uint32_t stores = 0;     // bulk groups this warp has committed (selects the staging buffer)
    for (int t = unit; t < P.total_tiles && !idle; t += units, ++iter) {
      const TileCoord tc = decode_tile<CG>(P, t);
      const GemmProblem& pr = P.prob[tc.p];
      const int acc = iter & 1;
      const uint32_t acc_par = (iter >> 1) & 1;
      // The tile's scale (and, in launches whose epilogue is exposed, the
      // first addend chunk) is read before the wait for the accumulator: it
      // does not depend on it, and in launches of one tile per CTA these
      // loads would otherwise start only after the main loop.
      const int row0 = tc.tm * Cfg::TILE_M + static_cast<int>(rank) * BM + q * 32;
      const int row = row0 + lane;
      const bool row_ok = row < pr.M;
      // Mirrored tiles: strictly below the 256 x 256 diagonal blocks.
      const bool mirror = pr.tri && pr.mirror && tc.tm * Cfg::TILE_M >= (tc.tn + 1) * BN;
      float f = pr.f0;
      if (pr.s_pow > 0) {
        const float s = 1.0f / (sqrtf(pr.sumsq[tc.slice]) + pr.eps);
        f *= (pr.s_pow == 2) ? s * s : s;
      }
      const long long add_slice = static_cast<long long>(tc.slice) * pr.add_bs;
      const bool use_add = pr.beta != 0.0f && pr.addend != nullptr;
      float rss0 = 0.0f, rss1 = 0.0f;   // sums of squares of the tile's two 128-column halves
      // The addend of a whole 32-column chunk (64 bytes of this row) is loaded
      // one chunk ahead, so its global-memory latency overlaps the previous
      // chunk's work instead of stalling every chunk.
      uint4 add_cur[4], add_nxt[4];
      auto load_addend = [&](int c, uint4 (&dst)[4]) {
        const int col0 = tc.tn * BN + c * 32;
        if (use_add && row_ok && col0 + 32 <= pr.N) {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(pr.addend) + add_slice +
                                                            static_cast<long long>(row) * pr.add_ld + col0);
#pragma unroll
          for (int w = 0; w < 4; ++w) dst[w] = src[w];
        }
      };
      // Split epilogues: the row's first addend chunk into registers and the
      // second into L1 before the wait (the loop loads each next chunk one
      // chunk ahead); long-K launches load the first chunk after it.
      if (split) {
        load_addend(c_begin, add_cur);
        if (use_add && row_ok && c_begin + 1 < c_end && tc.tn * BN + (c_begin + 1) * 32 + 32 <= pr.N)
          prefetch_l1(reinterpret_cast<const uint16_t*>(pr.addend) + add_slice + static_cast<long long>(row) * pr.add_ld +
                      tc.tn * BN + (c_begin + 1) * 32);
      }
      bool ok = mbar_wait_bounded(&tfull[acc], acc_par, abort_flag, limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) record_error(P.err, abort_flag, kErrEpilogue);
        break;
      }
      tc_fence_after();
      if (!split) load_addend(c_begin, add_cur);

      for (int c = c_begin; c < c_end; ++c) {
        if (c + 1 < c_end) load_addend(c + 1, add_nxt);
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN + c * 32),
                           r);
        tmem_ld_wait();
        const int col0 = tc.tn * BN + c * 32;
        if (col0 >= pr.N) continue;                       // warp-uniform (every later chunk too)
        const bool full_chunk = col0 + 32 <= pr.N;
        float v[32];
        if (pr.alpha == 1.0f) {                            // x * 1 == x: skip the multiply (uniform)
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = pr.alpha * __uint_as_float(r[j]);
        }
        if (use_add && row_ok) {
          const long long aoff = add_slice + static_cast<long long>(row) * pr.add_ld + col0;
          if (full_chunk) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              uint4 u = add_cur[w];
              const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const uint16_t lo = static_cast<uint16_t>(words[h] & 0xFFFFu);
                const uint16_t hi = static_cast<uint16_t>(words[h] >> 16);
                float flo, fhi;
                if (pr.add_f16) {
                  flo = __half2float(__ushort_as_half(lo));
                  fhi = __half2float(__ushort_as_half(hi));
                } else {
                  flo = __bfloat162float(__ushort_as_bfloat16(lo));
                  fhi = __bfloat162float(__ushort_as_bfloat16(hi));
                }
                v[w * 8 + h * 2] += pr.beta * flo;
                v[w * 8 + h * 2 + 1] += pr.beta * fhi;
              }
            }
          } else {
            for (int j = 0; j < 32 && col0 + j < pr.N; ++j)
              v[j] += pr.beta * load_elem(pr.addend, aoff + j, pr.add_f16);
          }
        }
        // Round to the output type once (two values per conversion); these
        // are the values stored.  The identity term touches only chunks that
        // cross the diagonal (warp-uniform test), and whole chunks of a valid
        // row sum every square without per-column tests.
        uint32_t w32[16];
        float css = 0.0f;
        const bool diag = pr.gamma != 0.0f && col0 < row0 + 32 && row0 < col0 + 32;
        const int ncol = row_ok ? min(32, pr.N - col0) : 0;  // columns of this row that count
        const float gm = diag ? pr.gamma : 0.0f;
        const int dj = diag ? row - col0 : -1;
        if (pr.row_ss != nullptr) {                       // sums of squares only where they are stored
          if (pr.out_f16)
            round_chunk<true, true>(v, f, gm, dj, ncol, w32, css);
          else
            round_chunk<false, true>(v, f, gm, dj, ncol, w32, css);
        } else {
          if (pr.out_f16)
            round_chunk<true, false>(v, f, gm, dj, ncol, w32, css);
          else
            round_chunk<false, false>(v, f, gm, dj, ncol, w32, css);
        }
        if (c < EPI_CHUNKS)
          rss0 += css;
        else
          rss1 += css;
        // Boxes whose innermost extent lies fully inside the slice go out by
        // TMA; the ragged last chunk of a row is written element by element,
        // so nothing past the slice's last column is ever touched.  Mirrored
        // columns go straight to global memory: for each column j the warp's
        // 32 rows are 64 contiguous bytes of output row col0 + j.
        const bool st_d = full_chunk;
        const long long out_slice = static_cast<long long>(tc.slice) * pr.out_bs;
        uint16_t* out16 = reinterpret_cast<uint16_t*>(pr.out);
        if (st_d) {
          // The staging buffer used two stores ago must have been read out.
          uint8_t* sd = stg + (stores & 1u) * STG_BYTES;
          if (lane == 0 && stores >= 2) bulk_wait_group_read<1>();
          __syncwarp();
          // Row `lane`, 64 bytes, 16-byte chunks placed by the 64-byte swizzle.
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint4 val = make_uint4(w32[4 * w], w32[4 * w + 1], w32[4 * w + 2], w32[4 * w + 3]);
            *reinterpret_cast<uint4*>(sd + lane * 64 + ((w ^ ((lane >> 1) & 3)) << 4)) = val;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&P.mapC[tc.p], sd, col0, row0, tc.slice);
            bulk_commit_group();
          }
          ++stores;
        } else if (row_ok) {
          for (int j = 0; j < 32 && col0 + j < pr.N; ++j)
            out16[out_slice + static_cast<long long>(row) * pr.out_ld + col0 + j] = half16(w32, j);
        }
        if (mirror && row_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < pr.N) out16[out_slice + static_cast<long long>(col0 + j) * pr.out_ld + row] = half16(w32, j);
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) add_cur[w] = add_nxt[w];
      }
      if (pr.row_ss != nullptr && row_ok) {
        float* rs = pr.row_ss + (static_cast<long long>(tc.slice) * 2 * pr.nt + 2 * tc.tn) * pr.M + row;
        if (split) {
          rs[static_cast<long long>(ch) * pr.M] = ch == 0 ? rss0 : rss1;
        } else {
          rs[0] = rss0;
          rs[pr.M] = rss1;
        }
      }
      // The MMA issuer reuses this accumulator only for a later tile of
      // this CTA; after the last one nothing waits for it.
      if (t + units < P.total_tiles) {
        tc_fence_before();
        if (CG == 2)
          mbar_arrive_leader(&tempty[acc]);
        else
          mbar_arrive(&tempty[acc]);
      }
    }
    // Every store has landed before the kernel (and its shared memory) ends.
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA of a pair leaves while the other may still signal its barriers.
  if (CG == 2) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Failure-path probe: waits with the same bounded wait on a barrier that no
// one arrives on, and records the timeout like the GEMM roles do.
__global__ void bounded_wait_probe_kernel(int* err, unsigned long long limit_ns, int code) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns)) record_error(err, &abort_flag, code);
}

__global__ void __launch_bounds__(GEMM_THREADS, 1) ns_gemm_kernel(const __grid_constant__ GemmParams P) {
  ns_gemm_body<1>(P);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    ns_gemm_pair_kernel(const __grid_constant__ GemmParams P) {
  ns_gemm_body<2>(P);
}

}  // namespace muon
