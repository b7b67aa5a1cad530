// Fused Newton-Schulz for slices whose short side is at most 128 (sm_100a).
//
// For a slice X (m x n, stored row-major, m = rows <= cols, m <= 128) every
// quintic step is
//   A = X X^T,  B = b A + c A^2,  X <- a X + B X
// (Newton-Schulz iteration as the Megatron-Core layer_sharded_muon docs and
// DeepSpeed issue #8437 describe it; the first step works on the Frobenius-
// normalized X0 = s U, s = 1 / (||U||_F + eps), formed in fp16 as the input
// is read).  With m this small each product is a few MFLOP, so the
// GEMM path spends its time in launches and pipeline fill.  Here one
// thread-block cluster of C CTAs (C = 1, 2, 4 or 8) runs all steps of one
// slice in one launch:
//
//   * CTA r keeps columns [r w, (r+1) w) of X resident in shared memory for
//     the whole iteration (w <= 512, 128 rows: rows past m are zero and stay
//     zero, since A, B and X vanish there);
//   * A = sum_r X_r X_r^T: each CTA multiplies its own columns on the tensor
//     core (fp32 in TMEM) and pushes the lower triangle of each row of its
//     partial to the CTA that owns the row's 8-row block, with distributed-
//     shared-memory stores that count their bytes on the owner's mbarrier;
//     once all C partials of its rows have arrived each owner sums them in
//     rank order (deterministic), scales and rounds them to fp16 and pushes
//     them into every CTA's copy of A the same way; once all of A's lower
//     triangle has arrived each CTA fills the upper triangle from it (A is
//     exactly symmetric, as on the GEMM path);
//   * each CTA forms B = b A + c A^2 over its copy of A (128^3, redundantly;
//     cheaper than another exchange) and its own columns of a X + B X, which
//     need no other CTA's data, and writes them back over X;
//   * after the last step the resident columns go to ns_out by TMA.
//
// The Gram form (ns_small_gram_kernel) runs the same exchange once, for
// G = kappa s^2 X0 X0^T in fp16 (kappa = 2^14, as on the GEMM path), and then
// iterates on the m x m side inside every CTA of the cluster (redundantly:
// each product is 128^3): P = a I + (b/kappa) A + (c/kappa^2) A^2,
// Q <- P Q, A <- P (P A), all fp16 with the symmetric results mirrored from
// their lower triangles; the last Q is rounded to bf16 and O = s Q X0 is
// formed on the resident columns.
//
// Precision: fp32 accumulation; in the standard form X, A and B are
// rounded to fp16 between products (every entry is at most about 1 in
// magnitude: X0 is normalized and the iteration keeps singular values near
// 1) and the last X to bf16, the output type.  bf16 iterates, as on the GEMM
// path, lose too much on slices with a very short side: with 3 or 4 rows the
// few singular values sit where the composed quintic is steep, and a model
// of bf16 arithmetic lands up to 0.05 from the exact result (fp16: <= 0.008
// for every short side up to 128).  The Gram form keeps its m x m side in
// fp16 and its X side in bf16.  Operand layouts are the 128-byte swizzled
// tiles TMA writes (64 columns x 128 rows per 16 KB block, 16-bit values
// of either type): X is read K-major for X X^T and MN-major for B X without
// any copy.
//
// 256 threads, one CTA per SM (the shared-memory request reserves the SM):
// thread 0 issues TMA and MMAs; in the epilogues warp w reads TMEM lanes
// 32 (w % 4) .. + 31 (one row per thread) and half w / 4 of the columns.
// Every mbarrier wait is bounded; a CTA that gives up records an error,
// stops issuing work and still takes every cluster barrier, so its peers
// finish too (their bounded waits for its data run out).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include "ptx_sm100.cuh"

namespace muon {

constexpr int SMALL_THREADS = 256;
constexpr int SMALL_MAX_STEPS = 16;
constexpr int SMALL_MAX_CLUSTER = 8;
constexpr int SMALL_MAX_M = 128;
constexpr int SMALL_MAX_W = 512;                       // resident columns per CTA
constexpr int SMALL_BLK = 128 * 128;                   // one 64-column block of 128 rows (16-bit)
constexpr int SMALL_X_BYTES = SMALL_MAX_W / 64 * SMALL_BLK;   // 128 KB
constexpr int SMALL_A_BYTES = 2 * SMALL_BLK;                  // A (then B in place): 128 x 128, 16-bit
constexpr int SMALL_RECV_BYTES = 128 * 512;                   // C slots of fp32 partial rows
constexpr int SMALL_SMEM_BYTES = 1024 + SMALL_X_BYTES + SMALL_A_BYTES + SMALL_RECV_BYTES + 64;

enum SmallError : int { kSmallErrLoad = 5, kSmallErrMma = 6, kSmallErrExchange = 7 };

struct __align__(64) SmallParams {
  CUtensorMap map_in;        // ns_in  [slices][m][n] bf16, box {64, 128, 1}, 128-B swizzle
  CUtensorMap map_out;       // ns_out, same geometry (used when tma_store)
  __nv_bfloat16* out;        // ns_out, for element stores
  long long out_ld, out_bs;
  const float* sumsq;        // [slices] sum of squares of each input slice
  float eps;
  int m, n;                  // short side (rows) and long side (cols)
  int w;                     // columns per CTA, a multiple of 64, <= SMALL_MAX_W
  int slice0;                // first slice of this launch
  int steps;
  int tma_store;             // n is a multiple of 8: whole 16-byte chunks, TMA clips exactly
  float kappa;               // Gram form: A is kept as kappa * A in fp16
  float a[SMALL_MAX_STEPS], b[SMALL_MAX_STEPS], c[SMALL_MAX_STEPS];
  int* err;
  unsigned long long timeout_ns;
  float* row_ss;             // optional [slices][2 C][m]: per CTA and column half, each output
                             // row's sum of squares of its stored bf16 values
  int restart;               // Gram form: restart period in iterations (0: none)
};

// Byte offset of the 16-byte chunk holding columns [8 ch, 8 ch + 8) of row r
// in a stack of 64-column SW128 blocks of 128 rows.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * SMALL_BLK + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// Byte offset of the 16-byte chunk holding columns [4 j, 4 j + 4) of row t
// of the partial-sum receive buffer (512-byte rows; chunks XOR-swizzled by
// the row so that the rows pushed by one warp land in distinct banks).
__device__ __forceinline__ uint32_t recv_chunk(int t, int j) {
  return static_cast<uint32_t>(t * 512 + ((j ^ (t & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    f[2 * h] = __uint_as_float(w[h] << 16);
    f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack_f16x8(const float (&o)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __half2 v = __floats2half2_rn(o[2 * h], o[2 * h + 1]);
    w[h] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void unpack_f16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __half2 v = *reinterpret_cast<const __half2*>(&w[h]);
    const float2 t = __half22float2(v);
    f[2 * h] = t.x;
    f[2 * h + 1] = t.y;
  }
}

// 16-bit element e (0..7, a compile-time constant after unrolling) of 8 packed values.
__device__ __forceinline__ uint32_t bf16_at(const uint4& u, int e) {
  const uint32_t word = (e >> 1) == 0 ? u.x : (e >> 1) == 1 ? u.y : (e >> 1) == 2 ? u.z : u.w;
  return (e & 1) ? (word >> 16) : (word & 0xFFFFu);
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&o)[8]) {
  return make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                    pack_bf16x2(o[6], o[7]));
}

// In place over nbytes (a multiple of 16) of 16-bit values: bf16 x -> fp16 (s x).
// The standard form's first iterate X0 = s U, s = 1 / (||U||_F + eps), so
// every entry is at most 1 in magnitude.  The caller orders the stores before
// tensor-core reads (the fence below, then a CTA barrier).
__device__ __forceinline__ void to_f16_scaled(uint8_t* p, int nbytes, float s, int tid) {
  for (int i = tid * 16; i < nbytes; i += SMALL_THREADS * 16) {
    float f[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(p + i), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] *= s;
    *reinterpret_cast<uint4*>(p + i) = pack_f16x8(f);
  }
  fence_proxy_async_smem();
}

__device__ __forceinline__ void small_record_error(int* err, volatile int* abort_flag, int code) {
  *abort_flag = 1;
  if (err) atomicCAS(err, 0, code);
}

// Two 32-column TMEM loads (64 columns of this thread's row) and one wait.
__device__ __forceinline__ void tmem_ld_64(uint32_t taddr, uint32_t (&v)[64]) {
  tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
  tmem_ld_32x32b_x32(taddr + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
  tmem_ld_wait();
}

// Fills the upper triangle of the symmetric m8 x m8 corner (G = m8 / 8 blocks
// of 8) of a 16-bit SW128 matrix from its lower triangle, in 8 x 8 blocks.
__device__ __forceinline__ void mirror_upper(uint8_t* M, int G, int tid) {
  for (int it = tid; it < G * (G + 1) / 2; it += SMALL_THREADS) {
    int bi = 0, rest = it;
    while (rest >= G - bi) {
      rest -= G - bi;
      ++bi;
    }
    const int bj = bi + rest;                       // block (bi, bj) on or above the diagonal
    uint4 src[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) src[r] = *reinterpret_cast<const uint4*>(M + sw128_chunk(8 * bj + r, bi));
    // src[r] holds M[8 bj + r][8 bi .. 8 bi + 7]; row r' of the result is
    // column r' of that block (above the diagonal of a diagonal block, the
    // row's own entries below it are kept).
#pragma unroll
    for (int rp = 0; rp < 8; ++rp) {
      uint32_t w4[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t e2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cp = 2 * h + u;                 // column of the result row
          const uint32_t mine = bf16_at(src[rp], cp);     // M[8 bi + rp][8 bi + cp] (diagonal block)
          const uint32_t mirr = bf16_at(src[cp], rp);     // M[8 bj + cp][8 bi + rp]
          e2[u] = (bi == bj && cp <= rp) ? mine : mirr;
        }
        w4[h] = e2[0] | (e2[1] << 16);
      }
      *reinterpret_cast<uint4*>(M + sw128_chunk(8 * bi + rp, bj)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  fence_proxy_async_smem();
}

// D[tmem, 128 x 128] = X Y^T over K = 128, both 128 x 128 K-major SW128
// operands in shared memory; issued by one thread, completion on `bar`.
__device__ __forceinline__ void issue_square(uint32_t d_tmem, uint32_t x0, uint32_t y0, uint32_t idesc, uint64_t* bar) {
  fence_proxy_async_smem();
  tc_fence_after();
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t xd = smem_desc_sw128(x0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
    const uint64_t yd = smem_desc_sw128(y0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
    tc_mma_f16(d_tmem, xd, yd, idesc, kk > 0 ? 1u : 0u);
  }
  tc_commit(bar);
}

// Epilogue of a 128 x 128 product for row `row` (< m8), columns
// [64 half, 64 half + 64): out = alpha acc + beta D + gamma [row == col < m],
// rounded once to fp16 or bf16.  D may be `out` itself (read first).
__device__ __forceinline__ void epi_square(uint32_t taddr, int row, int half, int m8, int m, float alpha, float beta,
                                           const uint8_t* D, bool d_f16, float gamma, uint8_t* out, bool out_f16) {
  uint32_t v[64];
  tmem_ld_64(taddr + static_cast<uint32_t>(half * 64), v);
  if (row >= m8) return;
  uint4 dv[8];
  if (D != nullptr) {
#pragma unroll
    for (int h = 0; h < 8; ++h) dv[h] = *reinterpret_cast<const uint4*>(D + sw128_chunk(row, half * 8 + h));
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    float df[8], o[8];
    if (D != nullptr) {
      if (d_f16)
        unpack_f16x8(dv[h], df);
      else
        unpack_bf16x8(dv[h], df);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = alpha * __uint_as_float(v[h * 8 + e]);
      if (D != nullptr) x += beta * df[e];
      const int col = half * 64 + h * 8 + e;
      if (gamma != 0.0f && col == row && row < m) x += gamma;
      o[e] = x;
    }
    *reinterpret_cast<uint4*>(out + sw128_chunk(row, half * 8 + h)) = out_f16 ? pack_f16x8(o) : pack_bf16x8(o);
  }
}

// Epilogue of the product on the resident columns for row `row`, columns
// [half w/2, half w/2 + w/2): X <- f (acc + a X), in place; X is read as
// fp16 (x_f16) or bf16 and written as fp16 (out_f16) or bf16.  With rss
// non-null, also the sum of squares of the stored values of those columns
// (zero outside the slice) is written to *rss for rows below m.
__device__ __forceinline__ void epi_columns(uint32_t taddr, int row, int half, int w, int m8, float a, float f,
                                            uint8_t* Xs, bool x_f16, bool out_f16, float* rss = nullptr, int m = 0) {
  const int hw = w >> 1;
  const int cend = half * hw + hw;
  float ss = 0.0f;
#pragma unroll 1
  for (int c0 = half * hw; c0 < cend; c0 += 64) {
    const bool two = c0 + 64 <= cend;               // warp-uniform: 64 or 32 columns
    uint32_t v[64];
    if (two) {
      tmem_ld_64(taddr + static_cast<uint32_t>(c0), v);
    } else {
      tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0), *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld_wait();
    }
    if (row < m8) {
      const int nch = two ? 8 : 4;
      uint4 xv[8];
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < nch) xv[h] = *reinterpret_cast<const uint4*>(Xs + sw128_chunk(row, (c0 >> 3) + h));
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h < nch) {
          float xf[8], o[8];
          if (x_f16)
            unpack_f16x8(xv[h], xf);
          else
            unpack_bf16x8(xv[h], xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x = __uint_as_float(v[h * 8 + e]);
            x += a * xf[e];
            o[e] = x * f;
          }
          const uint4 pk = out_f16 ? pack_f16x8(o) : pack_bf16x8(o);
          *reinterpret_cast<uint4*>(Xs + sw128_chunk(row, (c0 >> 3) + h)) = pk;
          if (rss != nullptr) {
            float st[8];
            if (out_f16)
              unpack_f16x8(pk, st);
            else
              unpack_bf16x8(pk, st);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += st[e] * st[e];
          }
        }
      }
    }
  }
  if (rss != nullptr && row < m) *rss = ss;
  fence_proxy_async_smem();
}

// ---------------------------------------------------------------------------
// Per-CTA state shared by the two clustered kernels (resident and streaming)
// and the steps they have in common: the bounded wait on the MMA barrier and
// the cluster exchange that turns each CTA's partial X_r X_r^T (fp32, TMEM
// columns [0, 128)) into the full A = fA * X X^T in every CTA's As.
// ---------------------------------------------------------------------------
struct SmallCta {
  int tid, warp, quarter, half, row;
  uint32_t tlane, rank;
  int C, m, m8, G, kb, Rm;
  uint32_t tmem;
  uint8_t* As;               // A (B = b A + c A^2 in place), K-major SW128, 128 x 128
  uint8_t* Rv;               // receive slots; Gram: P and Q after the first exchange
  uint32_t a0, rv0;
  uint64_t* mma_bar;
  uint64_t* recv_bar;        // owner: partial rows of its blocks received
  uint64_t* a_bar;           // A's lower triangle received
  uint32_t mph = 0;          // completed phases of the MMA barrier
  uint32_t xphase = 0;       // completed exchanges
  uint32_t recv_bytes = 0, a_bytes = 0;
  bool ok = true;
  bool pending = false;      // an MMA commit whose wait gave up
  volatile int* abort_flag;
  int* err;
  unsigned long long timeout;

  // Row blocks of 8 are dealt to the C CTAs in the order 0, G-1, 1, G-2, ...
  // in runs of kb, so that every CTA reduces about the same share of the
  // lower triangle; a receive slot holds the kb blocks of one owner.
  __device__ __forceinline__ int fold(int b) const {
    const int lo = min(b, G - 1 - b);
    return 2 * lo + (b > G - 1 - b ? 1 : 0);
  }
  __device__ __forceinline__ int unfold(int p) const { return (p & 1) ? G - 1 - (p >> 1) : (p >> 1); }

  __device__ __forceinline__ void init(int m_, volatile int* abort_, int* err_, unsigned long long timeout_) {
    tid = threadIdx.x;
    warp = tid >> 5;
    quarter = warp & 3;                       // TMEM lanes 32 quarter .. + 31
    half = warp >> 2;                         // column half handled in the epilogues
    row = quarter * 32 + (tid & 31);          // TMEM lane = row of the 128-row tiles
    tlane = static_cast<uint32_t>(quarter * 32) << 16;
    rank = cluster_ctarank();
    C = static_cast<int>(gridDim.x);          // the cluster spans gridDim.x
    m = m_;
    m8 = (m + 7) & ~7;                        // rows / columns of A that can be nonzero
    G = m8 >> 3;
    kb = (G + C - 1) / C;
    Rm = kb * 8;                              // rows per receive slot (C * Rm <= 128)
    abort_flag = abort_;
    err = err_;
    timeout = timeout_;
    // Bytes one exchange delivers to this CTA: as an owner, the partial rows
    // of its blocks from every CTA (16 bytes per 4 columns up to the
    // diagonal); and A's lower triangle in 8 x 8 blocks from all owners.
    recv_bytes = 0;
    for (int lb = 0; lb < kb && static_cast<int>(rank) * kb + lb < G; ++lb) {
      const int b = unfold(static_cast<int>(rank) * kb + lb);
      for (int r8 = 0; r8 < 8; ++r8) recv_bytes += 16u * static_cast<uint32_t>(((8 * b + r8) >> 2) + 1);
    }
    recv_bytes *= static_cast<uint32_t>(C);
    a_bytes = 64u * static_cast<uint32_t>(G * (G + 1));
  }

  // Waits (all threads) for the MMA barrier's next phase.
  __device__ __forceinline__ bool wait_mma() {
    const bool got = mbar_wait_bounded(mma_bar, mph & 1u, abort_flag, timeout);
    const bool all = __syncthreads_and(got) != 0;
    if (!all) {
      pending = true;
      if (tid == 0) small_record_error(err, abort_flag, kSmallErrMma);
    }
    ++mph;
    return all;
  }

  // A = fA * (sum over the cluster of the partials in TMEM [0, 128)), into
  // every CTA's As (fp16), upper triangle mirrored.
  // Partial rows and A's rows travel as st.async stores that complete bytes
  // on the receiver's mbarrier, so each CTA waits only for the data it needs.
  // (Every CTA's next exchange starts after it holds this exchange's A,
  // which needs every owner to have finished reading its receive slots: the
  // slots and barriers are never overwritten early.)
  __device__ __forceinline__ void exchange(float fA) {
    if (C == 1) {
      exchange_local(fA);
      return;
    }
    if (ok && tid == 0) {
      mbar_arrive_expect_tx(recv_bar, recv_bytes);
      mbar_arrive_expect_tx(a_bar, a_bytes);
    }
    // push row `row` of the partial, its lower triangle (4-column chunks up
    // to the diagonal) within columns [64 half, 64 half + 64), to the CTA
    // that owns the row's 8-row block
    if (ok && half * 64 < m8) {
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_64(tmem + tlane + static_cast<uint32_t>(half * 64), v);
      if (row < m8) {
        const int p = fold(row >> 3);
        const int owner = p / kb;
        const int t = static_cast<int>(rank) * Rm + (p - owner * kb) * 8 + (row & 7);   // slot `rank`
        const int jn = min(16, (row >> 2) + 1 - half * 16);                             // chunks to send
        const uint32_t rbar = mapa_shared(smem_u32(recv_bar), static_cast<uint32_t>(owner));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < jn) {
            const uint32_t dst = mapa_shared(rv0 + recv_chunk(t, half * 16 + j), static_cast<uint32_t>(owner));
            st_async_v4(dst, make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]), rbar);
          }
        }
      }
    }
    tc_fence_before();        // the TMEM reads above precede the next product's writes
    // owner: wait for its slots, then for its row blocks b,
    // A[8b .. 8b+7][0 .. 8b+7] = fA * sum over the slots in rank order,
    // pushed to every CTA (the diagonal block's upper half carries unsent
    // entries; the mirror below replaces it)
    if (ok) {
      const bool got = mbar_wait_cluster_bounded(recv_bar, xphase & 1u, abort_flag, timeout);
      ok = __syncthreads_and(got) != 0;
      if (!ok && tid == 0) small_record_error(err, abort_flag, kSmallErrExchange);
    }
    if (ok) {
      int items = 0;
      for (int lb = 0; lb < kb && static_cast<int>(rank) * kb + lb < G; ++lb)
        items += 8 * (unfold(static_cast<int>(rank) * kb + lb) + 1);
      for (int it = tid; it < items; it += SMALL_THREADS) {
        int lb = 0, rest = it, b = unfold(static_cast<int>(rank) * kb);
        while (rest >= 8 * (b + 1)) {
          rest -= 8 * (b + 1);
          ++lb;
          b = unfold(static_cast<int>(rank) * kb + lb);
        }
        const int r8 = rest / (b + 1);
        const int g = rest - r8 * (b + 1);
        const int tl = lb * 8 + r8;                 // row within each slot
        float4 lo[SMALL_MAX_CLUSTER], hi[SMALL_MAX_CLUSTER];
#pragma unroll
        for (int q = 0; q < SMALL_MAX_CLUSTER; ++q) {
          if (q < C) {
            lo[q] = *reinterpret_cast<const float4*>(Rv + recv_chunk(q * Rm + tl, 2 * g));
            hi[q] = *reinterpret_cast<const float4*>(Rv + recv_chunk(q * Rm + tl, 2 * g + 1));
          }
        }
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int q = 0; q < SMALL_MAX_CLUSTER; ++q) {
          if (q < C) {
            acc[0] += lo[q].x; acc[1] += lo[q].y; acc[2] += lo[q].z; acc[3] += lo[q].w;
            acc[4] += hi[q].x; acc[5] += hi[q].y; acc[6] += hi[q].z; acc[7] += hi[q].w;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= fA;
        const uint4 pk = pack_f16x8(acc);
        const uint32_t dst = a0 + sw128_chunk(8 * b + r8, g);
        const uint32_t abar = smem_u32(a_bar);
        for (int q = 0; q < C; ++q)
          st_async_v4(mapa_shared(dst, static_cast<uint32_t>(q)), pk, mapa_shared(abar, static_cast<uint32_t>(q)));
      }
    }
    // every CTA: wait for all of A's lower triangle
    if (ok) {
      const bool got = mbar_wait_cluster_bounded(a_bar, xphase & 1u, abort_flag, timeout);
      ok = __syncthreads_and(got) != 0;
      if (!ok && tid == 0) small_record_error(err, abort_flag, kSmallErrExchange);
    }
    ++xphase;
    // upper triangle of A from the lower one (local; ends with the async-proxy fence)
    if (ok) mirror_upper(As, G, tid);
    __syncthreads();
  }

  // A cluster of one: its partial is the sum, written as A from TMEM (the
  // same bits as the exchange, which adds the one slot to zero and scales).
  __device__ __forceinline__ void exchange_local(float fA) {
    if (ok && half * 64 < m8) {
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_64(tmem + tlane + static_cast<uint32_t>(half * 64), v);
      if (row < m8) {
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) {
          const int g = half * 8 + gg;
          if (g <= (row >> 3)) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = (0.0f + __uint_as_float(v[8 * gg + e])) * fA;
            *reinterpret_cast<uint4*>(As + sw128_chunk(row, g)) = pack_f16x8(acc);
          }
        }
      }
    }
    tc_fence_before();        // the TMEM reads above precede the next product's writes
    ++xphase;
    __syncthreads();
    if (ok) mirror_upper(As, G, tid);    // ends with the async-proxy fence
    __syncthreads();
  }

  // A^2 -> TMEM columns [128, 256), then B = c A^2 + b A in place over A (fp16).
  __device__ __forceinline__ void form_b(float cb, float cc) {
    const uint32_t idesc_sq = mma_idesc_f16(0, 0, 0, 128, 128);
    if (ok) {
      if (tid == 0) {
        fence_proxy_async_smem();
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t d = smem_desc_sw128(a0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
          tc_mma_f16(tmem + 128, d, d, idesc_sq, kk > 0 ? 1u : 0u);
        }
        tc_commit(mma_bar);
      }
      ok = wait_mma();
    }
    if (ok) {
      tc_fence_after();
      epi_square(tmem + tlane + 128u, row, half, m8, m, cc, cb, As, true, 0.0f, As, true);
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
  }
};

// The whole iteration, for a kernel whose columns `X` provide
//   to_half(c, s)          : X_r <- fp16(s X_r) before the first product (the
//                            streaming kernel converts each block as it reads the input)
//   partial(c, k, h)       : TMEM [0, 128) = this CTA's X_r X_r^T before step k, X in
//                            fp16 (h) or bf16 (the input's at k = 0; the streaming kernel
//                            accumulates the later ones during its passes, so it only
//                            does k = 0)
//   apply(c, F, a, f, rss, next, h, ho) : X_r <- f (F X_r + a X_r) with F a 128 x 128
//                            K-major matrix in shared memory, F and X in fp16 (h) or
//                            bf16, the result stored as fp16 (ho) or bf16; rss (or
//                            null): this thread's row sum of squares of the stored
//                            values; next: a later exchange will need this X's partial
// Standard form: X0 = s U in fp16, then per step exchange, B, apply, all in
// fp16 (X, A, B; fp32 accumulation) with the last X stored as bf16.  (bf16
// iterates, as on the GEMM path, miss the 3e-2 bar on slices with a short
// side of 3 or 4, whose few singular values sit where the composed quintic
// is steep; fp16 keeps every short side within a fifth of it.)  Gram form:
// one exchange of kappa s^2 X0 X0^T, the m x m iteration on P and Q (fp16,
// kappa-scaled A, every CTA alike), restarts every P.restart steps
// (X <- xf Q X, A again from an exchange, Q = I), and O = xf Q X, the X
// side in bf16.
template <bool GRAM, class Cols>
__device__ __forceinline__ void small_iterate(SmallCta& c, Cols& X, const SmallParams& P, float s, float* row_slot) {
  if (!GRAM) {
    X.to_half(c, s);
    for (int k = 0; k < P.steps; ++k) {
      X.partial(c, k, true);
      c.exchange(1.0f);
      c.form_b(P.b[k], P.c[k]);
      const bool last = k == P.steps - 1;
      X.apply(c, c.a0, P.a[k], 1.0f, (last && P.row_ss != nullptr) ? row_slot : nullptr, !last, true, !last);
    }
    return;
  }
  X.partial(c, 0, false);
  c.exchange(P.kappa * (s * s));
  uint8_t* Pb = c.Rv;                             // P (and, at a segment's start, the first Q)
  uint8_t* Qb = c.Rv + SMALL_A_BYTES;             // Q
  const int tid = c.tid;
  auto clear_pq = [&]() {
    for (int i = tid; i < 2 * SMALL_A_BYTES / 16; i += SMALL_THREADS)
      reinterpret_cast<uint4*>(c.Rv)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    __syncthreads();
  };
  clear_pq();
  const uint32_t idesc_h = mma_idesc_f16(0, 0, 0, 128, 128);
  const float kap = P.kappa;
  const int R = P.restart;
  auto restart_at = [&](int k) { return R > 0 && k > 0 && k < P.steps && k % R == 0; };
  float xf = s;                                   // X's factor: s while X is the input
  int seg_start = 0;
  for (int k = 0; k < P.steps; ++k) {
    if (restart_at(k)) {
      // X <- xf Q X (Q in bf16)
      X.apply(c, smem_u32(Qb), 0.0f, xf, nullptr, true, false, false);
      xf = 1.0f;
      X.partial(c, k, false);
      tc_fence_before();
      __syncthreads();
      cluster_sync();       // no CTA still reads its Q when peers push partial rows over it
      c.exchange(kap);
      clear_pq();
      seg_start = k;
    }
    const bool first = k == seg_start;
    const bool end = k == P.steps - 1 || restart_at(k + 1);
    uint8_t* Pd = first ? Qb : Pb;               // Q = P at a segment's start
    // P = a I + (b / kappa) A + (c / kappa^2) A^2; bf16 when it is the segment's final Q
    if (c.ok) {
      if (tid == 0) issue_square(c.tmem, c.a0, c.a0, idesc_h, c.mma_bar);
      c.ok = c.wait_mma();
    }
    if (c.ok) {
      tc_fence_after();
      epi_square(c.tmem + c.tlane, c.row, c.half, c.m8, c.m, P.c[k] / (kap * kap), P.b[k] / kap, c.As, true, P.a[k],
                 Pd, !(first && end));
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (c.ok) mirror_upper(Pd, c.G, tid);
    __syncthreads();
    if (!first) {
      // Q <- P Q, bf16 when the segment ends
      if (c.ok) {
        if (tid == 0) issue_square(c.tmem, smem_u32(Pb), smem_u32(Qb), idesc_h, c.mma_bar);
        c.ok = c.wait_mma();
      }
      if (c.ok) {
        tc_fence_after();
        epi_square(c.tmem + c.tlane, c.row, c.half, c.m8, c.m, 1.0f, 0.0f, nullptr, false, 0.0f, Qb, !end);
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncthreads();
      if (c.ok) mirror_upper(Qb, c.G, tid);
      __syncthreads();
    }
    if (!end) {
      // R = P A, then A <- P R (fp16, each over A in place once its product is done)
      for (int h = 0; h < 2; ++h) {
        if (c.ok) {
          if (tid == 0) issue_square(c.tmem, smem_u32(Pd), c.a0, idesc_h, c.mma_bar);
          c.ok = c.wait_mma();
        }
        if (c.ok) {
          tc_fence_after();
          epi_square(c.tmem + c.tlane, c.row, c.half, c.m8, c.m, 1.0f, 0.0f, nullptr, false, 0.0f, c.As, true);
          fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        if (c.ok) mirror_upper(c.As, c.G, tid);
        __syncthreads();
      }
    }
  }
  // O = xf Q X (Q in bf16)
  X.apply(c, smem_u32(Qb), 0.0f, xf, P.row_ss != nullptr ? row_slot : nullptr, false, false, false);
}

// ---------------------------------------------------------------------------
// Resident columns: CTA r keeps X[:, r w, (r+1) w) in shared memory (w <= 512).
// ---------------------------------------------------------------------------
struct ResidentCols {
  uint8_t* Xs;
  int w;

  __device__ __forceinline__ void to_half(SmallCta& c, float s) {
    if (c.ok) to_f16_scaled(Xs, (w >> 6) * SMALL_BLK, s, c.tid);
    __syncthreads();
  }

  __device__ __forceinline__ void partial(SmallCta& c, int, bool h) {
    if (!c.ok) return;
    const uint32_t idesc_sq = mma_idesc_f16(h ? 0u : 1u, 0, 0, 128, 128);
    if (c.tid == 0) {
      fence_proxy_async_smem();
      tc_fence_after();
      const uint32_t x0 = smem_u32(Xs);
      for (int kk = 0; kk < w / 16; ++kk) {
        const uint64_t d = smem_desc_sw128(x0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
        tc_mma_f16(c.tmem, d, d, idesc_sq, kk > 0 ? 1u : 0u);
      }
      tc_commit(c.mma_bar);
    }
    c.ok = c.wait_mma();
  }

  __device__ __forceinline__ void apply(SmallCta& c, uint32_t f0, float a, float f, float* rss, bool, bool h,
                                        bool ho) {
    // F X_r -> TMEM [0, w)
    if (c.ok) {
      if (c.tid == 0) {
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t x0 = smem_u32(Xs);
        for (int nc = 0; nc < w; nc += 256) {
          const int N = min(256, w - nc);
          const uint32_t idesc = mma_idesc_f16(h ? 0u : 1u, 0, 1, 128, static_cast<uint32_t>(N));
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = smem_desc_sw128(f0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(x0 + (nc >> 6) * SMALL_BLK + kk * 16 * 128, SMALL_BLK, 1024);
            tc_mma_f16(c.tmem + static_cast<uint32_t>(nc), ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(c.mma_bar);
      }
      c.ok = c.wait_mma();
    }
    // X <- f (F X + a X), in place
    if (c.ok) {
      tc_fence_after();
      epi_columns(c.tmem + c.tlane, c.row, c.half, w, c.m8, a, f, Xs, h, ho, rss, c.m);
    }
    tc_fence_before();
    __syncthreads();
  }
};

template <bool GRAM>
__device__ __forceinline__ void ns_small_body(const SmallParams& P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Xs = smem;
  uint8_t* As = Xs + SMALL_X_BYTES;   // A, overwritten in place by B = b A + c A^2
  uint8_t* Rv = As + SMALL_A_BYTES;   // partial rows pushed here by every CTA of the cluster
  // [0] load, [1] MMA, [2] partial rows received (owner), [3] A received
  uint64_t* bars = reinterpret_cast<uint64_t*>(Rv + SMALL_RECV_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  SmallCta c;
  c.init(P.m, abort_flag, P.err, P.timeout_ns);
  const int tid = c.tid;
  const int slice = P.slice0 + static_cast<int>(blockIdx.y);
  const int w = P.w;
  const int nblk = w >> 6;
  const uint32_t ncols = w > 256 ? 512u : 256u;     // P and A^2 take 256 columns; a X + B X takes w
  // This thread's slot for its row's partial sum of squares of the output.
  float* row_slot = P.row_ss == nullptr
                        ? nullptr
                        : P.row_ss + (static_cast<long long>(slice) * (2 * c.C) + 2 * static_cast<int>(c.rank) + c.half) *
                                         P.m + c.row;

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_desc(&P.map_in);
    tma_prefetch_desc(&P.map_out);
  }
  if (c.warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  // A outside its m8 x m8 corner is never written by the exchange: zero it once.
  for (int i = tid; i < SMALL_A_BYTES / 16; i += SMALL_THREADS)
    reinterpret_cast<uint4*>(As)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *tmem_slot;
  c.As = As;
  c.Rv = Rv;
  c.a0 = smem_u32(As);
  c.rv0 = smem_u32(Rv);
  c.mma_bar = &bars[1];
  c.recv_bar = &bars[2];
  c.a_bar = &bars[3];

  // Nothing above touched global memory: let the next kernel of the stream
  // start its prologue, then wait for the previous one's results.
  pdl_launch_dependents();
  pdl_wait_prerequisites();

  // ---- resident columns of the slice (zero outside it)
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], static_cast<uint32_t>(nblk * SMALL_BLK));
    for (int j = 0; j < nblk; ++j)
      tma_load_3d(Xs + j * SMALL_BLK, &P.map_in, &bars[0], static_cast<int>(c.rank) * w + 64 * j, 0, slice);
  }
  c.ok = __syncthreads_and(mbar_wait_bounded(&bars[0], 0, abort_flag, P.timeout_ns)) != 0;
  if (!c.ok && tid == 0) small_record_error(P.err, abort_flag, kSmallErrLoad);
  cluster_sync();             // every CTA of the cluster runs before its shared memory is addressed remotely

  const float s = 1.0f / (sqrtf(P.sumsq[slice]) + P.eps);
  ResidentCols X{Xs, w};
  small_iterate<GRAM>(c, X, P, s, row_slot);

  // ---- resident columns -> ns_out (rows < m, columns < n)
  if (c.ok) {
    const int col_base = static_cast<int>(c.rank) * w;
    if (P.tma_store) {
      if (tid == 0) {
        for (int j = 0; j < nblk && col_base + 64 * j < P.n; ++j)
          tma_store_3d(&P.map_out, Xs + j * SMALL_BLK, col_base + 64 * j, 0, slice);
        bulk_commit_group();
        bulk_wait_group_all();
      }
    } else {
      const int chunks = w >> 3;
      __nv_bfloat16* out = P.out + static_cast<long long>(slice) * P.out_bs;
      for (int it = tid; it < P.m * chunks; it += SMALL_THREADS) {
        const int r = it / chunks;
        const int ch = it - r * chunks;
        const int col = col_base + ch * 8;
        if (col >= P.n) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(Xs + sw128_chunk(r, ch));
        __nv_bfloat16* dst = out + static_cast<long long>(r) * P.out_ld + col;
        if (col + 8 <= P.n && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
          *reinterpret_cast<uint4*>(dst) = v;
        } else {
          const uint16_t* e16 = reinterpret_cast<const uint16_t*>(&v);
          for (int e = 0; e < 8 && col + e < P.n; ++e) reinterpret_cast<uint16_t*>(dst)[e] = e16[e];
        }
      }
    }
  }

  // A commit whose wait gave up may still be running: give it one more
  // bounded wait before its TMEM is released.
  if (c.pending && tid == 0) {
    volatile int never = 0;
    (void)mbar_wait_bounded(&bars[1], (c.mph - 1u) & 1u, &never, P.timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();             // no CTA leaves while a peer may still address its shared memory
  if (c.warp == 0) tmem_dealloc(c.tmem, ncols);
}

__global__ void __launch_bounds__(SMALL_THREADS, 1) ns_small_kernel(const __grid_constant__ SmallParams P) {
  ns_small_body<false>(P);
}

__global__ void __launch_bounds__(SMALL_THREADS, 1) ns_small_gram_kernel(const __grid_constant__ SmallParams P) {
  ns_small_body<true>(P);
}

// ---------------------------------------------------------------------------
// Streaming columns: for slices too long to keep resident on a 4-CTA cluster
// (n > 2048), CTA r owns columns [r w, (r+1) w) of X (w = 128 * npair, any
// length) in global memory (ns_out after the first pass; the slice's 1 MB at
// 128 x 4096 stays in L2) and streams them through shared memory in pairs of
// 64-column blocks every step.  One pass computes, per pair p,
//   F X_p on the tensor core (TMEM [256, 384)),
//   X_p' = f (F X_p + a X_p) (bf16, staged in shared memory),
//   the next exchange's partial += X_p' X_p'^T (TMEM [0, 128)),
//   and stores X_p' back by TMA;
// a first pass over the input forms its partial only.  With 4-CTA clusters
// the B200 runs 37 clusters at once, so a 32-head batch takes one wave where
// the resident kernel's 8-CTA clusters take three.
// ---------------------------------------------------------------------------
constexpr int STREAM_PAIR = 2 * SMALL_BLK;          // two 64-column blocks [128 rows][64], 32 KB
constexpr int STREAM_STAGES = 2;                   // block pairs in flight
constexpr int STREAM_CLUSTER = 4;
constexpr int STREAM_MAX_N = 16384;
constexpr int STREAM_SMEM_BYTES = 1024 + SMALL_A_BYTES + SMALL_RECV_BYTES + STREAM_STAGES * STREAM_PAIR +
                                  2 * STREAM_PAIR + 128;

struct StreamCols {
  const CUtensorMap* map_in;
  const CUtensorMap* map_out;
  uint8_t* ring;             // STREAM_STAGES block pairs, SW128
  uint8_t* Xo;               // two block pairs: X_p' (MMA operand and TMA store source)
  uint64_t* ld_bar;          // one per ring stage
  int npair, col0, slice, n;
  uint32_t loads = 0;        // pairs loaded so far over all passes: stage g % STAGES, parity (g / STAGES) & 1
  bool src_out = false;      // X lives in ns_out (after the first pass that stored it)
  float conv = 0.0f;         // nonzero: pairs read from the input become fp16(conv x) first

  __device__ __forceinline__ void issue_load(const CUtensorMap* src, int p, uint32_t g) {
    const int st = static_cast<int>(g % STREAM_STAGES);
    uint8_t* dst = ring + st * STREAM_PAIR;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&ld_bar[st], static_cast<uint32_t>(STREAM_PAIR));
    tma_load_3d(dst, src, &ld_bar[st], col0 + 128 * p, 0, slice);
    tma_load_3d(dst + SMALL_BLK, src, &ld_bar[st], col0 + 128 * p + 64, 0, slice);
  }

  __device__ __forceinline__ bool wait_load(SmallCta& c, uint32_t g) {
    const bool got =
        mbar_wait_bounded(&ld_bar[g % STREAM_STAGES], (g / STREAM_STAGES) & 1u, c.abort_flag, c.timeout);
    const bool all = __syncthreads_and(got) != 0;
    if (!all && c.tid == 0) small_record_error(c.err, c.abort_flag, kSmallErrLoad);
    return all;
  }

  // One pass over this CTA's block pairs.  product = false: partial X X^T of
  // the input only.  product = true: X <- f (F X + a X) pair by pair, stored
  // to ns_out, with the next partial when `next` and row sums when rss != null.
  // F and X are fp16 (h) or bf16; the stored X (and its partial) fp16 (ho) or bf16.
  __device__ __forceinline__ void pass(SmallCta& c, bool product, uint32_t f0, float a, float f, float* rss,
                                       bool next, bool h, bool ho) {
    const CUtensorMap* src = src_out ? map_out : map_in;
    const uint32_t base = loads;
    const uint32_t idesc_sq = mma_idesc_f16(h ? 0u : 1u, 0, 0, 128, 128);
    const uint32_t idesc_fx = mma_idesc_f16(h ? 0u : 1u, 0, 1, 128, 128);
    const uint32_t idesc_nx = mma_idesc_f16(ho ? 0u : 1u, 0, 0, 128, 128);
    const bool convert = conv != 0.0f && !src_out;
    // thread io issues this pass's TMA loads and stores: thread 0 in the
    // input pass; in an apply pass thread 32 (another warp), so that its TMA
    // work proceeds beside thread 0's tensor-core issue
    const int io = product ? 32 : 0;
    if (c.ok && c.tid == io)
      for (int p = 0; p < min(STREAM_STAGES, npair); ++p) issue_load(src, p, base + static_cast<uint32_t>(p));
    float ss = 0.0f;
    for (int p = 0; p < npair; ++p) {
      const uint32_t g = base + static_cast<uint32_t>(p);
      if (c.ok) c.ok = wait_load(c, g);
      uint8_t* xp = ring + (g % STREAM_STAGES) * STREAM_PAIR;
      const uint32_t xp0 = smem_u32(xp);
      if (convert) {                                // the input pair as fp16(conv x), in place
        if (c.ok) to_f16_scaled(xp, STREAM_PAIR, conv, c.tid);
        __syncthreads();
      }
      if (!product) {
        if (c.ok) {
          if (c.tid == 0) {
            tc_fence_after();
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t d = smem_desc_sw128(xp0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
              tc_mma_f16(c.tmem, d, d, idesc_sq, (p | kk) != 0 ? 1u : 0u);
            }
            tc_commit(c.mma_bar);
            if (convert) {        // keep fp16 X0 in ns_out: the next pass reads it instead of converting again
              for (int b = 0; b < 2; ++b)
                if (col0 + 128 * p + 64 * b < n) tma_store_3d(map_out, xp + b * SMALL_BLK, col0 + 128 * p + 64 * b, 0, slice);
              bulk_commit_group();
            }
          }
          c.ok = c.wait_mma();
        }
      } else {
        uint8_t* xo = Xo + (p & 1) * STREAM_PAIR;
        if (c.ok && c.tid == io) bulk_wait_group_read<1>();   // the store from xo two pairs ago has read it
        // F X_p -> TMEM [256, 384); its commit also covers the previous pair's partial product
        if (c.ok) {
          if (c.tid == 0) {
            tc_fence_after();
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t ad = smem_desc_sw128(f0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(xp0 + kk * 16 * 128, SMALL_BLK, 1024);
              tc_mma_f16(c.tmem + 256u, ad, bd, idesc_fx, kk > 0 ? 1u : 0u);
            }
            tc_commit(c.mma_bar);
          }
          c.ok = c.wait_mma();
        }
        // X_p' = f (F X_p + a X_p): row `row`, columns [64 half, 64 half + 64) of the pair
        if (c.ok) {
          tc_fence_after();
          uint32_t v[64];
          tmem_ld_64(c.tmem + c.tlane + 256u + static_cast<uint32_t>(c.half * 64), v);
#pragma unroll
          for (int hh = 0; hh < 8; ++hh) {
            const uint32_t off = sw128_chunk(c.row, c.half * 8 + hh);
            float xf[8], o[8];
            if (h)
              unpack_f16x8(*reinterpret_cast<const uint4*>(xp + off), xf);
            else
              unpack_bf16x8(*reinterpret_cast<const uint4*>(xp + off), xf);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = (__uint_as_float(v[hh * 8 + e]) + a * xf[e]) * f;
            const uint4 pk = ho ? pack_f16x8(o) : pack_bf16x8(o);
            *reinterpret_cast<uint4*>(xo + off) = pk;
            if (rss != nullptr) {
              float st[8];
              if (ho)
                unpack_f16x8(pk, st);
              else
                unpack_bf16x8(pk, st);
#pragma unroll
              for (int e = 0; e < 8; ++e) ss += st[e] * st[e];
            }
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        if (c.ok && c.tid == 0 && next) {
          tc_fence_after();
          const uint32_t xo0 = smem_u32(xo);
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = smem_desc_sw128(xo0 + (kk >> 2) * SMALL_BLK + (kk & 3) * 32, 16, 1024);
            tc_mma_f16(c.tmem, d, d, idesc_nx, (p | kk) != 0 ? 1u : 0u);
          }
        }
        if (c.ok && c.tid == io) {
          for (int b = 0; b < 2; ++b)
            if (col0 + 128 * p + 64 * b < n) tma_store_3d(map_out, xo + b * SMALL_BLK, col0 + 128 * p + 64 * b, 0, slice);
          bulk_commit_group();
        }
      }
      // The stage's pair has been read by its product and by the epilogue
      // (before the barrier above), and by its store when X0 was kept: load
      // the pair STAGES ahead into it.
      if (c.ok && c.tid == io && p + STREAM_STAGES < npair) {
        if (!product && convert) bulk_wait_group_read<0>();
        issue_load(src, p + STREAM_STAGES, g + static_cast<uint32_t>(STREAM_STAGES));
      }
    }
    loads = base + static_cast<uint32_t>(npair);
    if (!product && convert) {
      if (c.tid == 0) bulk_wait_group_all();     // X0 in ns_out before the next pass loads it
      src_out = true;
    }
    if (product) {
      // the last partial product, and every store, complete before the next pass or exchange
      if (c.ok) {
        if (c.tid == 0) tc_commit(c.mma_bar);
        c.ok = c.wait_mma();
      }
      if (c.tid == io) bulk_wait_group_all();
      src_out = true;
      if (rss != nullptr && c.row < c.m) *rss = ss;
    }
    tc_fence_before();
    __syncthreads();
  }

  __device__ __forceinline__ void to_half(SmallCta&, float s) { conv = s; }   // applied as the input is read

  __device__ __forceinline__ void partial(SmallCta& c, int k, bool h) {
    if (k == 0) pass(c, false, 0u, 0.0f, 1.0f, nullptr, false, h, h);   // later partials come from the passes
  }

  __device__ __forceinline__ void apply(SmallCta& c, uint32_t f0, float a, float f, float* rss, bool next, bool h,
                                        bool ho) {
    pass(c, true, f0, a, f, rss, next, h, ho);
  }
};

template <bool GRAM>
__device__ __forceinline__ void ns_stream_body(const SmallParams& P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* As = smem;
  uint8_t* Rv = As + SMALL_A_BYTES;
  uint8_t* ring = Rv + SMALL_RECV_BYTES;
  uint8_t* Xo = ring + STREAM_STAGES * STREAM_PAIR;
  // [0, STAGES) ring loads, then MMA, partial rows received (owner), A received
  uint64_t* bars = reinterpret_cast<uint64_t*>(Xo + 2 * STREAM_PAIR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + STREAM_STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  SmallCta c;
  c.init(P.m, abort_flag, P.err, P.timeout_ns);
  const int tid = c.tid;
  const int slice = P.slice0 + static_cast<int>(blockIdx.y);
  constexpr uint32_t ncols = 512;                  // partial [0,128), products [128,256), F X_p [256,384)
  float* row_slot = P.row_ss == nullptr
                        ? nullptr
                        : P.row_ss + (static_cast<long long>(slice) * (2 * c.C) + 2 * static_cast<int>(c.rank) + c.half) *
                                         P.m + c.row;

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < STREAM_STAGES + 3; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    tma_prefetch_desc(&P.map_in);
    tma_prefetch_desc(&P.map_out);
  }
  if (c.warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  // A outside its m8 x m8 corner is never written by the exchange: zero it once.
  for (int i = tid; i < SMALL_A_BYTES / 16; i += SMALL_THREADS)
    reinterpret_cast<uint4*>(As)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *tmem_slot;
  c.As = As;
  c.Rv = Rv;
  c.a0 = smem_u32(As);
  c.rv0 = smem_u32(Rv);
  c.mma_bar = &bars[STREAM_STAGES];
  c.recv_bar = &bars[STREAM_STAGES + 1];
  c.a_bar = &bars[STREAM_STAGES + 2];
  cluster_sync();             // every CTA's barriers exist before peers address them

  // Nothing above touched global memory: let the next kernel of the stream
  // start its prologue, then wait for the previous one's results.
  pdl_launch_dependents();
  pdl_wait_prerequisites();

  const float s = 1.0f / (sqrtf(P.sumsq[slice]) + P.eps);
  StreamCols X;
  X.map_in = &P.map_in;
  X.map_out = &P.map_out;
  X.ring = ring;
  X.Xo = Xo;
  X.ld_bar = bars;
  X.npair = P.w >> 7;
  X.col0 = static_cast<int>(c.rank) * P.w;
  X.slice = slice;
  X.n = P.n;
  small_iterate<GRAM>(c, X, P, s, row_slot);

  // A product whose wait gave up may still be running: one more commit tracks
  // every product issued so far; give it a bounded wait before TMEM is released.
  if (c.pending && tid == 0) {
    volatile int never = 0;
    tc_commit(c.mma_bar);
    (void)mbar_wait_bounded(c.mma_bar, c.mph & 1u, &never, P.timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();             // no CTA leaves while a peer may still address its shared memory
  if (c.warp == 0) tmem_dealloc(c.tmem, ncols);
}

__global__ void __launch_bounds__(SMALL_THREADS, 1) ns_stream_kernel(const __grid_constant__ SmallParams P) {
  ns_stream_body<false>(P);
}

__global__ void __launch_bounds__(SMALL_THREADS, 1) ns_stream_gram_kernel(const __grid_constant__ SmallParams P) {
  ns_stream_body<true>(P);
}

}  // namespace muon
