// Bandwidth-bound kernels of the Muon / NorMuon step (sm_100a):
//   momentum + Nesterov + per-chunk sum of squares, the per-slice
//   finalization of those sums, NorMuon row statistics and slice factors,
//   and the weight update.
//
// Work is split into fixed chunks of CHUNK elements of one slice's
// row-major [rows, cols] index space, so every reduction has a fixed order
// (a chunk's partial is reduced by a fixed tree; a slice's partials are then
// summed in chunk order): results are bitwise reproducible and independent
// of the batch a slice is in.  Threads move 8 consecutive elements of a row
// at a time (16-byte loads for bf16) when the row length and strides allow,
// else one element.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx_sm100.cuh"

namespace muon {

constexpr int EW_THREADS = 256;
constexpr int CHUNK = 8192;       // elements per chunk (a multiple of EW_THREADS * 8)
constexpr int MAX_SEGS = 16;      // batches per elementwise launch

struct EwSeg {
  long long n, rows, cols;
  long long chunks_per_slice;
  long long chunk_begin;          // first global chunk of this segment
  long long slice_begin;          // first global slice of this segment (for per-slice arrays)
  long long row_begin;            // first global row of this segment (for per-row arrays)
  int vec8;                       // 1: cols, strides and pointers allow 8-wide vectors
  int flat;                       // 1: every tensor the kernel touches is one dense [n*rows*cols] array
  // tensors: (ptr, ld, batch stride, dtype: 0 f32, 1 bf16)
  const void* g; long long g_ld, g_bs; int g_dt;
  void* m; long long m_ld, m_bs; int m_dt;
  void* u; long long u_ld, u_bs;                 // bf16
  const void* o; long long o_ld, o_bs;           // bf16 (update: Newton-Schulz output)
  void* w; long long w_ld, w_bs; int w_dt;
  void* wc; long long wc_ld, wc_bs;              // optional bf16 copy
  float* variance;                               // [n*rows]
  const float* rsq;                              // [n*rows] per-row sum of O^2 from the NS call, or null
  float lr_scale;
};

struct EwParams {
  EwSeg seg[MAX_SEGS];
  int nseg;
  long long total_chunks;
  long long total_slices;
  long long total_rows;
  float mu;
  int nesterov;
  float* partials;                // [total_chunks]
  float* sumsq_ws;                // [total_slices] (finalize writes here when a segment has no sumsq)
  float* sumsq_out[MAX_SEGS];     // per segment output (may be null -> sumsq_ws)
  // NorMuon / update
  float beta2, nor_eps, lr, wd;
  int use_normuon;
  float* row_ss;                  // [total_rows]
  float* row_d;                   // [total_rows]
  float* slice_factor;            // [total_slices]
};

__device__ __forceinline__ int find_seg_by_chunk(const EwParams& P, long long c) {
  int s = 0;
  while (s + 1 < P.nseg && c >= P.seg[s + 1].chunk_begin) ++s;
  return s;
}

__device__ __forceinline__ float ld_f(const void* p, long long off, int dt) {
  if (dt == 0) return reinterpret_cast<const float*>(p)[off];
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[off]);
}

__device__ __forceinline__ void st_f(void* p, long long off, float v, int dt) {
  if (dt == 0)
    reinterpret_cast<float*>(p)[off] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(p)[off] = __float2bfloat16_rn(v);
}

// 8 consecutive values (16-byte aligned) in f32 or bf16.
__device__ __forceinline__ void ld8(const void* p, long long off, int dt, float (&v)[8]) {
  if (dt == 0) {
    const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + off);
    float4 a = q[0], b = q[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + off);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // bf16 -> f32 is a 16-bit shift of the bit pattern.
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Stores 8 values; returns them as rounded to the stored type.
__device__ __forceinline__ void st8(void* p, long long off, int dt, float (&v)[8]) {
  if (dt == 0) {
    float4* q = reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + off);
    q[0] = make_float4(v[0], v[1], v[2], v[3]);
    q[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);   // .x = low half
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Fixed-order block sum (butterfly within warps, then warp 0 over warp sums).
__device__ __forceinline__ float block_sum(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float t = 0.0f;
  if (warp == 0) {
    t = lane < (blockDim.x >> 5) ? scratch[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;  // valid in thread 0
}

// ---------------------------------------------------------------------------
// Momentum, Nesterov, U = bf16, partial sum of U^2 per chunk.
// With mode == 1 the kernel only reads U (ns_in) and forms the partial sums
// (the Frobenius norm of a Newton-Schulz input that came without one).
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(EW_THREADS) momentum_chunks_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  __shared__ float scratch[32];
  for (long long c = blockIdx.x; c < P.total_chunks; c += gridDim.x) {
    const int si = find_seg_by_chunk(P, c);
    const EwSeg& S = P.seg[si];
    const long long local = c - S.chunk_begin;
    const long long slice = local / S.chunks_per_slice;
    const long long lc = local - slice * S.chunks_per_slice;
    const long long total = S.rows * S.cols;
    const long long e0 = lc * CHUNK;
    const long long e1 = min(e0 + CHUNK, total);
    float acc = 0.0f;
    if (S.vec8) {
      const long long flat0 = slice * S.rows * S.cols;
      for (long long e = e0 + threadIdx.x * 8; e < e1; e += EW_THREADS * 8) {
        // Dense slices need no row/column split (a 64-bit division per vector).
        long long og, om, ou;
        if (S.flat) {
          og = om = ou = flat0 + e;
        } else {
          const long long r = e / S.cols, col = e - r * S.cols;
          og = slice * S.g_bs + r * S.g_ld + col;
          om = slice * S.m_bs + r * S.m_ld + col;
          ou = slice * S.u_bs + r * S.u_ld + col;
        }
        float u[8];
        if (MODE == 0) {
          float g[8], m[8];
          ld8(S.g, og, S.g_dt, g);
          ld8(S.m, om, S.m_dt, m);
          // One rounding per operation (fused multiply-adds), in this order:
          //   M_new = fl(mu*M + G),  U = fl(mu*M_new + G)  (from the unrounded M_new)
#pragma unroll
          for (int i = 0; i < 8; ++i) m[i] = fmaf(P.mu, m[i], g[i]);
          float mn[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mn[i] = m[i];
          st8(S.m, om, S.m_dt, m);                                  // m now holds the stored values
#pragma unroll
          for (int i = 0; i < 8; ++i) u[i] = P.nesterov ? fmaf(P.mu, mn[i], g[i]) : mn[i];
          st8(S.u, ou, 1, u);                                       // u now holds bf16(U)
        } else {
          ld8(S.u, ou, 1, u);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += u[i] * u[i];
      }
    } else {
      for (long long e = e0 + threadIdx.x; e < e1; e += EW_THREADS) {
        const long long r = e / S.cols, col = e - r * S.cols;
        float uv;
        if (MODE == 0) {
          const float g = ld_f(S.g, slice * S.g_bs + r * S.g_ld + col, S.g_dt);
          const float mo = ld_f(S.m, slice * S.m_bs + r * S.m_ld + col, S.m_dt);
          const float mn = fmaf(P.mu, mo, g);
          st_f(S.m, slice * S.m_bs + r * S.m_ld + col, mn, S.m_dt);
          const float u = P.nesterov ? fmaf(P.mu, mn, g) : mn;
          const __nv_bfloat16 ub = __float2bfloat16_rn(u);
          reinterpret_cast<__nv_bfloat16*>(S.u)[slice * S.u_bs + r * S.u_ld + col] = ub;
          uv = __bfloat162float(ub);
        } else {
          uv = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(S.u)[slice * S.u_bs + r * S.u_ld + col]);
        }
        acc += uv * uv;
      }
    }
    const float tot = block_sum(acc, scratch);
    if (threadIdx.x == 0) P.partials[c] = tot;
  }
}

// One warp per slice sums that slice's chunk partials in chunk order.
__global__ void __launch_bounds__(EW_THREADS) sumsq_finalize_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (EW_THREADS / 32);
  for (long long gs = blockIdx.x * (EW_THREADS / 32) + (threadIdx.x >> 5); gs < P.total_slices; gs += warps) {
    int si = 0;
    while (si + 1 < P.nseg && gs >= P.seg[si + 1].slice_begin) ++si;
    const EwSeg& S = P.seg[si];
    const long long slice = gs - S.slice_begin;
    const float* part = P.partials + S.chunk_begin + slice * S.chunks_per_slice;
    float acc = 0.0f;
    for (long long k = lane; k < S.chunks_per_slice; k += 32) acc += part[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      float* dst = P.sumsq_out[si] ? P.sumsq_out[si] : (P.sumsq_ws + S.slice_begin);
      dst[slice] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// NorMuon row statistics.
//   ss = sum_j O_ij^2;  v <- beta2*v + (1-beta2)*ss/cols;  d = 1/(sqrt(v)+eps)
// Segments whose Newton-Schulz call left the row sums (rsq) take them from
// there, one thread per row; the others read O, one warp per row.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void normuon_row_finish(const EwParams& P, const EwSeg& S, long long lr, long long gr,
                                                   float ss) {
  float* vp = S.variance + lr;
  const float vn = P.beta2 * (*vp) + (1.0f - P.beta2) * (ss / static_cast<float>(S.cols));
  *vp = vn;
  P.row_ss[gr] = ss;
  P.row_d[gr] = 1.0f / (sqrtf(vn) + P.nor_eps);
}

__device__ __forceinline__ int find_seg_by_row(const EwParams& P, long long gr) {
  int si = 0;
  while (si + 1 < P.nseg && gr >= P.seg[si + 1].row_begin) ++si;
  return si;
}

__global__ void __launch_bounds__(EW_THREADS) normuon_rows_from_sums_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const long long threads = static_cast<long long>(gridDim.x) * EW_THREADS;
  for (long long gr = static_cast<long long>(blockIdx.x) * EW_THREADS + threadIdx.x; gr < P.total_rows;
       gr += threads) {
    const EwSeg& S = P.seg[find_seg_by_row(P, gr)];
    if (S.rsq == nullptr) continue;
    const long long lr = gr - S.row_begin;
    normuon_row_finish(P, S, lr, gr, S.rsq[lr]);
  }
}

__global__ void __launch_bounds__(EW_THREADS) normuon_rows_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (EW_THREADS / 32);
  for (long long gr = blockIdx.x * (EW_THREADS / 32) + (threadIdx.x >> 5); gr < P.total_rows; gr += warps) {
    const int si = find_seg_by_row(P, gr);
    const EwSeg& S = P.seg[si];
    if (S.rsq != nullptr) continue;                 // warp-uniform
    const long long lr = gr - S.row_begin;
    const long long slice = lr / S.rows, r = lr - slice * S.rows;
    const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(S.o) + slice * S.o_bs + r * S.o_ld;
    float acc = 0.0f;
    if (S.vec8) {
      for (long long j = lane * 8; j < S.cols; j += 256) {
        float v[8];
        ld8(o, j, 1, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += v[i] * v[i];
      }
    } else {
      for (long long j = lane; j < S.cols; j += 32) {
        const float v = __bfloat162float(o[j]);
        acc += v * v;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) normuon_row_finish(P, S, lr, gr, acc);
  }
}

// Per-row sums of squares of a Newton-Schulz output from per-tile partials:
// out[s][r] = sum over t < nt, in order, of part[(s nt + t) rows + r].
__global__ void __launch_bounds__(EW_THREADS) row_partials_finalize_kernel(const float* part, int nt, long long rows,
                                                                           long long n, float* out) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const long long total = n * rows;
  const long long threads = static_cast<long long>(gridDim.x) * EW_THREADS;
  for (long long i = static_cast<long long>(blockIdx.x) * EW_THREADS + threadIdx.x; i < total; i += threads) {
    const long long sl = i / rows, r = i - sl * rows;
    const float* p = part + sl * nt * rows + r;
    float acc = 0.0f;
    for (int t = 0; t < nt; ++t) acc += p[static_cast<long long>(t) * rows];
    out[i] = acc;
  }
}

// Per-row sums of squares of a bf16 [n][rows][cols] strided view, one warp
// per row: out[s][r] = sum_j O[s][r][j]^2.
__global__ void __launch_bounds__(EW_THREADS) rows_sumsq_kernel(const __nv_bfloat16* O, long long ld, long long bs,
                                                                long long rows, long long cols, long long n,
                                                                float* out) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (EW_THREADS / 32);
  for (long long i = blockIdx.x * (EW_THREADS / 32) + (threadIdx.x >> 5); i < n * rows; i += warps) {
    const long long sl = i / rows, r = i - sl * rows;
    const __nv_bfloat16* o = O + sl * bs + r * ld;
    float acc = 0.0f;
    for (long long j = lane; j < cols; j += 32) {
      const float v = __bfloat162float(o[j]);
      acc += v * v;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) out[i] = acc;
  }
}

// One block per slice: factor = ||O||_F / ||O * d||_F (0 when the latter is 0).
__global__ void __launch_bounds__(EW_THREADS) normuon_slices_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  __shared__ float scratch[32];
  for (long long gs = blockIdx.x; gs < P.total_slices; gs += gridDim.x) {
    int si = 0;
    while (si + 1 < P.nseg && gs >= P.seg[si + 1].slice_begin) ++si;
    const EwSeg& S = P.seg[si];
    const long long slice = gs - S.slice_begin;
    const long long r0 = S.row_begin + slice * S.rows;
    float s1 = 0.0f, s2 = 0.0f;
    for (long long r = threadIdx.x; r < S.rows; r += EW_THREADS) {
      const float ss = P.row_ss[r0 + r], d = P.row_d[r0 + r];
      s1 += ss;
      s2 += ss * d * d;
    }
    const float t1 = block_sum(s1, scratch);
    const float t2 = block_sum(s2, scratch);
    if (threadIdx.x == 0) P.slice_factor[gs] = t2 > 0.0f ? sqrtf(t1 / t2) : 0.0f;
  }
}

// ---------------------------------------------------------------------------
// W <- W*(1 - lr*wd) - lr*lr_scale*factor*d_row * O ; optional bf16 copy.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(EW_THREADS) update_kernel(const __grid_constant__ EwParams P) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const float keep = 1.0f - P.lr * P.wd;
  for (long long c = blockIdx.x; c < P.total_chunks; c += gridDim.x) {
    const int si = find_seg_by_chunk(P, c);
    const EwSeg& S = P.seg[si];
    const long long local = c - S.chunk_begin;
    const long long slice = local / S.chunks_per_slice;
    const long long lc = local - slice * S.chunks_per_slice;
    const long long total = S.rows * S.cols;
    const long long e0 = lc * CHUNK;
    const long long e1 = min(e0 + CHUNK, total);
    const float base = P.lr * S.lr_scale * (P.use_normuon ? P.slice_factor[S.slice_begin + slice] : 1.0f);
    const float* rowd = P.use_normuon ? P.row_d + S.row_begin + slice * S.rows : nullptr;
    if (S.vec8) {
      const long long flat0 = slice * S.rows * S.cols;
      // The row of element e changes at most once per 8 consecutive elements
      // (cols is a multiple of 8), so track it instead of dividing.
      long long r = (e0 + threadIdx.x * 8) / S.cols;
      long long rstart = r * S.cols;
      for (long long e = e0 + threadIdx.x * 8; e < e1; e += EW_THREADS * 8) {
        while (e >= rstart + S.cols) {
          rstart += S.cols;
          ++r;
        }
        const long long col = e - rstart;
        const float coef = rowd ? base * rowd[r] : base;
        long long oo, ow, oc;
        if (S.flat) {
          oo = ow = oc = flat0 + e;
        } else {
          oo = slice * S.o_bs + r * S.o_ld + col;
          ow = slice * S.w_bs + r * S.w_ld + col;
          oc = slice * S.wc_bs + r * S.wc_ld + col;
        }
        float o[8], w[8];
        ld8(S.o, oo, 1, o);
        ld8(S.w, ow, S.w_dt, w);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = fmaf(-coef, o[i], w[i] * keep);
        st8(S.w, ow, S.w_dt, w);
        if (S.wc) st8(S.wc, oc, 1, w);
      }
    } else {
      for (long long e = e0 + threadIdx.x; e < e1; e += EW_THREADS) {
        const long long r = e / S.cols, col = e - r * S.cols;
        const float coef = rowd ? base * rowd[r] : base;
        const float o = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(S.o)[slice * S.o_bs + r * S.o_ld + col]);
        const long long wo = slice * S.w_bs + r * S.w_ld + col;
        float w = ld_f(S.w, wo, S.w_dt);
        w = fmaf(-coef, o, w * keep);
        st_f(S.w, wo, w, S.w_dt);
        if (S.wc) {
          const float ws = S.w_dt == 0 ? w : __bfloat162float(__float2bfloat16_rn(w));
          reinterpret_cast<__nv_bfloat16*>(S.wc)[slice * S.wc_bs + r * S.wc_ld + col] = __float2bfloat16_rn(ws);
        }
      }
    }
  }
}

// Clears the error word at the start of a call, as a kernel so that it keeps
// the stream's chain of programmatically dependent launches.
__global__ void clear_word_kernel(int* word) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  if (threadIdx.x == 0) *word = 0;
}

// out[s][j][i] = in[s][i][j] for i < rows, j < cols: 16-bit elements, 32 x 32
// tiles staged in shared memory (one padded column against bank conflicts).
// Lets tall small slices use the fused Newton-Schulz kernel, which works on
// the short side laid out as rows.  Block (32, 8); grid (cols/32, rows/32, z)
// with the slices strided over z.
__global__ void __launch_bounds__(256) transpose16_kernel(const uint16_t* in, long long in_ld, long long in_bs,
                                                          uint16_t* out, long long out_ld, long long out_bs,
                                                          int rows, int cols, int slices) {
  __shared__ uint16_t tile[32][33];
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int s = blockIdx.z; s < slices; s += gridDim.z) {
    const uint16_t* src = in + static_cast<long long>(s) * in_bs;
    uint16_t* dst = out + static_cast<long long>(s) * out_bs;
    for (int k = threadIdx.y; k < 32; k += 8) {
      const int i = r0 + k, j = c0 + threadIdx.x;
      if (i < rows && j < cols) tile[k][threadIdx.x] = src[static_cast<long long>(i) * in_ld + j];
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += 8) {
      const int j = c0 + k, i = r0 + threadIdx.x;
      if (j < cols && i < rows) dst[static_cast<long long>(j) * out_ld + i] = tile[threadIdx.x][k];
    }
    __syncthreads();
  }
}

}  // namespace muon
