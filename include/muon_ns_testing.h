/*
 * muon_ns_testing.h — test hook exported by libmuon_ns for unit tests of the
 * tensor-core GEMM that the Newton-Schulz calls are built from.  The pages
 * have no counterpart: this exists so that the sm_100a kernel can be checked
 * one product at a time against a plain matrix product.
 *
 * muon_testing_gemm computes, for every slice s < slices,
 *     C[s] = f * (alpha * opA(A[s]) opB(B[s]) + beta * D[s]) + gamma * I
 * with opA M x K and opB K x N:
 *     a_mn == 0: A[s] is stored [M][K] row-major;  a_mn == 1: stored [K][M]
 *     b_mn == 0: B[s] is stored [N][K] row-major (C = A B^T); b_mn == 1: [K][N]
 * f = f0 * (1/(sqrt(sumsq[s]) + eps))^s_pow (s_pow 0, 1 or 2; sumsq device [slices]).
 * tri != 0 requires M == N and computes only the lower triangle, mirrored.
 * in_dtype (MUON_BF16 | MUON_F16) is the type of A and B; out_dtype and
 * add_dtype (MUON_BF16 | MUON_F16) the types of C and D.  D may be NULL
 * when beta == 0.  All pointers are device memory; ld/bs are in elements.
 * row_ss (device, may be NULL; non-tri only) receives, per slice, per
 * 128-column block and per row, the sum of squares of the stored C values
 * ([slices][ceil(N / 128) rounded up to even][M]).
 * cta_pair: 0 lets the library choose the tile kernel, 1 forces single-CTA
 * 128 x 256 tiles, 2 forces 2-CTA (cta_group::2) 256 x 256 tiles.
 * raster_group: row tiles per raster band of a non-symmetric problem
 * (0: the library's default).
 * The workspace (>= 256 bytes, 256-byte aligned) receives the error word.
 */
#ifndef MUON_NS_TESTING_H_
#define MUON_NS_TESTING_H_

#include "muon_ns.h"

#ifdef __cplusplus
extern "C" {
#endif

MUON_API muon_status muon_testing_gemm(int M, int N, int K, int slices, int tri, int in_dtype,
                              const void* A, int64_t lda, int64_t bsa, int a_mn,
                              const void* B, int64_t ldb, int64_t bsb, int b_mn,
                              const void* D, int64_t ldd, int64_t bsd, int add_dtype,
                              void* C, int64_t ldc, int64_t bsc, int out_dtype,
                              float alpha, float beta, float gamma, float f0,
                              int s_pow, const float* sumsq, float eps, float* row_ss,
                              int cta_pair, int raster_group, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/*
 * Failure-path hook: one thread waits, with the GEMM kernel's bounded wait,
 * on an mbarrier that nothing ever arrives on.  After `limit_ns` of global
 * time the wait gives up, the kernel writes MUON_TESTING_WAIT_TIMEOUT at
 * workspace offset 0 and returns; the context stays usable.  Workspace:
 * >= 256 bytes, 256-byte aligned, device memory.
 */
#define MUON_TESTING_WAIT_TIMEOUT 4
MUON_API muon_status muon_testing_bounded_wait(uint64_t limit_ns, void* workspace, size_t workspace_bytes,
                                               cudaStream_t stream);

/*
 * Kernel-selection switches for tests and experiments, process-wide (all
 * devices, all threads); production callers never need them.  Defaults:
 *   fused_small   1: slices with short side <= 128 run the fused clustered
 *                    kernels (long side <= 2048, or <= 4096 when not a
 *                    multiple of 8: columns resident in shared memory; long
 *                    side 2049..16384 and a multiple of 8: columns streamed
 *                    from L2); 0: every slice takes the GEMM path
 *   max_waves    32: waves of tiles per GEMM launch (0: no cap)
 *   max_problems  1: problems that share a GEMM launch beyond one wave (1..8)
 *   pdl           1: programmatic dependent launch; 0: plain launches
 *   overlap       1: a call with both fused and GEMM-path slices runs the
 *                    fused ones on a second stream of the calling thread,
 *                    joined back before the call's later work; 0: one stream
 * Sets *opts when non-NULL (after range checks: MUON_INVALID_ARG and no
 * change when a value is out of range) and returns the previous switches in
 * *previous when non-NULL.  Not to be called while another thread enqueues
 * work through the library.
 */
typedef struct {
  int32_t fused_small;
  int32_t max_waves;
  int32_t max_problems;
  int32_t pdl;
  int32_t overlap;
} muon_testing_options;

MUON_API muon_status muon_testing_set_options(const muon_testing_options* opts, muon_testing_options* previous);

#ifdef __cplusplus
}
#endif
#endif /* MUON_NS_TESTING_H_ */
