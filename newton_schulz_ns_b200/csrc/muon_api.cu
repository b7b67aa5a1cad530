// C ABI of the Muon / NorMuon step: host-side validation, workspace layout,
// TMA descriptor encoding and the launch sequence of every call.
//
// Nothing here allocates, frees or synchronizes: every kernel and memset is
// enqueued on the caller's stream, and all scratch lives in the caller's
// workspace.  Arguments are checked before the first enqueue; a call that
// returns an error has enqueued nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/muon_ns.h"
#include "../../include/muon_ns_testing.h"
#include "elementwise.cuh"
#include "ns_gemm.cuh"
#include "ns_small.cuh"
#include "polar_express.hpp"

using namespace muon;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kErrBytes = 256;                         // error word + padding at offset 0
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s
constexpr float kGramScale = 16384.0f;                    // A is kept as kGramScale*A in fp16
constexpr int kMaxDevices = 64;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t round_up64(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- device state
struct DeviceInfo {
  bool ready = false;
  bool ok = false;
  unsigned long long ctx_id = 0;   // context the set-up was done in (0: none yet)
  int sms = 0;
  int pair_units = 0;   // 2-CTA clusters of the pair GEMM that fit on the device at once
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<unsigned long long> g_launches{0};

// Kernel-selection switches (muon_testing_set_options); production values by default.
struct Options {
  std::atomic<int> fused_small{1};
  std::atomic<int> max_waves{32};
  std::atomic<int> max_problems{1};
  std::atomic<int> pdl{1};
  std::atomic<int> overlap{1};
};
Options g_opt;

// The driver's context queries, resolved at run time like the tensor-map
// encoder (the library does not link the driver).
typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);
PFN_ctx_get_current g_ctx_current = nullptr;
PFN_ctx_get_id g_ctx_id = nullptr;

template <typename F>
bool driver_entry(const char* name, F* out) {
  if (*out) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess ||
      fn == nullptr) {
    (void)cudaGetLastError();
    return false;
  }
  *out = reinterpret_cast<F>(fn);
  return true;
}

// Unique id of the calling thread's current context (0 when there is none
// yet or the query is unavailable).  Per-device set-up is keyed by it, so a
// context torn down and re-created (cudaDeviceReset) gets fresh set-up.
unsigned long long current_ctx_id() {
  if (!driver_entry("cuCtxGetCurrent", &g_ctx_current) || !driver_entry("cuCtxGetId", &g_ctx_id)) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Checks the launch just enqueued and counts it.
inline bool launched() {
  if (cudaGetLastError() != cudaSuccess) return false;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return true;
}

// Programmatic dependent launch for every kernel of the step: each kernel
// lets the next one start its prologue and waits for its predecessor before
// its first global access (switchable for tests, muon_testing_set_options).
inline bool pdl_enabled() { return g_opt.pdl.load(std::memory_order_relaxed) != 0; }

template <typename... KArgs, typename... Args>
bool launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return launched();
}

// Zeroes the error word at workspace offset 0 (a kernel, so the launch chain holds).
inline bool clear_error_word(void* ws, cudaStream_t stream) {
  return launch_pdl(clear_word_kernel, dim3(1), dim3(32), 0, stream, reinterpret_cast<int*>(ws));
}

muon_status device_setup(int* sms_out, int* pair_units_out = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUON_CUDA_ERROR;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  const unsigned long long ctx = current_ctx_id();
  if (d.ready && ctx != 0 && ctx != d.ctx_id) d.ready = false;   // a new context: kernel attributes are gone
  if (!d.ready) {
    d.ready = true;
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.ready = false;
      return MUON_CUDA_ERROR;
    }
    d.sms = sms;
    d.ok = (major == 10 && minor == 0);
    if (d.ok) {
      if (cudaFuncSetAttribute(ns_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               GemmCfg<1>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ns_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               GemmCfg<2>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMALL_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ns_small_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMALL_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ns_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               STREAM_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ns_stream_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               STREAM_SMEM_BYTES) != cudaSuccess) {
        d.ready = false;
        return MUON_CUDA_ERROR;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
      cfg.dynamicSmemBytes = GemmCfg<2>::SMEM_BYTES;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, ns_gemm_pair_kernel, &cfg) != cudaSuccess || clusters <= 0) {
        (void)cudaGetLastError();
        clusters = sms / 2;
      }
      d.pair_units = std::min(clusters, sms / 2);
    }
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr) {
        d.ready = false;
        return MUON_CUDA_ERROR;
      }
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ctx_id = current_ctx_id();   // the calls above made the context current if it was not
  }
  if (!d.ok) return MUON_UNSUPPORTED_DEVICE;
  *sms_out = d.sms;
  if (pair_units_out) *pair_units_out = d.pair_units;
  return MUON_OK;
}

// ------------------------------------------------------------ second stream
// A call whose batches take both the fused small-side kernels and the GEMM
// path runs the fused slices on a second stream beside the GEMM launches:
// the two touch disjoint workspace regions and outputs, and the fused
// kernel holds one cluster per slice for the whole iteration while the GEMM
// chain of the other slices is a series of short launches that leave most
// SMs idle.  The second stream (highest priority, so the fused clusters are
// placed first when both are waiting) and its two events belong to the
// calling thread and device, and are made again when the device's context
// changes.  Fork and join are an event record plus a wait on each side, a
// pattern that stream capture accepts; the join is issued on every return
// path once the fork was made.
struct SideStream {
  unsigned long long ctx = 0;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  // Released when the thread ends, while their context is still the
  // current one (handles of a context that is gone are not touched).
  ~SideStream() {
    if (s == nullptr || ctx == 0 || ctx != current_ctx_id()) return;
    (void)cudaEventDestroy(fork);
    (void)cudaEventDestroy(join);
    (void)cudaStreamDestroy(s);
  }
};
thread_local SideStream t_side[kMaxDevices];

class SideFork {
 public:
  SideFork() = default;
  SideFork(const SideFork&) = delete;
  SideFork& operator=(const SideFork&) = delete;
  ~SideFork() { (void)close(); }

  // *work receives the stream the fused slices go to: the second stream
  // when `want`, else `main` itself.
  muon_status open(cudaStream_t main, bool want, cudaStream_t* work) {
    *work = main;
    if (!want) return MUON_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUON_CUDA_ERROR;
    SideStream& t = t_side[dev];
    const unsigned long long ctx = current_ctx_id();
    if (t.s == nullptr || ctx != t.ctx) {   // first use on this thread, or a new context (old handles are gone)
      // Creating a stream or an event enqueues nothing; relaxed capture mode
      // lets a first call made under stream capture do it.
      cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
      (void)cudaThreadExchangeStreamCaptureMode(&mode);
      int lo = 0, hi = 0;
      const bool ok = cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess &&
                      cudaStreamCreateWithPriority(&t.s, cudaStreamNonBlocking, hi) == cudaSuccess &&
                      cudaEventCreateWithFlags(&t.fork, cudaEventDisableTiming) == cudaSuccess &&
                      cudaEventCreateWithFlags(&t.join, cudaEventDisableTiming) == cudaSuccess;
      (void)cudaThreadExchangeStreamCaptureMode(&mode);
      if (!ok) {
        (void)cudaGetLastError();
        t.s = nullptr;   // whatever was made is left to the context
        t.fork = t.join = nullptr;
        t.ctx = 0;
        return MUON_CUDA_ERROR;
      }
      t.ctx = ctx;
    }
    if (cudaEventRecord(t.fork, main) != cudaSuccess || cudaStreamWaitEvent(t.s, t.fork, 0) != cudaSuccess) {
      (void)cudaGetLastError();
      return MUON_CUDA_ERROR;
    }
    main_ = main;
    side_ = t.s;
    join_ = t.join;
    *work = side_;
    return MUON_OK;
  }

  // Makes `main` wait for everything enqueued on the second stream.
  muon_status close() {
    if (side_ == nullptr) return MUON_OK;
    const cudaStream_t s = side_;
    side_ = nullptr;
    if (cudaEventRecord(join_, s) != cudaSuccess || cudaStreamWaitEvent(main_, join_, 0) != cudaSuccess) {
      (void)cudaGetLastError();
      return MUON_CUDA_ERROR;
    }
    return MUON_OK;
  }

 private:
  cudaStream_t main_ = nullptr, side_ = nullptr;
  cudaEvent_t join_ = nullptr;
};

// ---------------------------------------------------------------- validation
inline bool dtype_is(int32_t dt, std::initializer_list<int> allowed) {
  for (int a : allowed)
    if (dt == a) return true;
  return false;
}
inline int esize(int32_t dt) { return dt == MUON_F32 ? 4 : 2; }

bool batch_empty(const muon_batch& b) { return b.n == 0 || b.rows == 0 || b.cols == 0; }

muon_status check_shape(const muon_batch& b) {
  if (b.n < 0 || b.rows < 0 || b.cols < 0) return MUON_BAD_SHAPE;
  if (b.rows > (1 << 20) || b.cols > (1 << 20) || b.rows * b.cols > INT32_MAX || b.n > INT32_MAX)
    return MUON_BAD_SHAPE;
  return MUON_OK;
}

muon_status check_view(const muon_batch& b, const muon_view& v, std::initializer_list<int> dts, bool tma) {
  if (v.ptr == nullptr) return MUON_INVALID_ARG;
  if (!dtype_is(v.dtype, dts)) return MUON_UNSUPPORTED_DTYPE;
  if (v.ld < b.cols) return MUON_BAD_SHAPE;
  if (b.n > 1 && v.batch_stride < v.ld * (b.rows - 1) + b.cols) return MUON_BAD_SHAPE;
  if (v.batch_stride < 0) return MUON_BAD_SHAPE;
  const int es = esize(v.dtype);
  if (reinterpret_cast<uintptr_t>(v.ptr) % es) return MUON_MISALIGNED;
  if (tma) {
    if (reinterpret_cast<uintptr_t>(v.ptr) % 16 || (v.ld * es) % 16 || (b.n > 1 && (v.batch_stride * es) % 16))
      return MUON_MISALIGNED;
  }
  return MUON_OK;
}

// Every given view is one dense [n][rows][cols] array (rows ld = cols apart, slices rows*cols apart).
bool flat_ok(const muon_batch& b, std::initializer_list<const muon_view*> views) {
  for (const muon_view* v : views) {
    if (v->ptr == nullptr) continue;
    if (v->ld != b.cols || (b.n > 1 && v->batch_stride != b.rows * b.cols)) return false;
  }
  return true;
}

bool vec8_ok(const muon_batch& b, std::initializer_list<const muon_view*> views) {
  if (b.cols % 8) return false;
  for (const muon_view* v : views) {
    if (v->ptr == nullptr) continue;
    const int es = esize(v->dtype);
    if (reinterpret_cast<uintptr_t>(v->ptr) % 16 || (v->ld * es) % 16 || (v->batch_stride * es) % 16) return false;
  }
  return true;
}

muon_status check_hp(const muon_hparams* hp) {
  if (!hp) return MUON_INVALID_ARG;
  if (hp->ns_steps < 1 || hp->ns_steps > 16) return MUON_INVALID_ARG;
  const float vals[] = {hp->mu, hp->ns_eps, hp->a, hp->b, hp->c, hp->beta2, hp->nor_eps, hp->lr, hp->weight_decay};
  for (float v : vals)
    if (!std::isfinite(v)) return MUON_INVALID_ARG;
  if (hp->abc_schedule)
    for (int i = 0; i < 3 * hp->ns_steps; ++i)
      if (!std::isfinite(hp->abc_schedule[i])) return MUON_INVALID_ARG;
  if (hp->scale_mode != MUON_SCALE_SPECTRAL && hp->scale_mode != MUON_SCALE_RMS_NORM) return MUON_INVALID_ARG;
  if (!std::isfinite(hp->extra_scale_factor)) return MUON_INVALID_ARG;
  if (hp->gram_restart < 0 || hp->gram_restart > 16) return MUON_INVALID_ARG;
  return MUON_OK;
}

// The update's shape factor of a parameter [fan_out, fan_in] (see
// muon_update_scale in the header for the two modes and their sources).
bool update_scale(int64_t fan_out, int64_t fan_in, int32_t mode, float extra, float* out) {
  if (fan_out < 1 || fan_in < 1 || !std::isfinite(extra)) return false;
  const double fo = static_cast<double>(fan_out), fi = static_cast<double>(fan_in);
  double base;
  if (mode == MUON_SCALE_SPECTRAL)
    base = std::sqrt(std::max(1.0, fo / fi));
  else if (mode == MUON_SCALE_RMS_NORM)
    base = 0.2 * std::sqrt(std::max(fo, fi));
  else
    return false;
  const double v = base * static_cast<double>(extra);
  if (!std::isfinite(v)) return false;
  *out = static_cast<float>(v);
  return true;
}

muon_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return MUON_OK;
  if (ws == nullptr) return MUON_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MUON_MISALIGNED;
  if (have < need) return MUON_WORKSPACE_TOO_SMALL;
  return MUON_OK;
}

// ---------------------------------------------------------------- workspace layout
struct NsBatchWs {
  size_t off[6] = {0, 0, 0, 0, 0, 0};   // standard: A, B, X ; gram: Ah, P, Qa, Qb, R, X
  int64_t ldm = 0, bsm = 0;         // m x m buffers
  int64_t ldx = 0, bsx = 0;         // X buffer
  size_t t_off = 0;                 // tall slices on the fused path: the transposed slice [cols][rows]
  int64_t ldt = 0, bst = 0;
  size_t rs_off = 0;                // row_sumsq requested: per-tile partial row sums [n][rs_nt][rows]
  int rs_nt = 0;
};

// Partial row sums per output row that the last product leaves: one per
// 128-column half of a 256-column tile on the GEMM path, one per CTA and
// column half on the fused path (clusters of at most SMALL_MAX_CLUSTER CTAs).
inline int row_partials_per_row(int64_t cols) {
  return static_cast<int>(std::max<int64_t>(2 * ((cols + BN - 1) / BN), 2 * SMALL_MAX_CLUSTER));
}

bool small_shape_ok(int64_t rows, int64_t cols);

struct Layout {
  size_t total = 0;
  size_t partials = 0, sumsq = 0;   // norm reduction scratch
  size_t row_ss = 0, row_d = 0, factor = 0;
  std::vector<NsBatchWs> nsb;
  int64_t total_chunks = 0, total_slices = 0, total_rows = 0;
};

Layout plan_layout(const muon_batch* bs, int nb, int which) {
  Layout L;
  size_t cur = kErrBytes;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = bs[i];
    if (batch_empty(b)) continue;
    L.total_chunks += b.n * cdiv(b.rows * b.cols, CHUNK);
    L.total_slices += b.n;
    L.total_rows += b.n * b.rows;
  }
  auto take = [&](size_t bytes) {
    const size_t o = cur;
    cur = align_up(cur + bytes, kAlign);
    return o;
  };
  L.nsb.resize(nb > 0 ? nb : 0);
  if (which == 0 || which == 1 || which == 2) {
    L.partials = take(sizeof(float) * std::max<int64_t>(L.total_chunks, 1));
    L.sumsq = take(sizeof(float) * std::max<int64_t>(L.total_slices, 1));
  }
  if (which == 1 || which == 2) {
    for (int i = 0; i < nb; ++i) {
      const muon_batch& b = bs[i];
      if (batch_empty(b)) continue;
      const int64_t m = std::min(b.rows, b.cols);
      NsBatchWs& w = L.nsb[i];
      w.ldm = round_up64(m, 64);
      w.bsm = w.ldm * m;
      const size_t mm = sizeof(uint16_t) * static_cast<size_t>(w.bsm) * static_cast<size_t>(b.n);
      w.ldx = round_up64(b.cols, 64);
      w.bsx = w.ldx * b.rows;
      const size_t xbytes = sizeof(uint16_t) * static_cast<size_t>(w.bsx) * static_cast<size_t>(b.n);
      if (which == 1) {
        w.off[0] = take(mm);
        w.off[1] = take(mm);
        w.off[2] = take(xbytes);
      } else {
        for (int k = 0; k < 5; ++k) w.off[k] = take(mm);
        w.off[5] = take(xbytes);    // the iterate a restart forms (the fused kernel keeps it on chip)
      }
      if (b.row_sumsq != nullptr) {
        w.rs_nt = row_partials_per_row(b.cols);
        w.rs_off = take(sizeof(float) * static_cast<size_t>(b.n) * static_cast<size_t>(w.rs_nt) *
                        static_cast<size_t>(b.rows));
      }
      if (b.rows > b.cols && small_shape_ok(b.cols, b.rows)) {
        w.ldt = round_up64(b.rows, 64);
        w.bst = w.ldt * b.cols;
        w.t_off = take(sizeof(uint16_t) * static_cast<size_t>(w.bst) * static_cast<size_t>(b.n));
      }
    }
  }
  if (which == 3) {
    L.row_ss = take(sizeof(float) * std::max<int64_t>(L.total_rows, 1));
    L.row_d = take(sizeof(float) * std::max<int64_t>(L.total_rows, 1));
    L.factor = take(sizeof(float) * std::max<int64_t>(L.total_slices, 1));
  }
  L.total = cur;
  return L;
}

// ---------------------------------------------------------------- tensor maps
struct Mat {                 // a strided batch of row-major [rows][cols] matrices
  const void* ptr;
  int64_t rows, cols, ld, bs, n;
  int f16;                   // element type: 1 fp16, 0 bf16
};

bool encode_map(CUtensorMap* map, const Mat& m, int box_x, int box_y,
                CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(m.cols), static_cast<cuuint64_t>(m.rows),
                        static_cast<cuuint64_t>(m.n)};
  const int64_t bs = m.n > 1 ? m.bs : m.ld * m.rows;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(m.ld * 2), static_cast<cuuint64_t>(round_up64(bs * 2, 16))};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_y), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, m.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                              const_cast<void*>(m.ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One GEMM problem as the planner describes it.
struct ProblemSpec {
  int M, N, K, slices;
  int tri;
  Mat a;
  int a_mn;                  // a is [M][K] (0) or [K][M] (1)
  Mat b;
  int b_mn;                  // b is [N][K] (0) or [K][N] (1)
  int in_f16;
  float alpha, beta, gamma, f0;
  int s_pow;
  float eps;
  const float* sumsq;
  const void* addend;
  int64_t add_ld, add_bs;
  int add_f16;
  void* out;
  int64_t out_ld, out_bs;
  int out_f16;
  float* row_ss;
  int mirror;                // tri: write the upper triangle too
  int a_sym, b_sym;          // symmetric operands stored as their lower 256-blocks
};

// m x m matrices with m >= 256 are computed by the 2-CTA kernel and stored
// as their lower 256 x 256 blocks only; every consumer reads them as
// symmetric operands.  Smaller ones are stored whole (mirrored).
inline bool sym_compact(int64_t m) { return m >= 256; }

// Builds every launch of `specs` (at most MAX_PROBLEMS problems each) and
// then enqueues them, so that an encoding error enqueues nothing.
// cta_pair: 0 chooses per launch (pairs when every problem has at least 256
// rows), 1 forces single-CTA tiles, 2 forces CTA pairs.
muon_status launch_gemms(const std::vector<ProblemSpec>& specs, int sms, int* err, cudaStream_t stream,
                         int cta_pair = 0, int raster_group = 0) {
  int pair_units = 0;
  {
    int s2 = 0;
    muon_status st = device_setup(&s2, &pair_units);
    if (st != MUON_OK) return st;
  }
  struct Launch {
    GemmParams P;
    int cg;
  };
  std::vector<Launch> launches;
  // Launch shaping.  Persistent CTAs walk their tiles on a fixed stride, so
  // over a long launch they drift apart and the tiles in flight stop sharing
  // operands in L2 (measured on the Llama-8B step: one launch over all seven
  // projection shapes read 3x the DRAM bytes of per-shape launches).
  // Launches are therefore kept short: at most `max_problems` problems and
  // about `max_waves` waves of tiles each (a problem's slices are split
  // across launches when needed).  Tests can change both
  // (muon_testing_set_options; 0 waves = no cap).
  const int max_problems = std::max(1, std::min(MAX_PROBLEMS, g_opt.max_problems.load(std::memory_order_relaxed)));
  const int max_waves = std::max(0, g_opt.max_waves.load(std::memory_order_relaxed));
  auto pick_cg = [&](const ProblemSpec& s) {
    if (cta_pair == 2) return 2;
    if (cta_pair == 1 || pair_units <= 0) return 1;
    return s.M >= 256 ? 2 : 1;
  };
  // Symmetric-operand reads need the pair kernel's stage geometry.
  for (const ProblemSpec& s : specs)
    if ((s.a_sym || s.b_sym) && s.slices > 0 && s.M > 0 && s.N > 0 && pick_cg(s) != 2) return MUON_BAD_SHAPE;
  auto tiles_per_slice = [](const ProblemSpec& s, int cg) {
    const int tm = BM * cg;
    const int mt = static_cast<int>(cdiv(s.M, tm)), nt = static_cast<int>(cdiv(s.N, BN));
    if (!s.tri) return static_cast<long long>(mt) * nt;
    long long cnt = 0;
    for (int j = 0; j < nt; ++j) cnt += std::max(0, mt - (BN / tm) * j);
    return cnt;
  };
  // Split problems into slice chunks.
  std::vector<ProblemSpec> chunks;
  std::vector<int> chunk_cg;
  for (const ProblemSpec& s : specs) {
    if (s.slices == 0 || s.M == 0 || s.N == 0) continue;
    const int cg = pick_cg(s);
    const long long per = std::max<long long>(1, tiles_per_slice(s, cg));
    const long long units = cg == 2 ? std::max(1, pair_units) : std::max(1, sms);
    int step_slices = s.slices;
    if (max_waves > 0) {
      // Among chunk sizes that fit the wave budget, take the one whose launches
      // leave the fewest idle tile slots in their last waves (largest on ties).
      const int kmax = static_cast<int>(std::max<long long>(1, std::min<long long>(s.slices, (units * max_waves) / per)));
      double best = 1e30;
      for (int k = kmax; k >= 1; --k) {
        double idle = 0.0;
        for (int s0 = 0; s0 < s.slices; s0 += k) {
          const long long t = per * std::min(k, s.slices - s0);
          idle += static_cast<double>(cdiv(t, units) * units - t);
        }
        if (idle < best - 0.5) {
          best = idle;
          step_slices = k;
        }
      }
    }
    for (int s0 = 0; s0 < s.slices; s0 += step_slices) {
      ProblemSpec c = s;
      const int n = std::min(step_slices, s.slices - s0);
      c.slices = n;
      c.a.ptr = static_cast<const uint16_t*>(s.a.ptr) + static_cast<int64_t>(s0) * s.a.bs;
      c.a.n = n;
      c.b.ptr = static_cast<const uint16_t*>(s.b.ptr) + static_cast<int64_t>(s0) * s.b.bs;
      c.b.n = n;
      if (c.addend) c.addend = static_cast<const uint16_t*>(s.addend) + static_cast<int64_t>(s0) * s.add_bs;
      c.out = static_cast<uint16_t*>(s.out) + static_cast<int64_t>(s0) * s.out_bs;
      if (c.sumsq) c.sumsq = s.sumsq + s0;
      if (c.row_ss) c.row_ss = s.row_ss + static_cast<int64_t>(s0) * 2 * cdiv(s.N, BN) * s.M;
      chunks.push_back(c);
      chunk_cg.push_back(cg);
    }
  }
  // Consecutive chunks share a launch up to max_problems; beyond that only
  // while the whole launch stays within one wave of tiles (small problems,
  // where a launch costs more than its tiles and nothing drifts apart).
  size_t i = 0;
  while (i < chunks.size()) {
    std::vector<const ProblemSpec*> group;
    const int cg = chunk_cg[i];
    const long long units = cg == 2 ? std::max(1, pair_units) : std::max(1, sms);
    long long group_tiles = 0;
    for (; i < chunks.size() && static_cast<int>(group.size()) < MAX_PROBLEMS && chunk_cg[i] == cg; ++i) {
      const long long t = tiles_per_slice(chunks[i], cg) * chunks[i].slices;
      if (static_cast<int>(group.size()) >= max_problems && group_tiles + t > units) break;
      group.push_back(&chunks[i]);
      group_tiles += t;
    }
    const int tile_m = BM * cg, b_rows = BN / cg, step = BN / tile_m;
    launches.emplace_back();
    Launch& L = launches.back();
    L.cg = cg;
    GemmParams& P = L.P;
    std::memset(&P, 0, sizeof(P));
    P.err = err;
    P.timeout_ns = kWaitLimitNs;
    long long tiles = 0;
    int np = 0;
    for (const ProblemSpec* sp : group) {
      const ProblemSpec& s = *sp;
      GemmProblem& g = P.prob[np];
      g.M = s.M;
      g.N = s.N;
      g.K = s.K;
      g.slices = s.slices;
      g.mt = static_cast<int>(cdiv(s.M, tile_m));
      g.nt = static_cast<int>(cdiv(s.N, BN));
      g.kt = static_cast<int>(cdiv(s.K, cg == 2 ? GemmCfg<2>::KB : GemmCfg<1>::KB));
      g.tri = s.tri;
      g.mirror = s.mirror;
      g.a_sym = s.a_sym;
      g.b_sym = s.b_sym;
      if (s.tri) {
        int cnt = 0;
        for (int j = 0; j < g.nt; ++j) cnt += std::max(0, g.mt - step * j);
        g.tiles_per_slice = cnt;
      } else {
        g.tiles_per_slice = g.mt * g.nt;
      }
      g.tile_begin = static_cast<int>(tiles);
      // Raster bands: about sqrt(units * 256 / tile_m) row tiles (16 single, 8 paired).
      g.group_m = std::max(1, std::min(g.mt, raster_group > 0 ? raster_group : (cg == 2 ? 8 : 16)));
      g.a_mn = s.a_mn;
      g.b_mn = s.b_mn;
      g.idesc = mma_idesc_f16(s.in_f16 ? 0u : 1u, static_cast<uint32_t>(s.a_mn), static_cast<uint32_t>(s.b_mn),
                              static_cast<uint32_t>(tile_m), BN);
      g.alpha = s.alpha;
      g.beta = s.beta;
      g.gamma = s.gamma;
      g.f0 = s.f0;
      g.s_pow = s.s_pow;
      g.eps = s.eps;
      g.sumsq = s.sumsq;
      g.addend = s.addend;
      g.add_ld = s.add_ld;
      g.add_bs = s.add_bs;
      g.add_f16 = s.add_f16;
      g.out = s.out;
      g.out_ld = s.out_ld;
      g.out_bs = s.out_bs;
      g.out_f16 = s.out_f16;
      g.row_ss = s.row_ss;
      // A: K-major box 64 (K) x 128 rows; MN-major box 64 (M) x (K per stage) rows.
      // B: K-major box 64 x (256 / CTAs) rows; MN-major as A.
      const int kb_rows = cg == 2 ? GemmCfg<2>::KB : GemmCfg<1>::KB;
      if (!encode_map(&P.mapA[np], s.a, 64, s.a_mn ? kb_rows : BM)) return MUON_CUDA_ERROR;
      if (!encode_map(&P.mapB[np], s.b, 64, s.b_mn ? kb_rows : b_rows)) return MUON_CUDA_ERROR;
      // Output: 32 x 32 boxes, swizzled for the staging layout.
      const Mat c{s.out, s.M, s.N, s.out_ld, s.out_bs, s.slices, s.out_f16};
      if (!encode_map(&P.mapC[np], c, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return MUON_CUDA_ERROR;
      tiles += static_cast<long long>(g.tiles_per_slice) * s.slices;
      if (tiles > INT32_MAX) return MUON_BAD_SHAPE;
      ++np;
    }
    P.num_problems = np;
    P.total_tiles = static_cast<int>(tiles);
    // Split each tile's epilogue over two warps per lane quadrant where it
    // would not hide behind the next tile's main loop: short K (<= 2048) or
    // at most one wave of tiles (each CTA's epilogue is then on the critical
    // path).  Long-K launches keep one warp per quadrant (measured: splitting
    // them cost the power-capped Llama-8B call about 1%).
    bool short_k = false;
    for (int k = 0; k < np; ++k) short_k |= P.prob[k].K <= 2048;
    P.epi_split = (short_k || tiles <= units) ? 1 : 0;
  }
  // Programmatic dependent launch: each GEMM may start its prologue (barrier
  // setup, TMEM allocation) on idle SMs while the previous kernel drains; the
  // kernel waits for its predecessor before touching global memory.
  const bool pdl = pdl_enabled();
  for (const Launch& L : launches) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e;
    if (L.cg == 2) {
      const int units = std::max(1, std::min(L.P.total_tiles, pair_units));
      cfg.gridDim = dim3(static_cast<unsigned>(2 * units), 1, 1);
      cfg.dynamicSmemBytes = GemmCfg<2>::SMEM_BYTES;
      e = cudaLaunchKernelEx(&cfg, ns_gemm_pair_kernel, L.P);
    } else {
      cfg.gridDim = dim3(static_cast<unsigned>(std::min(L.P.total_tiles, sms)), 1, 1);
      cfg.dynamicSmemBytes = GemmCfg<1>::SMEM_BYTES;
      e = cudaLaunchKernelEx(&cfg, ns_gemm_kernel, L.P);
    }
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return MUON_CUDA_ERROR;
    }
    if (!launched()) return MUON_CUDA_ERROR;
  }
  return MUON_OK;
}

// ---------------------------------------------------------------- elementwise launches
void fill_seg_common(EwSeg& S, const muon_batch& b, long long& chunk, long long& slice, long long& row) {
  S.n = b.n;
  S.rows = b.rows;
  S.cols = b.cols;
  S.chunks_per_slice = cdiv(b.rows * b.cols, CHUNK);
  S.chunk_begin = chunk;
  S.slice_begin = slice;
  S.row_begin = row;
  chunk += b.n * S.chunks_per_slice;
  slice += b.n;
  row += b.n * b.rows;
}

int ew_grid(long long work, int sms) {
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<int>(std::max<long long>(1, std::min(work, cap)));
}

// Launches the per-chunk U^2 partials (mode 0 also does the momentum) and the
// per-slice finalization for one list of batches.  sumsq_ws_dev receives the
// sums of batches whose own sumsq pointer is null.
muon_status launch_norm(const muon_batch* bs, int nb, const muon_hparams* hp, int mode, float* partials,
                        float* sumsq_ws_dev, int sms, cudaStream_t stream) {
  int i = 0;
  while (i < nb) {
    EwParams P;
    std::memset(&P, 0, sizeof(P));
    long long chunk = 0, slice = 0, row = 0;
    int ns = 0;
    for (; i < nb && ns < MAX_SEGS; ++i) {
      const muon_batch& b = bs[i];
      if (batch_empty(b)) continue;
      EwSeg& S = P.seg[ns];
      fill_seg_common(S, b, chunk, slice, row);
      S.g = b.grad.ptr;
      S.g_ld = b.grad.ld;
      S.g_bs = b.grad.batch_stride;
      S.g_dt = b.grad.dtype == MUON_F32 ? 0 : 1;
      S.m = b.momentum.ptr;
      S.m_ld = b.momentum.ld;
      S.m_bs = b.momentum.batch_stride;
      S.m_dt = b.momentum.dtype == MUON_F32 ? 0 : 1;
      S.u = b.ns_in.ptr;
      S.u_ld = b.ns_in.ld;
      S.u_bs = b.ns_in.batch_stride;
      S.vec8 = mode == 0 ? vec8_ok(b, {&b.grad, &b.momentum, &b.ns_in}) : vec8_ok(b, {&b.ns_in});
      S.flat = mode == 0 ? flat_ok(b, {&b.grad, &b.momentum, &b.ns_in}) : flat_ok(b, {&b.ns_in});
      P.sumsq_out[ns] = b.sumsq;
      ++ns;
    }
    if (ns == 0) continue;
    P.nseg = ns;
    P.total_chunks = chunk;
    P.total_slices = slice;
    P.total_rows = row;
    P.mu = hp ? hp->mu : 0.0f;
    P.nesterov = hp ? hp->nesterov : 0;
    P.partials = partials;
    P.sumsq_ws = sumsq_ws_dev;
    const bool ok = mode == 0
                        ? launch_pdl(momentum_chunks_kernel<0>, dim3(ew_grid(chunk, sms)), dim3(EW_THREADS), 0,
                                     stream, P)
                        : launch_pdl(momentum_chunks_kernel<1>, dim3(ew_grid(chunk, sms)), dim3(EW_THREADS), 0,
                                     stream, P);
    if (!ok) return MUON_CUDA_ERROR;
    if (!launch_pdl(sumsq_finalize_kernel, dim3(ew_grid(cdiv(slice, EW_THREADS / 32), sms)), dim3(EW_THREADS), 0,
                    stream, P))
      return MUON_CUDA_ERROR;
    partials += chunk;
    sumsq_ws_dev += slice;
  }
  return MUON_OK;
}

// ---------------------------------------------------------------- Newton-Schulz planning
struct Coefs {
  float a, b, c;
};

Coefs coefs_at(const muon_hparams* hp, int it) {
  if (hp->abc_schedule) return Coefs{hp->abc_schedule[3 * it], hp->abc_schedule[3 * it + 1], hp->abc_schedule[3 * it + 2]};
  return Coefs{hp->a, hp->b, hp->c};
}

Mat view_mat(const muon_batch& b, const muon_view& v) {
  return Mat{v.ptr, b.rows, b.cols, v.ld, v.batch_stride, b.n, 0};
}

// ---------------------------------------------------------------- fused small-side Newton-Schulz
// Column split of an m x n slice over a cluster: C CTAs of w columns each
// (w a multiple of 64, at most SMALL_MAX_W; C at most SMALL_MAX_CLUSTER).
struct SmallSplit {
  int C, w;
};

// C is a power of two (so it divides every multiple of 8 rows of A): the
// smallest that keeps w <= SMALL_MAX_W, raised to 4 where the slice has that
// many 64-column blocks.  Clusters of 4 tile the device's SMs well (clusters
// of 8 leave a fifth of the B200's SMs idle); the split depends on the shape
// only, so a slice's sums never depend on the rest of the batch.
SmallSplit small_split(int64_t n) {
  const int blocks = static_cast<int>(cdiv(n, 64));
  auto pow2_at_least = [](int x) {
    int p = 1;
    while (p < x) p *= 2;
    return p;
  };
  int C = pow2_at_least(static_cast<int>(cdiv(blocks, SMALL_MAX_W / 64)));
  C = std::max(C, std::min(4, pow2_at_least(blocks)));
  return SmallSplit{C, 64 * static_cast<int>(cdiv(blocks, C))};
}

// How a wide slice (rows <= cols) with at most 128 rows runs the whole
// iteration in one clustered launch: with its columns resident in the
// cluster's shared memory when they fit on 4 CTAs (cols <= 2048), streamed
// through 4-CTA clusters otherwise (cols a multiple of 8, at most
// STREAM_MAX_N: the 4-CTA clusters fill the device, where 8-CTA resident
// clusters fit only 15 at once), resident on 8 CTAs for the remaining
// cols <= 4096; larger slices take the GEMM path.  Shape only, so a slice's
// result never depends on the batch.
enum class SmallPath { kGemm, kResident, kStream };

SmallPath small_path(int64_t rows, int64_t cols) {
  if (rows > cols || rows > SMALL_MAX_M || rows < 1) return SmallPath::kGemm;
  const SmallSplit sp = small_split(cols);
  if (sp.C <= 4 && sp.w <= SMALL_MAX_W) return SmallPath::kResident;
  if (cols % 8 == 0 && cols <= STREAM_MAX_N) return SmallPath::kStream;
  if (sp.C <= SMALL_MAX_CLUSTER && sp.w <= SMALL_MAX_W) return SmallPath::kResident;
  return SmallPath::kGemm;
}

bool small_shape_ok(int64_t rows, int64_t cols) { return small_path(rows, cols) != SmallPath::kGemm; }

// Cluster split of a fused slice: C CTAs of w columns (a multiple of 64).
SmallSplit fused_split(int64_t rows, int64_t cols) {
  if (small_path(rows, cols) == SmallPath::kStream)     // pairs of 64-column blocks per CTA
    return SmallSplit{STREAM_CLUSTER, 128 * static_cast<int>(cdiv(cdiv(cols, 128), STREAM_CLUSTER))};
  return small_split(cols);
}

// Slices whose short side is at most 128 run the whole iteration in one
// clustered launch when small_path allows (ns_small.cuh); tall ones
// (rows > cols) are transposed into the workspace first and back after.
// The choice depends on the shape only, so a slice's result never depends
// on the rest of the batch (tests can send them through the GEMM path,
// muon_testing_set_options).
bool small_eligible(const muon_batch& b) {
  if (g_opt.fused_small.load(std::memory_order_relaxed) == 0) return false;
  return b.rows > b.cols ? small_shape_ok(b.cols, b.rows) : small_shape_ok(b.rows, b.cols);
}

// Row sums of squares of a Newton-Schulz output from its tile partials
// ([n][nt][rows], summed in tile order) into the caller's row_sumsq.
muon_status launch_row_finalize(const float* part, int nt, int64_t rows, int64_t n, float* out, int sms,
                                cudaStream_t stream) {
  const bool ok = launch_pdl(row_partials_finalize_kernel, dim3(ew_grid(cdiv(n * rows, EW_THREADS), sms)),
                             dim3(EW_THREADS), 0, stream, part, nt, static_cast<long long>(rows),
                             static_cast<long long>(n), out);
  return ok ? MUON_OK : MUON_CUDA_ERROR;
}

// Row sums of squares read from the output itself (tall slices of the fused path).
muon_status launch_rows_sumsq(const muon_batch& b, int sms, cudaStream_t stream) {
  const int64_t bs = b.n > 1 ? b.ns_out.batch_stride : b.rows * b.ns_out.ld;
  const bool ok = launch_pdl(rows_sumsq_kernel, dim3(ew_grid(cdiv(b.n * b.rows, EW_THREADS / 32), sms)),
                             dim3(EW_THREADS), 0, stream, static_cast<const __nv_bfloat16*>(b.ns_out.ptr),
                             static_cast<long long>(b.ns_out.ld), static_cast<long long>(bs),
                             static_cast<long long>(b.rows), static_cast<long long>(b.cols),
                             static_cast<long long>(b.n), b.row_sumsq);
  return ok ? MUON_OK : MUON_CUDA_ERROR;
}

muon_status launch_small(const muon_batch& b, const muon_hparams* hp, const float* sumsq, int* err, bool gram,
                         float* row_partials, cudaStream_t stream) {
  const bool streamed = small_path(b.rows, b.cols) == SmallPath::kStream;
  const SmallSplit sp = fused_split(b.rows, b.cols);
  SmallParams P;
  std::memset(&P, 0, sizeof(P));
  P.row_ss = row_partials;
  P.restart = gram ? hp->gram_restart : 0;
  if (!encode_map(&P.map_in, view_mat(b, b.ns_in), 64, 128)) return MUON_CUDA_ERROR;
  if (!encode_map(&P.map_out, view_mat(b, b.ns_out), 64, 128)) return MUON_CUDA_ERROR;
  P.tma_store = (b.cols % 8 == 0) ? 1 : 0;
  P.out = static_cast<__nv_bfloat16*>(const_cast<void*>(b.ns_out.ptr));
  P.out_ld = b.ns_out.ld;
  P.out_bs = b.ns_out.batch_stride;
  P.sumsq = sumsq;
  P.eps = hp->ns_eps;
  P.m = static_cast<int>(b.rows);
  P.n = static_cast<int>(b.cols);
  P.w = sp.w;
  P.steps = hp->ns_steps;
  for (int k = 0; k < hp->ns_steps; ++k) {
    const Coefs cf = coefs_at(hp, k);
    P.a[k] = cf.a;
    P.b[k] = cf.b;
    P.c[k] = cf.c;
  }
  P.kappa = kGramScale;
  P.err = err;
  P.timeout_ns = kWaitLimitNs;
  constexpr int64_t kMaxGridY = 65535;
  for (int64_t s0 = 0; s0 < b.n; s0 += kMaxGridY) {
    P.slice0 = static_cast<int>(s0);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sp.C), static_cast<unsigned>(std::min(kMaxGridY, b.n - s0)), 1);
    cfg.blockDim = dim3(SMALL_THREADS, 1, 1);
    cfg.dynamicSmemBytes = streamed ? STREAM_SMEM_BYTES : SMALL_SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(sp.C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    auto kernel = streamed ? (gram ? ns_stream_gram_kernel : ns_stream_kernel)
                           : (gram ? ns_small_gram_kernel : ns_small_kernel);
    if (cudaLaunchKernelEx(&cfg, kernel, P) != cudaSuccess) {
      (void)cudaGetLastError();
      return MUON_CUDA_ERROR;
    }
    if (!launched()) return MUON_CUDA_ERROR;
  }
  return MUON_OK;
}

muon_status launch_transpose16(const void* in, int64_t in_ld, int64_t in_bs, void* out, int64_t out_ld,
                               int64_t out_bs, int64_t rows, int64_t cols, int64_t slices, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(cdiv(cols, 32)), static_cast<unsigned>(cdiv(rows, 32)),
                  static_cast<unsigned>(std::min<int64_t>(slices, 65535)));
  const bool ok = launch_pdl(transpose16_kernel, grid, dim3(32, 8, 1), 0, stream, static_cast<const uint16_t*>(in),
                             static_cast<long long>(in_ld), static_cast<long long>(in_bs), static_cast<uint16_t*>(out),
                             static_cast<long long>(out_ld), static_cast<long long>(out_bs), static_cast<int>(rows),
                             static_cast<int>(cols), static_cast<int>(slices));
  return ok ? MUON_OK : MUON_CUDA_ERROR;
}

// The fused kernel on one batch; a tall batch goes through its transposed
// copy in the workspace (the kernel then works in place on that copy: each
// CTA reads its columns before writing them back).
muon_status run_small(const muon_batch& b, const NsBatchWs& w, uint8_t* ws, const muon_hparams* hp,
                      const float* sumsq, int* err, bool gram, int sms, cudaStream_t stream) {
  if (b.rows <= b.cols) {
    float* part = b.row_sumsq ? reinterpret_cast<float*>(ws + w.rs_off) : nullptr;
    muon_status st = launch_small(b, hp, sumsq, err, gram, part, stream);
    if (st != MUON_OK || part == nullptr) return st;
    return launch_row_finalize(part, 2 * fused_split(b.rows, b.cols).C, b.rows, b.n, b.row_sumsq, sms, stream);
  }
  void* T = ws + w.t_off;
  const int64_t in_bs = b.n > 1 ? b.ns_in.batch_stride : b.rows * b.ns_in.ld;
  const int64_t out_bs = b.n > 1 ? b.ns_out.batch_stride : b.rows * b.ns_out.ld;
  muon_status st = launch_transpose16(b.ns_in.ptr, b.ns_in.ld, in_bs, T, w.ldt, w.bst, b.rows, b.cols, b.n, stream);
  if (st != MUON_OK) return st;
  muon_batch v = b;
  v.rows = b.cols;
  v.cols = b.rows;
  v.ns_in = muon_view{T, w.ldt, w.bst, MUON_BF16, 0};
  v.ns_out = v.ns_in;
  if ((st = launch_small(v, hp, sumsq, err, gram, nullptr, stream)) != MUON_OK) return st;
  if ((st = launch_transpose16(T, w.ldt, w.bst, const_cast<void*>(b.ns_out.ptr), b.ns_out.ld, out_bs, b.cols, b.rows,
                               b.n, stream)) != MUON_OK)
    return st;
  // The kernel's rows were the slice's columns: the output rows' sums are read back from ns_out.
  return b.row_sumsq ? launch_rows_sumsq(b, sms, stream) : MUON_OK;
}

// SYRK of the slice storage X ([rows][cols]) on the short side: out = f * X X^T (rows <= cols)
// or f * X^T X (rows > cols), lower triangle + mirror.
ProblemSpec syrk_spec(const muon_batch& b, const Mat& x, void* out, int64_t ldm, int64_t bsm, int out_f16, float f0,
                      int s_pow, const float* sumsq, float eps) {
  const bool T = b.rows > b.cols;
  const int m = static_cast<int>(std::min(b.rows, b.cols)), n = static_cast<int>(std::max(b.rows, b.cols));
  ProblemSpec s{};
  s.M = m;
  s.N = m;
  s.K = n;
  s.slices = static_cast<int>(b.n);
  s.tri = 1;
  s.a = x;
  s.a_mn = T ? 1 : 0;
  s.b = x;
  s.b_mn = T ? 1 : 0;
  s.in_f16 = x.f16;
  s.alpha = 1.0f;
  s.f0 = f0;
  s.s_pow = s_pow;
  s.eps = eps;
  s.sumsq = sumsq;
  s.out = out;
  s.out_ld = ldm;
  s.out_bs = bsm;
  s.out_f16 = out_f16;
  s.mirror = sym_compact(m) ? 0 : 1;
  return s;
}

// Symmetric m x m product out = f * (alpha * P S + beta * D) + gamma I (lower triangle,
// mirrored when m < 256); both factors are symmetric and read as such.
ProblemSpec sym_spec(int m, int slices, const Mat& p, const Mat& q, void* out, int64_t ldm, int64_t bsm, int out_f16,
                     float alpha, float beta, const void* add, int add_f16, float gamma) {
  ProblemSpec s{};
  s.M = m;
  s.N = m;
  s.K = m;
  s.slices = slices;
  s.tri = 1;
  s.a = p;
  s.a_mn = 0;
  s.b = q;
  s.b_mn = 0;
  s.in_f16 = p.f16;
  s.alpha = alpha;
  s.beta = beta;
  s.gamma = gamma;
  s.f0 = 1.0f;
  s.addend = add;
  s.add_ld = ldm;
  s.add_bs = bsm;
  s.add_f16 = add_f16;
  s.out = out;
  s.out_ld = ldm;
  s.out_bs = bsm;
  s.out_f16 = out_f16;
  s.mirror = sym_compact(m) ? 0 : 1;
  s.a_sym = s.b_sym = sym_compact(m) ? 1 : 0;
  return s;
}

// Applies the symmetric m x m factor F (bf16) to the slice storage X on the
// short side: out = f * (F X + beta X) when rows <= cols, or
// out = f * (X F + beta X) in the transposed case; out has X's layout.
ProblemSpec apply_spec(const muon_batch& b, const Mat& f, const Mat& x, void* out, int64_t out_ld, int64_t out_bs,
                       float beta, int s_pow, const float* sumsq, float eps, float* row_ss) {
  const bool T = b.rows > b.cols;
  const int m = static_cast<int>(std::min(b.rows, b.cols));
  ProblemSpec s{};
  s.slices = static_cast<int>(b.n);
  s.tri = 0;
  s.in_f16 = 0;
  if (!T) {
    s.M = m;
    s.N = static_cast<int>(b.cols);
    s.K = m;
    s.a = f;
    s.a_mn = 0;
    s.a_sym = sym_compact(m) ? 1 : 0;
    s.b = x;
    s.b_mn = 1;
  } else {
    s.M = static_cast<int>(b.rows);
    s.N = m;
    s.K = m;
    s.a = x;
    s.a_mn = 0;
    s.b = f;
    s.b_mn = 0;
    s.b_sym = sym_compact(m) ? 1 : 0;
  }
  s.alpha = 1.0f;
  s.beta = beta;
  s.f0 = 1.0f;
  s.s_pow = s_pow;
  s.eps = eps;
  s.sumsq = sumsq;
  s.addend = beta != 0.0f ? x.ptr : nullptr;
  s.add_ld = x.ld;
  s.add_bs = x.bs;
  s.add_f16 = 0;
  s.out = out;
  s.out_ld = out_ld;
  s.out_bs = out_bs;
  s.out_f16 = 0;
  s.row_ss = row_ss;
  return s;
}

// Byte range [first, last) a view of batch b spans.
struct ByteRange {
  uintptr_t first, last;
};
ByteRange view_range(const muon_batch& b, const muon_view& v) {
  const int64_t span = (b.n - 1) * v.batch_stride + (b.rows - 1) * v.ld + b.cols;
  const uintptr_t p = reinterpret_cast<uintptr_t>(v.ptr);
  return ByteRange{p, p + static_cast<uintptr_t>(span) * static_cast<uintptr_t>(esize(v.dtype))};
}
inline bool overlaps(const ByteRange& a, const ByteRange& b) { return a.first < b.last && b.first < a.last; }

muon_status validate_ns(const muon_batch* bs, int nb, const muon_hparams* hp) {
  if (nb < 0 || (nb > 0 && bs == nullptr)) return MUON_INVALID_ARG;
  muon_status st = check_hp(hp);
  if (st != MUON_OK) return st;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = bs[i];
    if ((st = check_shape(b)) != MUON_OK) return st;
    if (batch_empty(b)) continue;
    if ((st = check_view(b, b.ns_in, {MUON_BF16}, true)) != MUON_OK) return st;
    if ((st = check_view(b, b.ns_out, {MUON_BF16}, true)) != MUON_OK) return st;
  }
  // The iteration reads ns_in while it writes ns_out (and, on the fused
  // path, keeps its intermediate iterates there): no output may share a byte
  // with any input or with another batch's output of the call.
  for (int i = 0; i < nb; ++i) {
    if (batch_empty(bs[i])) continue;
    const ByteRange out = view_range(bs[i], bs[i].ns_out);
    for (int j = 0; j < nb; ++j) {
      if (batch_empty(bs[j])) continue;
      if (overlaps(out, view_range(bs[j], bs[j].ns_in))) return MUON_INVALID_ARG;
      if (j > i && overlaps(out, view_range(bs[j], bs[j].ns_out))) return MUON_INVALID_ARG;
    }
  }
  return MUON_OK;
}

// Clears the error word and makes sure every batch has a per-slice sum of squares.
// Returns the per-batch sumsq pointers to use.
muon_status prepare_norms(const muon_batch* bs, int nb, const Layout& L, uint8_t* ws, int sms, cudaStream_t stream,
                          std::vector<const float*>& sumsq, bool clear_err = true) {
  if (clear_err && !clear_error_word(ws, stream)) return MUON_CUDA_ERROR;
  sumsq.assign(nb, nullptr);
  std::vector<muon_batch> missing;
  float* base = reinterpret_cast<float*>(ws + L.sumsq);
  float* cur = base;
  for (int i = 0; i < nb; ++i) {
    if (batch_empty(bs[i])) continue;
    if (bs[i].sumsq) {
      sumsq[i] = bs[i].sumsq;
    } else {
      muon_batch c = bs[i];
      c.sumsq = nullptr;
      missing.push_back(c);
      sumsq[i] = cur;
      cur += bs[i].n;
    }
  }
  if (!missing.empty())
    return launch_norm(missing.data(), static_cast<int>(missing.size()), nullptr, 1,
                       reinterpret_cast<float*>(ws + L.partials), base, sms, stream);
  return MUON_OK;
}

}  // namespace

// Scratch of muon_momentum_norm_noalloc: per-chunk partial sums in static
// device memory, so that entry point allocates nothing.  Host code must not
// pass the symbol itself to a kernel (on the host it names a shadow
// variable); it passes the device address looked up per device below.
static __device__ __align__(256) float g_noalloc_partials[MUON_NOALLOC_SCRATCH_FLOATS];

namespace {
std::mutex g_noalloc_mu;
float* g_noalloc_addr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};

// Device address of g_noalloc_partials on the current device, looked up once
// per device (and again if the device's context was re-created, which can
// load the module at another address) with that device current.
muon_status noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUON_CUDA_ERROR;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  const unsigned long long ctx = current_ctx_id();
  if (!g_noalloc_addr[dev] || (ctx != 0 && ctx != g_noalloc_ctx[dev])) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return MUON_CUDA_ERROR;
    }
    g_noalloc_addr[dev] = static_cast<float*>(p);
    g_noalloc_ctx[dev] = current_ctx_id();
  }
  *out = g_noalloc_addr[dev];
  return MUON_OK;
}
}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char* muon_version(void) { return "0.1.0"; }

muon_status muon_polar_express_schedule(double lower, int steps, double safety, float* abc_out, double* err_out) {
  namespace pe = muon::polar_express;
  if (abc_out == nullptr || !(lower > 0.0 && lower < 1.0) || steps < 1 || steps > 16 || !(safety >= 1.0) ||
      !(safety <= 2.0))
    return MUON_INVALID_ARG;
  float abc[3 * 16];
  double errs[16];
  double lo = lower, hi = 1.0;
  for (int t = 0; t < steps; ++t) {
    pe::Quintic p;
    double E = 0.0;
    if (!pe::minimax_quintic(lo, hi, &p, &E)) return MUON_BAD_SHAPE;
    const double s = safety;
    const pe::Quintic q{p.a / s, p.b / (s * s * s), p.c / (s * s * s * s * s)};
    double mn = 0.0, mx = 0.0;
    pe::image(q, lo, hi, &mn, &mx);
    if (!(mn > 0.0) || !std::isfinite(mx)) return MUON_BAD_SHAPE;
    abc[3 * t] = static_cast<float>(q.a);
    abc[3 * t + 1] = static_cast<float>(q.b);
    abc[3 * t + 2] = static_cast<float>(q.c);
    errs[t] = std::max(std::fabs(1.0 - mn), std::fabs(mx - 1.0));
    lo = mn;
    hi = mx;
  }
  std::memcpy(abc_out, abc, sizeof(float) * 3 * steps);
  if (err_out) std::memcpy(err_out, errs, sizeof(double) * steps);
  return MUON_OK;
}

uint64_t muon_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

muon_status muon_update_scale(int64_t fan_out, int64_t fan_in, int32_t scale_mode, float extra, float* scale_out) {
  if (scale_out == nullptr) return MUON_INVALID_ARG;
  float v = 0.0f;
  if (!update_scale(fan_out, fan_in, scale_mode, extra, &v)) return MUON_INVALID_ARG;
  *scale_out = v;
  return MUON_OK;
}

muon_status muon_testing_set_options(const muon_testing_options* opts, muon_testing_options* previous) {
  muon_testing_options cur;
  cur.fused_small = g_opt.fused_small.load();
  cur.max_waves = g_opt.max_waves.load();
  cur.max_problems = g_opt.max_problems.load();
  cur.pdl = g_opt.pdl.load();
  cur.overlap = g_opt.overlap.load();
  if (opts) {
    if ((opts->fused_small != 0 && opts->fused_small != 1) || opts->max_waves < 0 || opts->max_waves > 1000000 ||
        opts->max_problems < 1 || opts->max_problems > MAX_PROBLEMS || (opts->pdl != 0 && opts->pdl != 1) ||
        (opts->overlap != 0 && opts->overlap != 1))
      return MUON_INVALID_ARG;
  }
  if (previous) *previous = cur;
  if (opts) {
    g_opt.fused_small.store(opts->fused_small);
    g_opt.max_waves.store(opts->max_waves);
    g_opt.max_problems.store(opts->max_problems);
    g_opt.pdl.store(opts->pdl);
    g_opt.overlap.store(opts->overlap);
  }
  return MUON_OK;
}

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "ok";
    case MUON_INVALID_ARG: return "invalid argument";
    case MUON_BAD_SHAPE: return "bad shape or strides";
    case MUON_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case MUON_MISALIGNED: return "misaligned pointer or stride (16-byte TMA rule, 256-byte workspace rule)";
    case MUON_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MUON_CUDA_ERROR: return "CUDA error";
    case MUON_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
  }
  return "unknown status";
}

size_t muon_workspace_size(const muon_batch* batches, int nb, int which) {
  if (nb < 0 || (nb > 0 && !batches) || which < -1 || which > 3) return 0;
  for (int i = 0; i < nb; ++i)
    if (check_shape(batches[i]) != MUON_OK) return 0;
  if (which == -1) {
    size_t m = 0;
    for (int w = 0; w < 4; ++w) m = std::max(m, plan_layout(batches, nb, w).total);
    return m;
  }
  return plan_layout(batches, nb, which).total;
}

muon_status muon_workspace_error(const void* workspace, cudaStream_t stream, int32_t* error_word) {
  if (!workspace || !error_word) return MUON_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MUON_CUDA_ERROR;
  if (cudaMemcpy(error_word, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_CUDA_ERROR;
  return MUON_OK;
}

muon_status muon_momentum_norm(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream) {
  if (nb < 0 || (nb > 0 && !batches)) return MUON_INVALID_ARG;
  muon_status st = check_hp(hp);
  if (st != MUON_OK) return st;
  bool any = false;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = batches[i];
    if ((st = check_shape(b)) != MUON_OK) return st;
    if (batch_empty(b)) continue;
    any = true;
    if ((st = check_view(b, b.grad, {MUON_F32, MUON_BF16}, false)) != MUON_OK) return st;
    if ((st = check_view(b, b.momentum, {MUON_F32, MUON_BF16}, false)) != MUON_OK) return st;
    if ((st = check_view(b, b.ns_in, {MUON_BF16}, false)) != MUON_OK) return st;
    if (!b.sumsq) return MUON_INVALID_ARG;
  }
  if (!any) return MUON_OK;
  const Layout L = plan_layout(batches, nb, 0);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != MUON_OK) return st;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return launch_norm(batches, nb, hp, 0, reinterpret_cast<float*>(ws + L.partials),
                     reinterpret_cast<float*>(ws + L.sumsq), sms, stream);
}

muon_status muon_momentum_norm_noalloc(const muon_batch* batches, int nb, const muon_hparams* hp,
                                       cudaStream_t stream) {
  if (nb < 0 || (nb > 0 && !batches)) return MUON_INVALID_ARG;
  muon_status st = check_hp(hp);
  if (st != MUON_OK) return st;
  bool any = false;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = batches[i];
    if ((st = check_shape(b)) != MUON_OK) return st;
    if (batch_empty(b)) continue;
    any = true;
    if ((st = check_view(b, b.grad, {MUON_F32, MUON_BF16}, false)) != MUON_OK) return st;
    if ((st = check_view(b, b.momentum, {MUON_F32, MUON_BF16}, false)) != MUON_OK) return st;
    if ((st = check_view(b, b.ns_in, {MUON_BF16}, false)) != MUON_OK) return st;
    if (!b.sumsq) return MUON_INVALID_ARG;
  }
  if (!any) return MUON_OK;
  const Layout L = plan_layout(batches, nb, 0);
  if (L.total_chunks > MUON_NOALLOC_SCRATCH_FLOATS) return MUON_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  float* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != MUON_OK) return st;
  // Every batch carries its own sumsq, so the finalize step never writes the
  // fallback array; it is given the scratch only as a valid pointer.
  return launch_norm(batches, nb, hp, 0, scratch, scratch, sms, stream);
}

muon_status ns_standard_impl(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream, bool clear_err);
muon_status ns_gram_impl(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream, bool clear_err);

muon_status muon_ns_batched(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  return ns_standard_impl(batches, nb, hp, workspace, workspace_bytes, stream, true);
}

muon_status muon_gram_ns_batched(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  return ns_gram_impl(batches, nb, hp, workspace, workspace_bytes, stream, true);
}

}  // extern "C"

// Row sums of squares of the GEMM path's outputs from the last product's tile partials.
muon_status finalize_gemm_row_sums(const muon_batch* batches, int nb, const Layout& L, uint8_t* ws,
                                   const std::vector<char>& fused, int sms, cudaStream_t stream) {
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = batches[i];
    if (batch_empty(b) || fused[i] || !b.row_sumsq) continue;
    const muon_status st = launch_row_finalize(reinterpret_cast<const float*>(ws + L.nsb[i].rs_off),
                                               static_cast<int>(2 * cdiv(b.cols, BN)), b.rows, b.n, b.row_sumsq, sms,
                                               stream);
    if (st != MUON_OK) return st;
  }
  return MUON_OK;
}

// Marks the batches that take the fused small-side kernels and enqueues
// them: on a second stream when the call also has GEMM-path batches (and
// the overlap switch is on), else on the call's stream.
muon_status start_fused(const muon_batch* batches, int nb, const Layout& L, uint8_t* ws, const muon_hparams* hp,
                        const std::vector<const float*>& sumsq, int* err, bool gram, int sms, cudaStream_t stream,
                        std::vector<char>& fused, SideFork& side, cudaStream_t& fstream) {
  fused.assign(nb, 0);
  bool any_fused = false, any_gemm = false;
  for (int i = 0; i < nb; ++i) {
    if (batch_empty(batches[i])) continue;
    fused[i] = small_eligible(batches[i]) ? 1 : 0;
    if (fused[i]) any_fused = true;
    else any_gemm = true;
  }
  const bool fork = any_fused && any_gemm && g_opt.overlap.load(std::memory_order_relaxed) != 0;
  muon_status st = side.open(stream, fork, &fstream);
  for (int i = 0; i < nb && st == MUON_OK; ++i)
    if (fused[i]) st = run_small(batches[i], L.nsb[i], ws, hp, sumsq[i], err, gram, sms, fstream);
  return st;
}

muon_status ns_standard_impl(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream, bool clear_err) {
  muon_status st = validate_ns(batches, nb, hp);
  if (st != MUON_OK) return st;
  bool any = false;
  for (int i = 0; i < nb; ++i) any |= !batch_empty(batches[i]);
  if (!any) return MUON_OK;
  const Layout L = plan_layout(batches, nb, 1);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != MUON_OK) return st;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  std::vector<const float*> sumsq;
  if ((st = prepare_norms(batches, nb, L, ws, sms, stream, sumsq, clear_err)) != MUON_OK) return st;
  int* err = reinterpret_cast<int*>(ws);

  std::vector<char> fused;
  SideFork side;
  cudaStream_t fstream = stream;
  if ((st = start_fused(batches, nb, L, ws, hp, sumsq, err, false, sms, stream, fused, side, fstream)) != MUON_OK)
    return st;
  const int S = hp->ns_steps;
  for (int it = 0; it < S; ++it) {
    const Coefs cf = coefs_at(hp, it);
    std::vector<ProblemSpec> syrk, poly, apply;
    for (int i = 0; i < nb; ++i) {
      const muon_batch& b = batches[i];
      if (batch_empty(b) || fused[i]) continue;
      const NsBatchWs& w = L.nsb[i];
      const int m = static_cast<int>(std::min(b.rows, b.cols));
      void* Abuf = ws + w.off[0];
      void* Bbuf = ws + w.off[1];
      void* Xws = ws + w.off[2];
      // Writes alternate between ns_out and the X workspace so the last lands in ns_out.
      auto buf = [&](int k) -> Mat {
        if (k < 0) return view_mat(b, b.ns_in);
        if ((S - 1 - k) % 2 == 0) return view_mat(b, b.ns_out);
        return Mat{Xws, b.rows, b.cols, w.ldx, w.bsx, b.n, 0};
      };
      const Mat src = buf(it - 1), dst = buf(it);
      const Mat Am{Abuf, m, m, w.ldm, w.bsm, b.n, 0};
      const Mat Bm{Bbuf, m, m, w.ldm, w.bsm, b.n, 0};
      syrk.push_back(syrk_spec(b, src, Abuf, w.ldm, w.bsm, 0, 1.0f, it == 0 ? 2 : 0, sumsq[i], hp->ns_eps));
      poly.push_back(sym_spec(m, static_cast<int>(b.n), Am, Am, Bbuf, w.ldm, w.bsm, 0, cf.c, cf.b, Abuf, 0, 0.0f));
      float* rs = (it == S - 1 && b.row_sumsq) ? reinterpret_cast<float*>(ws + w.rs_off) : nullptr;
      apply.push_back(apply_spec(b, Bm, src, const_cast<void*>(dst.ptr), dst.ld, dst.bs, cf.a, it == 0 ? 1 : 0,
                                 sumsq[i], hp->ns_eps, rs));
    }
    if ((st = launch_gemms(syrk, sms, err, stream)) != MUON_OK) return st;
    if ((st = launch_gemms(poly, sms, err, stream)) != MUON_OK) return st;
    if ((st = launch_gemms(apply, sms, err, stream)) != MUON_OK) return st;
  }
  if ((st = finalize_gemm_row_sums(batches, nb, L, ws, fused, sms, stream)) != MUON_OK) return st;
  return side.close();
}

muon_status ns_gram_impl(const muon_batch* batches, int nb, const muon_hparams* hp, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream, bool clear_err) {
  muon_status st = validate_ns(batches, nb, hp);
  if (st != MUON_OK) return st;
  bool any = false;
  for (int i = 0; i < nb; ++i) any |= !batch_empty(batches[i]);
  if (!any) return MUON_OK;
  const Layout L = plan_layout(batches, nb, 2);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != MUON_OK) return st;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  std::vector<const float*> sumsq;
  if ((st = prepare_norms(batches, nb, L, ws, sms, stream, sumsq, clear_err)) != MUON_OK) return st;
  int* err = reinterpret_cast<int*>(ws);
  const int S = hp->ns_steps;
  const float kap = kGramScale;

  std::vector<char> fused;
  SideFork side;
  cudaStream_t fstream = stream;
  if ((st = start_fused(batches, nb, L, ws, hp, sumsq, err, true, sms, stream, fused, side, fstream)) != MUON_OK)
    return st;
  // G: kappa * s^2 * X X^T (short side) in fp16.
  {
    std::vector<ProblemSpec> g;
    for (int i = 0; i < nb; ++i) {
      const muon_batch& b = batches[i];
      if (batch_empty(b) || fused[i]) continue;
      const NsBatchWs& w = L.nsb[i];
      g.push_back(syrk_spec(b, view_mat(b, b.ns_in), ws + w.off[0], w.ldm, w.bsm, 1, kap, 2, sumsq[i], hp->ns_eps));
    }
    if ((st = launch_gemms(g, sms, err, stream)) != MUON_OK) return st;
  }
  // Restarts: before iterations R, 2R, ... (R = gram_restart) the iterate
  // X = f Q X_prev is formed in bf16 (f = s while X_prev is the unnormalized
  // input) and the iteration starts again from it: A = kappa X X^T, Q = I.
  // Writes of X alternate between the X workspace and ns_out so that the
  // final O = f Q X lands in ns_out; ns_in is only read.
  const int R = hp->gram_restart;
  auto restart_at = [&](int k) { return R > 0 && k > 0 && k < S && k % R == 0; };
  const int restarts = R > 0 ? (S - 1) / R : 0;
  int xwrites = 0;                     // X-sized outputs written so far (restarts, then O)
  const int xtotal = restarts + 1;
  auto x_dst_is_out = [&](int j) { return (xtotal - 1 - j) % 2 == 0; };
  // Buffers: 0 Ah (kappa*A), 1 P, 2 Qa, 3 Qb, 4 R, 5 X.  At the start of a
  // segment P is written straight into the current Q buffer (Q = P).
  int qcur = 2;
  int seg_start = 0;
  for (int k = 0; k < S; ++k) {
    const Coefs cf = coefs_at(hp, k);
    const bool last = (k == S - 1);
    const bool end = last || restart_at(k + 1);   // last iteration of its segment: Q goes into an X product
    if (restart_at(k)) {
      std::vector<ProblemSpec> xs, gs;
      for (int i = 0; i < nb; ++i) {
        const muon_batch& b = batches[i];
        if (batch_empty(b) || fused[i]) continue;
        const NsBatchWs& w = L.nsb[i];
        const int m = static_cast<int>(std::min(b.rows, b.cols));
        const Mat Q{ws + w.off[qcur], m, m, w.ldm, w.bsm, b.n, 0};
        const Mat xws{ws + w.off[5], b.rows, b.cols, w.ldx, w.bsx, b.n, 0};
        const Mat src = xwrites == 0 ? view_mat(b, b.ns_in) : (x_dst_is_out(xwrites - 1) ? view_mat(b, b.ns_out) : xws);
        const Mat dst = x_dst_is_out(xwrites) ? view_mat(b, b.ns_out) : xws;
        xs.push_back(apply_spec(b, Q, src, const_cast<void*>(dst.ptr), dst.ld, dst.bs, 0.0f, xwrites == 0 ? 1 : 0,
                                sumsq[i], hp->ns_eps, nullptr));
        gs.push_back(syrk_spec(b, dst, ws + w.off[0], w.ldm, w.bsm, 1, kap, 0, sumsq[i], hp->ns_eps));
      }
      if ((st = launch_gemms(xs, sms, err, stream)) != MUON_OK) return st;
      if ((st = launch_gemms(gs, sms, err, stream)) != MUON_OK) return st;
      ++xwrites;
      seg_start = k;
    }
    const bool first = (k == seg_start);
    std::vector<ProblemSpec> t_l, qr_l, a_l;
    int qnext = qcur;
    for (int i = 0; i < nb; ++i) {
      const muon_batch& b = batches[i];
      if (batch_empty(b) || fused[i]) continue;
      const NsBatchWs& w = L.nsb[i];
      const int m = static_cast<int>(std::min(b.rows, b.cols));
      const int sl = static_cast<int>(b.n);
      auto M16 = [&](int idx, int f16) { return Mat{ws + w.off[idx], m, m, w.ldm, w.bsm, b.n, f16}; };
      const int pidx = first ? qcur : 1;
      // P = a I + (b/kappa) Ah + (c/kappa^2) Ah^2 ; bf16 when it is the segment's final Q.
      const int p_f16 = (first && end) ? 0 : 1;
      t_l.push_back(sym_spec(m, sl, M16(0, 1), M16(0, 1), ws + w.off[pidx], w.ldm, w.bsm, p_f16, cf.c / (kap * kap),
                             cf.b / kap, ws + w.off[0], 1, cf.a));
      if (!first) {
        qnext = (qcur == 2) ? 3 : 2;
        qr_l.push_back(sym_spec(m, sl, M16(1, 1), M16(qcur, 1), ws + w.off[qnext], w.ldm, w.bsm, end ? 0 : 1, 1.0f,
                                0.0f, nullptr, 1, 0.0f));
      }
      if (!end) {
        qr_l.push_back(sym_spec(m, sl, M16(pidx, 1), M16(0, 1), ws + w.off[4], w.ldm, w.bsm, 1, 1.0f, 0.0f, nullptr,
                                1, 0.0f));
        a_l.push_back(sym_spec(m, sl, M16(pidx, 1), M16(4, 1), ws + w.off[0], w.ldm, w.bsm, 1, 1.0f, 0.0f, nullptr,
                               1, 0.0f));
      }
    }
    if ((st = launch_gemms(t_l, sms, err, stream)) != MUON_OK) return st;
    if ((st = launch_gemms(qr_l, sms, err, stream)) != MUON_OK) return st;
    if ((st = launch_gemms(a_l, sms, err, stream)) != MUON_OK) return st;
    qcur = qnext;
  }
  // O = f Q X on the short side, Q in bf16 (f = s when no restart happened).
  {
    std::vector<ProblemSpec> o;
    for (int i = 0; i < nb; ++i) {
      const muon_batch& b = batches[i];
      if (batch_empty(b) || fused[i]) continue;
      const NsBatchWs& w = L.nsb[i];
      const int m = static_cast<int>(std::min(b.rows, b.cols));
      const Mat Q{ws + w.off[qcur], m, m, w.ldm, w.bsm, b.n, 0};
      const Mat xws{ws + w.off[5], b.rows, b.cols, w.ldx, w.bsx, b.n, 0};
      const Mat src = xwrites == 0 ? view_mat(b, b.ns_in) : (x_dst_is_out(xwrites - 1) ? view_mat(b, b.ns_out) : xws);
      const Mat out = view_mat(b, b.ns_out);
      float* rs = b.row_sumsq ? reinterpret_cast<float*>(ws + w.rs_off) : nullptr;
      o.push_back(apply_spec(b, Q, src, const_cast<void*>(out.ptr), out.ld, out.bs, 0.0f, xwrites == 0 ? 1 : 0,
                             sumsq[i], hp->ns_eps, rs));
    }
    if ((st = launch_gemms(o, sms, err, stream)) != MUON_OK) return st;
  }
  if ((st = finalize_gemm_row_sums(batches, nb, L, ws, fused, sms, stream)) != MUON_OK) return st;
  return side.close();
}

extern "C" {

muon_status muon_ns_auto_batched(const muon_batch* batches, int nb, const muon_hparams* hp, float gram_min_ratio,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  muon_status st = validate_ns(batches, nb, hp);
  if (st != MUON_OK) return st;
  if (!std::isfinite(gram_min_ratio)) return MUON_INVALID_ARG;
  std::vector<muon_batch> std_b, gram_b;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = batches[i];
    if (batch_empty(b)) continue;
    const int64_t m = std::min(b.rows, b.cols), n = std::max(b.rows, b.cols);
    const bool gram = n > m && static_cast<double>(n) >= static_cast<double>(gram_min_ratio) * static_cast<double>(m);
    (gram ? gram_b : std_b).push_back(b);
  }
  const size_t need = std::max(plan_layout(std_b.data(), static_cast<int>(std_b.size()), 1).total,
                               plan_layout(gram_b.data(), static_cast<int>(gram_b.size()), 2).total);
  if (!std_b.empty() || !gram_b.empty())
    if ((st = check_ws(workspace, workspace_bytes, need)) != MUON_OK) return st;
  // One error word for the whole call: cleared once, kept across both forms.
  if (!clear_error_word(workspace, stream)) return MUON_CUDA_ERROR;
  if (!std_b.empty() && (st = ns_standard_impl(std_b.data(), static_cast<int>(std_b.size()), hp, workspace,
                                               workspace_bytes, stream, false)) != MUON_OK)
    return st;
  if (!gram_b.empty())
    return ns_gram_impl(gram_b.data(), static_cast<int>(gram_b.size()), hp, workspace, workspace_bytes, stream,
                        false);
  return MUON_OK;
}

muon_status normuon_update(const muon_batch* batches, int nb, const muon_hparams* hp, int use_normuon,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (nb < 0 || (nb > 0 && !batches)) return MUON_INVALID_ARG;
  muon_status st = check_hp(hp);
  if (st != MUON_OK) return st;
  bool any = false;
  for (int i = 0; i < nb; ++i) {
    const muon_batch& b = batches[i];
    if ((st = check_shape(b)) != MUON_OK) return st;
    if (batch_empty(b)) continue;
    any = true;
    if ((st = check_view(b, b.ns_out, {MUON_BF16}, false)) != MUON_OK) return st;
    if ((st = check_view(b, b.weight, {MUON_F32, MUON_BF16}, false)) != MUON_OK) return st;
    if (b.weight_copy.ptr && (st = check_view(b, b.weight_copy, {MUON_BF16}, false)) != MUON_OK) return st;
    if (use_normuon && !b.variance) return MUON_INVALID_ARG;
    float scale = 0.0f;
    if (!update_scale(b.fan_out, b.fan_in, hp->scale_mode, hp->extra_scale_factor, &scale)) return MUON_INVALID_ARG;
  }
  if (!any) return MUON_OK;
  const Layout L = plan_layout(batches, nb, 3);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != MUON_OK) return st;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* row_ss = reinterpret_cast<float*>(ws + L.row_ss);
  float* row_d = reinterpret_cast<float*>(ws + L.row_d);
  float* factor = reinterpret_cast<float*>(ws + L.factor);
  int i = 0;
  while (i < nb) {
    EwParams P;
    std::memset(&P, 0, sizeof(P));
    long long chunk = 0, slice = 0, row = 0;
    int ns = 0;
    bool any_rsq = false, any_o = false;   // segments with row sums from the NS call / without
    for (; i < nb && ns < MAX_SEGS; ++i) {
      const muon_batch& b = batches[i];
      if (batch_empty(b)) continue;
      EwSeg& S = P.seg[ns];
      fill_seg_common(S, b, chunk, slice, row);
      S.o = b.ns_out.ptr;
      S.o_ld = b.ns_out.ld;
      S.o_bs = b.ns_out.batch_stride;
      S.w = b.weight.ptr;
      S.w_ld = b.weight.ld;
      S.w_bs = b.weight.batch_stride;
      S.w_dt = b.weight.dtype == MUON_F32 ? 0 : 1;
      S.wc = b.weight_copy.ptr;
      S.wc_ld = b.weight_copy.ld;
      S.wc_bs = b.weight_copy.batch_stride;
      S.variance = b.variance;
      S.rsq = use_normuon ? b.row_sumsq : nullptr;
      (void)update_scale(b.fan_out, b.fan_in, hp->scale_mode, hp->extra_scale_factor, &S.lr_scale);
      any_rsq |= S.rsq != nullptr;
      any_o |= S.rsq == nullptr;
      S.vec8 = vec8_ok(b, {&b.ns_out, &b.weight, &b.weight_copy});
      S.flat = flat_ok(b, {&b.ns_out, &b.weight, &b.weight_copy});
      ++ns;
    }
    if (ns == 0) continue;
    P.nseg = ns;
    P.total_chunks = chunk;
    P.total_slices = slice;
    P.total_rows = row;
    P.beta2 = hp->beta2;
    P.nor_eps = hp->nor_eps;
    P.lr = hp->lr;
    P.wd = hp->weight_decay;
    P.use_normuon = use_normuon ? 1 : 0;
    P.row_ss = row_ss;
    P.row_d = row_d;
    P.slice_factor = factor;
    if (use_normuon) {
      if (any_rsq && !launch_pdl(normuon_rows_from_sums_kernel, dim3(ew_grid(cdiv(row, EW_THREADS), sms)),
                                 dim3(EW_THREADS), 0, stream, P))
        return MUON_CUDA_ERROR;
      if (any_o && !launch_pdl(normuon_rows_kernel, dim3(ew_grid(cdiv(row, EW_THREADS / 32), sms)), dim3(EW_THREADS),
                               0, stream, P))
        return MUON_CUDA_ERROR;
      if (!launch_pdl(normuon_slices_kernel, dim3(ew_grid(slice, sms)), dim3(EW_THREADS), 0, stream, P))
        return MUON_CUDA_ERROR;
    }
    if (!launch_pdl(update_kernel, dim3(ew_grid(chunk, sms)), dim3(EW_THREADS), 0, stream, P))
      return MUON_CUDA_ERROR;
  }
  return MUON_OK;
}

muon_status muon_testing_gemm(int M, int N, int K, int slices, int tri, int in_dtype, const void* A, int64_t lda,
                              int64_t bsa, int a_mn, const void* B, int64_t ldb, int64_t bsb, int b_mn,
                              const void* D, int64_t ldd, int64_t bsd, int add_dtype, void* C, int64_t ldc,
                              int64_t bsc, int out_dtype, float alpha, float beta, float gamma, float f0, int s_pow,
                              const float* sumsq, float eps, float* row_ss, int cta_pair, int raster_group,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 1 || slices < 0) return MUON_BAD_SHAPE;
  if (cta_pair < 0 || cta_pair > 2 || raster_group < 0) return MUON_INVALID_ARG;
  if (tri && M != N) return MUON_BAD_SHAPE;
  if (!A || !B || !C) return MUON_INVALID_ARG;
  if (beta != 0.0f && !D) return MUON_INVALID_ARG;
  if (s_pow < 0 || s_pow > 2 || (s_pow > 0 && !sumsq)) return MUON_INVALID_ARG;
  if (!dtype_is(in_dtype, {MUON_BF16, MUON_F16}) || !dtype_is(out_dtype, {MUON_BF16, MUON_F16}) ||
      !dtype_is(add_dtype, {MUON_BF16, MUON_F16}))
    return MUON_UNSUPPORTED_DTYPE;
  auto al = [](const void* p, int64_t ld, int64_t bs) {
    return reinterpret_cast<uintptr_t>(p) % 16 == 0 && (ld * 2) % 16 == 0 && (bs * 2) % 16 == 0;
  };
  if (!al(A, lda, bsa) || !al(B, ldb, bsb) || !al(C, ldc, bsc) || (D && !al(D, ldd, bsd))) return MUON_MISALIGNED;
  muon_status st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MUON_OK) return st;
  if (M == 0 || N == 0 || slices == 0) return MUON_OK;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), stream) != cudaSuccess) return MUON_CUDA_ERROR;
  const int f16 = in_dtype == MUON_F16;
  ProblemSpec s{};
  s.M = M;
  s.N = N;
  s.K = K;
  s.slices = slices;
  s.tri = tri;
  s.a = a_mn ? Mat{A, K, M, lda, bsa, slices, f16} : Mat{A, M, K, lda, bsa, slices, f16};
  s.a_mn = a_mn;
  s.b = b_mn ? Mat{B, K, N, ldb, bsb, slices, f16} : Mat{B, N, K, ldb, bsb, slices, f16};
  s.b_mn = b_mn;
  s.in_f16 = f16;
  s.alpha = alpha;
  s.beta = beta;
  s.gamma = gamma;
  s.f0 = f0;
  s.s_pow = s_pow;
  s.eps = eps;
  s.sumsq = sumsq;
  s.addend = D;
  s.add_ld = ldd;
  s.add_bs = bsd;
  s.add_f16 = add_dtype == MUON_F16;
  s.out = C;
  s.out_ld = ldc;
  s.out_bs = bsc;
  s.out_f16 = out_dtype == MUON_F16;
  s.row_ss = tri ? nullptr : row_ss;
  s.mirror = 1;
  std::vector<ProblemSpec> v{s};
  return launch_gemms(v, sms, reinterpret_cast<int*>(workspace), stream, cta_pair, raster_group);
}

muon_status muon_testing_bounded_wait(uint64_t limit_ns, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
  muon_status st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MUON_OK) return st;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return MUON_INVALID_ARG;
  int sms = 0;
  if ((st = device_setup(&sms)) != MUON_OK) return st;
  if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), stream) != cudaSuccess) return MUON_CUDA_ERROR;
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(reinterpret_cast<int*>(workspace), limit_ns,
                                                  MUON_TESTING_WAIT_TIMEOUT);
  return launched() ? MUON_OK : MUON_CUDA_ERROR;
}

}  // extern "C"
