#include <cstdlib>
// C ABI of libdit: argument checks, TMA descriptor encoding and kernel
// launches for every entry point declared in include/dit.h.
//
// Every entry point validates its arguments before enqueuing anything, never
// allocates device memory, never synchronises (except dit_get_device_error)
// and reports CUDA failures as DIT_ERR_CUDA.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "attention.cuh"
#include "common.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"

using dit::bf16;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kVecSmemMax = 200 * 1024;  // staged input vectors of dit_vec_linear (B * K fp32)
constexpr int kRowSmemMax = 200 * 1024;  // bulk-staged row rings (8 warps x 2 rows) + vectors
// Per-CTA budgets of the tcgen05 kernels: 227 KB of shared memory (dynamic,
// including the alignment slack each kernel adds) and the 512 TMEM columns.
static_assert(dit::gemm::SMEM_BYTES <= 227 * 1024, "GEMM shared memory above the per-CTA limit");
static_assert(dit::gemm::pair::SMEM_BYTES <= 227 * 1024, "pair GEMM shared memory above the per-CTA limit");
static_assert(dit::attn::SMEM_BYTES <= 227 * 1024, "attention shared memory above the per-CTA limit");
static_assert(dit::gemm::TMEM_COLS <= 512 && dit::gemm::pair::TMEM_COLS <= 512 && dit::attn::TMEM_COLS <= 512,
              "TMEM allocation above 512 columns");
constexpr int kVecPipeSmemMax = 144 * 1024;
constexpr int kVecRowsCtasPerSm = 1;  // vec_rows kernels: 512 threads (16 warps) per CTA  // adaLN: 4 warps x 4 weight rows of K <= 4096 bf16 + K fp32
uint64_t g_wait_limit_ns = 2000000000ull;

// Per-device state, filled once under g_mu.  `init` is published with a
// release store after every other field is written and read with an acquire
// load, so a thread that sees it set also sees the fields.
struct DeviceInfo {
  std::atomic<bool> init{false};
  bool supported = false;
  int num_sms = 0;
  bool attrs_set = false;
  // dit_set_weight_l2_persist: N-fastest GEMMs keep their weight in the
  // persisting L2 set-aside
  std::atomic<bool> keep_weights{false};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Last CUDA error seen by a library call on this host thread.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

inline dit_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = e;
  return DIT_ERR_CUDA;
}

#define DIT_CUDA_CHECK(expr)                      \
  do {                                            \
    cudaError_t e_ = (expr);                      \
    if (e_ != cudaSuccess) return cuda_fail(e_);  \
  } while (0)

dit_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DIT_OK : cuda_fail(e);
}

// Kernels of the block path are launched with programmatic stream
// serialization: a launch may begin while the previous kernel of the stream
// drains, and each of these kernels holds every global-memory access behind
// griddep_wait() (common.cuh), so only prologues overlap.  DIT_DISABLE_PDL=1
// in the environment launches them the plain way.  Errors surface through the
// caller's launch_status().
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("DIT_DISABLE_PDL");
    return !(v != nullptr && v[0] == '1');
  }();
  return on;
}

// Set while a profiled call records events between its kernels: those
// launches go the plain way, so each kernel's interval is its own.
thread_local bool t_plain_launches = false;
struct PlainLaunches {
  bool prev;
  PlainLaunches() : prev(t_plain_launches) { t_plain_launches = true; }
  ~PlainLaunches() { t_plain_launches = prev; }
};

template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (pdl_enabled() && !t_plain_launches) ? 1 : 0;
  (void)cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Per-device setup: SM count, capability check, kernel attributes, driver
// entry point for tensor-map encoding.
dit_status device_setup(int* num_sms) {
  int dev = 0;
  DIT_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return DIT_ERR_UNSUPPORTED;
  DeviceInfo& d = g_dev[dev];
  if (!d.init.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d.init.load(std::memory_order_relaxed)) {
      int major = 0, sms = 0;
      DIT_CUDA_CHECK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
      DIT_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
      d.supported = (major == 10);
      d.num_sms = sms;
      if (d.supported) {
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::gemm_kernel<DIT_EPI_NONE>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::gemm_kernel<DIT_EPI_BIAS>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::gemm_kernel<DIT_EPI_BIAS_GELU_COLS>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::gemm_kernel<DIT_EPI_BIAS_GATED_RESIDUAL>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::attn::attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            dit::attn::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::pair::gemm_pair_kernel<DIT_EPI_NONE>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::pair::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::pair::gemm_pair_kernel<DIT_EPI_BIAS>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::pair::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::pair::gemm_pair_kernel<DIT_EPI_BIAS_GELU_COLS>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::pair::SMEM_BYTES));
        DIT_CUDA_CHECK(cudaFuncSetAttribute(dit::gemm::pair::gemm_pair_kernel<DIT_EPI_BIAS_GATED_RESIDUAL>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, dit::gemm::pair::SMEM_BYTES));
        for (int nb = 1; nb <= 8; nb *= 2) {
          void* f = nb == 1   ? (void*)dit::vec_linear_kernel<1>
                    : nb == 2 ? (void*)dit::vec_linear_kernel<2>
                    : nb == 4 ? (void*)dit::vec_linear_kernel<4>
                              : (void*)dit::vec_linear_kernel<8>;
          DIT_CUDA_CHECK(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kVecSmemMax));
          void* fb = nb == 1   ? (void*)dit::vec_linear_bulk_kernel<1>
                     : nb == 2 ? (void*)dit::vec_linear_bulk_kernel<2>
                     : nb == 4 ? (void*)dit::vec_linear_bulk_kernel<4>
                               : (void*)dit::vec_linear_bulk_kernel<8>;
          DIT_CUDA_CHECK(cudaFuncSetAttribute(fb, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemMax));
        }
        const void* vec_pipe[8] = {
            (const void*)dit::vec_linear_pipe_kernel<1>, (const void*)dit::vec_linear_pipe_kernel<2>,
            (const void*)dit::vec_linear_pipe_kernel<3>, (const void*)dit::vec_linear_pipe_kernel<4>,
            (const void*)dit::vec_linear_pipe_kernel<6>, (const void*)dit::vec_linear_pipe_kernel<8>,
            (const void*)dit::vec_linear_pipe_kernel<12>, (const void*)dit::vec_linear_pipe_kernel<16>};
        const void* vec_multi[8] = {
            (const void*)dit::vec_linear_multi_kernel<1>, (const void*)dit::vec_linear_multi_kernel<2>,
            (const void*)dit::vec_linear_multi_kernel<3>, (const void*)dit::vec_linear_multi_kernel<4>,
            (const void*)dit::vec_linear_multi_kernel<6>, (const void*)dit::vec_linear_multi_kernel<8>,
            (const void*)dit::vec_linear_multi_kernel<12>, (const void*)dit::vec_linear_multi_kernel<16>};
        for (const void* f : vec_multi) {
          DIT_CUDA_CHECK(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kVecPipeSmemMax));
          DIT_CUDA_CHECK(cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        }
        // the grid assumes every CTA the occupancy calculator allows is resident: ask for the
        // largest shared-memory carveout so the launch does not pick a smaller one
        for (const void* f : vec_pipe) {
          DIT_CUDA_CHECK(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kVecPipeSmemMax));
          DIT_CUDA_CHECK(cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        }
        if (g_encode == nullptr) {
          void* fn = nullptr;
          cudaDriverEntryPointQueryResult q;
          DIT_CUDA_CHECK(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
          if (q != cudaDriverEntryPointSuccess || fn == nullptr) return DIT_ERR_CUDA;
          g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
      }
      d.init.store(true, std::memory_order_release);
    }
  }
  if (!d.supported) return DIT_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = d.num_sms;
  return DIT_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D bf16 tensor map: rows x cols (cols contiguous, row stride ld elements),
// box = box_rows x 64 columns, 128-byte swizzle, zero fill out of bounds.
dit_status make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int64_t ld, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_CUDA;
}

// 3-D bf16 tensor map over [batch][rows][cols] with row stride ld elements and
// batch stride rows*ld; box = box_rows rows x 64 columns x 1.
dit_status make_map_3d(CUtensorMap* m, const void* base, uint64_t batch, uint64_t rows, uint64_t cols, int64_t ld,
                       uint32_t box_rows) {
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * rows};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_CUDA;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Internal RoPE-only / norm+RoPE launch shared by the public call and blocks.
dit_status launch_qk(const bf16* q, const bf16* k, int64_t ld_in, const bf16* qs, const bf16* ks, const float* rope,
                     bf16* qo, bf16* ko, int64_t ld_out, int B, int S, int H, float eps, int do_norm,
                     cudaStream_t st) {
  if (B > 65535) return DIT_ERR_SHAPE;
  const dim3 grid((unsigned)S, (unsigned)B);  // one CTA per token row
  dit::qk_norm_rope_kernel<3><<<grid, 128, 0, st>>>(q, k, ld_in, qs, ks, reinterpret_cast<const float2*>(rope), qo,
                                                    ko, ld_out, S, H, eps, do_norm);
  return launch_status();
}

// LayerNorm + modulate row ring: resident CTAs per SM and the shared-memory
// budget of one CTA's ring of rows.
constexpr int kNormRingCtasPerSm = 4;
constexpr int kNormRingBytes = 18432;

template <typename Kern>
static dit_status ring_launch(Kern kernel, dim3 grid, int threads, int smem, cudaStream_t st, const bf16* x,
                              int64_t ldx, const float* shift, const float* scale, int64_t mod_stride, bf16* y,
                              int64_t ldy, int S, int D, float eps, int R) {
  // dynamic plus static shared memory above 48 KB needs the opt-in
  if (smem > 40 * 1024 && cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DIT_ERR_CUDA;
  launch_pdl(kernel, grid, threads, smem, st, x, ldx, shift, scale, mod_stride, y, ldy, S, D, eps, R,
             g_wait_limit_ns);
  return DIT_OK;
}

}  // namespace

extern "C" {

const char* dit_status_string(dit_status s) {
  switch (s) {
    case DIT_OK: return "ok";
    case DIT_ERR_INVALID_ARG: return "invalid argument";
    case DIT_ERR_SHAPE: return "unsupported shape";
    case DIT_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case DIT_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case DIT_ERR_CUDA: return "CUDA runtime error";
    case DIT_ERR_NOT_CAPTURABLE: return "not allowed while the stream is capturing";
    case DIT_ERR_TIMEOUT: return "device-side wait timed out";
    case DIT_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int dit_version(void) { return 100; }

const char* dit_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

dit_status dit_get_device_error(void* stream, uint32_t* code) {
  if (code == nullptr) return DIT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  DIT_CUDA_CHECK(cudaStreamIsCapturing(st, &cs));
  if (cs != cudaStreamCaptureStatusNone) return DIT_ERR_NOT_CAPTURABLE;
  unsigned int v = 0;
  DIT_CUDA_CHECK(cudaMemcpyFromSymbolAsync(&v, dit::g_dit_error, sizeof(v), 0, cudaMemcpyDeviceToHost, st));
  DIT_CUDA_CHECK(cudaStreamSynchronize(st));
  *code = v;
  return v == 0 ? DIT_OK : DIT_ERR_TIMEOUT;
}

dit_status dit_clear_device_error(void* stream) {
  static const unsigned int zero = 0;
  DIT_CUDA_CHECK(cudaMemcpyToSymbolAsync(dit::g_dit_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                         (cudaStream_t)stream));
  DIT_CUDA_CHECK(cudaStreamSynchronize((cudaStream_t)stream));
  return DIT_OK;
}

size_t dit_abi_struct_size(int which) {
  switch (which) {
    case 0: return sizeof(dit_gemm_args);
    case 1: return sizeof(dit_block_cfg);
    case 2: return sizeof(dit_single_weights);
    case 3: return sizeof(dit_stream_weights);
    case 4: return sizeof(dit_double_weights);
    case 5: return sizeof(dit_video_weights);
    case 6: return sizeof(dit_model);
    case 7: return sizeof(dit_loop_io);
    default: return 0;
  }
}

dit_status dit_set_weight_l2_persist(size_t bytes) {
  int dev = 0;
  DIT_CUDA_CHECK(cudaGetDevice(&dev));
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  int maxp = 0;
  DIT_CUDA_CHECK(cudaDeviceGetAttribute(&maxp, cudaDevAttrMaxPersistingL2CacheSize, dev));
  const size_t want = bytes < (size_t)maxp ? bytes : (size_t)maxp;
  DIT_CUDA_CHECK(cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, want));
  g_dev[dev].keep_weights.store(want > 0, std::memory_order_relaxed);
  return DIT_OK;
}

dit_status dit_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns == 0) return DIT_ERR_INVALID_ARG;
  g_wait_limit_ns = limit_ns;
  return DIT_OK;
}

dit_status dit_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  dit::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
  return launch_status();
}

dit_status dit_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (x == nullptr || y == nullptr || n < 1) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > INT32_MAX) return DIT_ERR_SHAPE;
  dit::selftest_exp2_poly_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(x, y, n);
  return launch_status();
}

dit_status dit_rope_table(const int32_t* ids, int S, int n_axes, const int* axes_pairs, double theta, float* rope,
                          void* stream) {
  if (ids == nullptr || rope == nullptr || axes_pairs == nullptr) return DIT_ERR_INVALID_ARG;
  if (S <= 0 || n_axes < 1 || n_axes > 3 || !(theta > 0)) return DIT_ERR_INVALID_ARG;
  int p[3] = {0, 0, 0};
  for (int a = 0; a < n_axes; ++a) {
    if (axes_pairs[a] < 0) return DIT_ERR_INVALID_ARG;
    p[a] = axes_pairs[a];
  }
  if (p[0] + p[1] + p[2] <= 0) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  const int64_t n = (int64_t)S * (p[0] + p[1] + p[2]);
  dit::rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
      ids, S, n_axes, p[0], p[1], p[2], theta, reinterpret_cast<float2*>(rope));
  return launch_status();
}

dit_status dit_vec_linear(const dit_bf16* x, int64_t ldx, const dit_bf16* W, int64_t ldw, const dit_bf16* bias,
                          void* out, int64_t ldo, int B, int N, int K, int flags, void* stream) {
  if (x == nullptr || W == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || B > 8 || N < 1 || K < 8 || K > 8192 || (K % 8) != 0) return DIT_ERR_SHAPE;
  if ((size_t)B * K * sizeof(float) > (size_t)kVecSmemMax) return DIT_ERR_SHAPE;
  if (ldx < K || ldw < K || ldo < N || (ldw % 8) != 0) return DIT_ERR_SHAPE;
  if (!aligned16(W)) return DIT_ERR_ALIGNMENT;
  if (flags & ~(DIT_VEC_SILU_IN | DIT_VEC_OUT_BF16)) return DIT_ERR_INVALID_ARG;
  int sms = 0;
  dit_status s = device_setup(&sms);
  if (s != DIT_OK) return s;
  const int threads = 256, wpb = threads / 32;
  int blocks = (N + wpb - 1) / wpb;
  if (blocks > sms * 8) blocks = sms * 8;
  const size_t smem = (size_t)B * K * sizeof(float);
  cudaStream_t st = (cudaStream_t)stream;
  const bf16* xb = reinterpret_cast<const bf16*>(x);
  const bf16* Wb = reinterpret_cast<const bf16*>(W);
  const bf16* bb = reinterpret_cast<const bf16*>(bias);
  if (B <= 2 && (K % 256) == 0 && K <= 3072) {
    // one warp per weight row, 16 warps per CTA, one CTA per SM
    int64_t grid = (int64_t)sms * kVecRowsCtasPerSm;
    if (N < grid * 16) grid = (N + 15) / 16;
    const size_t xs_smem = (size_t)B * K * 4;
#define DIT_VR_CASE(KC_)                                                                                       \
  case KC_:                                                                                                    \
    if (B == 1)                                                                                                \
      launch_pdl(dit::vec_rows_kernel<KC_, 1>, (unsigned)grid, 512, xs_smem, st, xb, ldx, Wb, ldw, bb, out, ldo, N, K, \
                                                                         flags);                               \
    else                                                                                                       \
      launch_pdl(dit::vec_rows_kernel<KC_, 2>, (unsigned)grid, 512, xs_smem, st, xb, ldx, Wb, ldw, bb, out, ldo, N, K, \
                                                                         flags);                               \
    return launch_status();
    switch (K / 256) {
      DIT_VR_CASE(1)
      DIT_VR_CASE(2)
      DIT_VR_CASE(3)
      DIT_VR_CASE(4)
      DIT_VR_CASE(6)
      DIT_VR_CASE(8)
      DIT_VR_CASE(12)
      default:
        break;
    }
#undef DIT_VR_CASE
  }
  if (B == 1 && (K % 256) == 0 && K <= 4096) {
    // weight rows in flight through warp-private shared-memory rings (cp.async, 3 rows ahead)
    const size_t ring_smem = (size_t)dit::kVecPipeWarps * dit::kVecPipeSlots * K * 2 + (size_t)K * 4;
    int rgrid = (N + dit::kVecPipeWarps - 1) / dit::kVecPipeWarps;
    const int per_sm = (int)(220 * 1024 / (ring_smem + 1024));
    if (rgrid > sms * per_sm) rgrid = sms * per_sm;
    switch (K / 256) {
      case 16:
        dit::vec_linear_pipe_kernel<16><<<rgrid, 128, ring_smem, st>>>(xb, Wb, ldw, bb, out, N, K, flags);
        return launch_status();
      default:
        break;
    }
  }
  const size_t bulk_smem = smem + (size_t)dit::kRowWarps * 2 * K * 2 + dit::kRowWarps * 2 * 8;
  if (bulk_smem <= (size_t)kRowSmemMax) {
    // weight rows staged through shared memory by bulk copies
    int bgrid = (N + dit::kRowWarps - 1) / dit::kRowWarps;
    const int per_sm = (int)(228 * 1024 / (bulk_smem + 1024));
    const int cap = sms * (per_sm > 0 ? per_sm : 1);
    if (bgrid > cap) bgrid = cap;
    if (B == 1)
      dit::vec_linear_bulk_kernel<1><<<bgrid, 256, bulk_smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags,
                                                                    g_wait_limit_ns);
    else if (B <= 2)
      dit::vec_linear_bulk_kernel<2><<<bgrid, 256, bulk_smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags,
                                                                    g_wait_limit_ns);
    else if (B <= 4)
      dit::vec_linear_bulk_kernel<4><<<bgrid, 256, bulk_smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags,
                                                                    g_wait_limit_ns);
    else
      dit::vec_linear_bulk_kernel<8><<<bgrid, 256, bulk_smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags,
                                                                    g_wait_limit_ns);
    return launch_status();
  }
  if (B == 1)
    dit::vec_linear_kernel<1><<<blocks, threads, smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags);
  else if (B <= 2)
    dit::vec_linear_kernel<2><<<blocks, threads, smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags);
  else if (B <= 4)
    dit::vec_linear_kernel<4><<<blocks, threads, smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags);
  else
    dit::vec_linear_kernel<8><<<blocks, threads, smem, st>>>(xb, ldx, Wb, ldw, bb, out, ldo, B, N, K, flags);
  return launch_status();
}

// One pass over every matrix of p (batch-1 input x shared by all): see
// vec_rows_multi_kernel (K <= 3072) and vec_linear_multi_kernel (K = 4096).
// K % 256 == 0, K <= 4096; used by the loop.
bool multi_linear_supported(int K) { return (K % 256) == 0 && K <= 4096; }

dit_status multi_linear(const dit_bf16* x, const dit::MultiLinear& p, int flags, cudaStream_t st) {
  if (!multi_linear_supported(p.K) || p.n_mats < 1 || p.n_mats > dit::kMultiMaxMats) return DIT_ERR_SHAPE;
  int sms = 0;
  dit_status s = device_setup(&sms);
  if (s != DIT_OK) return s;
  const int64_t N = p.row_begin[p.n_mats];
  if (p.K <= 3072) {
    int64_t rgrid = (int64_t)sms * kVecRowsCtasPerSm;
    if (N < rgrid * 16) rgrid = (N + 15) / 16;
    const size_t xs_smem = (size_t)p.K * 4;
    const bf16* xr = reinterpret_cast<const bf16*>(x);
    switch (p.K / 256) {
#define DIT_VRM_CASE(KC_)                                                                          \
  case KC_:                                                                                        \
    launch_pdl(dit::vec_rows_multi_kernel<KC_>, (unsigned)rgrid, 512, xs_smem, st, xr, p, flags);         \
    return launch_status();
      DIT_VRM_CASE(1)
      DIT_VRM_CASE(2)
      DIT_VRM_CASE(3)
      DIT_VRM_CASE(4)
      DIT_VRM_CASE(6)
      DIT_VRM_CASE(8)
      DIT_VRM_CASE(12)
#undef DIT_VRM_CASE
      default:
        break;
    }
  }
  const size_t smem = (size_t)dit::kVecPipeWarps * dit::kVecPipeSlots * p.K * 2 + (size_t)p.K * 4;
  int64_t grid = (N + dit::kVecPipeWarps - 1) / dit::kVecPipeWarps;
  const int per_sm = (int)(220 * 1024 / (smem + 1024));
  if (grid > (int64_t)sms * per_sm) grid = (int64_t)sms * per_sm;
  const bf16* xb = reinterpret_cast<const bf16*>(x);
  switch (p.K / 256) {
#define DIT_VM_CASE(KC_)                                                                        \
  case KC_:                                                                                     \
    dit::vec_linear_multi_kernel<KC_><<<(unsigned)grid, 128, smem, st>>>(xb, p, flags);        \
    return launch_status();
    DIT_VM_CASE(1)
    DIT_VM_CASE(2)
    DIT_VM_CASE(3)
    DIT_VM_CASE(4)
    DIT_VM_CASE(6)
    DIT_VM_CASE(8)
    DIT_VM_CASE(12)
    DIT_VM_CASE(16)
#undef DIT_VM_CASE
    default:
      return DIT_ERR_SHAPE;
  }
}

dit_status dit_adaln_modulation(const dit_bf16* vec, int64_t ldv, const dit_bf16* W, int64_t ldw,
                                const dit_bf16* bias, float* out, int64_t ldo, int B, int N, int K, void* stream) {
  return dit_vec_linear(vec, ldv, W, ldw, bias, out, ldo, B, N, K, DIT_VEC_SILU_IN, stream);
}

dit_status dit_modulate_norm(const dit_bf16* x, int64_t ldx, const float* shift, const float* scale,
                             int64_t mod_stride, dit_bf16* y, int64_t ldy, int B, int S, int D, float eps,
                             void* stream) {
  if (x == nullptr || y == nullptr) return DIT_ERR_INVALID_ARG;
  if ((shift == nullptr) != (scale == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || D < 8 || D > 8192 || (D % 8) != 0) return DIT_ERR_SHAPE;
  if (ldx < D || ldy < D || (ldx % 8) != 0 || (ldy % 8) != 0) return DIT_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y)) return DIT_ERR_ALIGNMENT;
  if (shift != nullptr && (!aligned16(shift) || !aligned16(scale) || (mod_stride % 4) != 0))
    return DIT_ERR_ALIGNMENT;
  if (!(eps >= 0)) return DIT_ERR_INVALID_ARG;
  if ((const void*)x == (const void*)y) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  const int64_t rows = (int64_t)B * S;
  const bf16* xb = reinterpret_cast<const bf16*>(x);
  bf16* yb = reinterpret_cast<bf16*>(y);
  cudaStream_t st = (cudaStream_t)stream;
  {
    int sms = 0;
    if ((s = device_setup(&sms)) != DIT_OK) return s;
    // one CTA per row: NC 16-byte chunks per thread, D / (8 NC) threads a multiple of 32 in [32, 256]
    int NC = 0;
    for (int c : {3, 4, 2, 1}) {
      const int t = D / (8 * c);
      if (D % (8 * c) == 0 && t % 32 == 0 && t >= 32 && t <= 256) {
        NC = c;
        break;
      }
    }
    if (NC != 0 && B <= 65535) {
      // persistent row ring: kNormRingCtasPerSm CTAs per SM in all, each with
      // R = kNormRingBytes / (2 D) rows (2..8) in flight
      const int threads = D / (8 * NC);
      const int R = std::max(2, std::min(dit::kNormRingMaxStages, kNormRingBytes / (2 * D)));
      const int smem = R * 2 * D;
      const int gx = (int)std::max<int64_t>(1, std::min<int64_t>(S, ((int64_t)kNormRingCtasPerSm * sms + B - 1) / B));
      const dim3 grid((unsigned)gx, (unsigned)B);
      if (NC == 1)
        s = ring_launch(dit::modulate_norm_ring_kernel<1>, grid, threads, smem, st, xb, ldx, shift, scale, mod_stride, yb,
                        ldy, S, D, eps, R);
      else if (NC == 2)
        s = ring_launch(dit::modulate_norm_ring_kernel<2>, grid, threads, smem, st, xb, ldx, shift, scale, mod_stride, yb,
                        ldy, S, D, eps, R);
      else if (NC == 3)
        s = ring_launch(dit::modulate_norm_ring_kernel<3>, grid, threads, smem, st, xb, ldx, shift, scale, mod_stride, yb,
                        ldy, S, D, eps, R);
      else
        s = ring_launch(dit::modulate_norm_ring_kernel<4>, grid, threads, smem, st, xb, ldx, shift, scale, mod_stride, yb,
                        ldy, S, D, eps, R);
      if (s != DIT_OK) return s;
      return launch_status();
    }
    // otherwise (D not a multiple of 256 or 768): persistent row stream, D/8 threads per CTA
    const int threads = ((D / 8 + 31) / 32) * 32;
    const int per_sm = 2048 / threads;
    int64_t grid = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    if (grid > rows) grid = rows;
    dit::modulate_norm_stream_kernel<<<(unsigned)grid, threads, 0, st>>>(xb, ldx, shift, scale, mod_stride, yb,
                                                                         ldy, rows, S, D, eps);
    return launch_status();
  }
}

dit_status dit_qk_norm_rope(const dit_bf16* q, const dit_bf16* k, int64_t ld_in, const dit_bf16* q_scale,
                            const dit_bf16* k_scale, const float* rope, dit_bf16* q_out, dit_bf16* k_out,
                            int64_t ld_out, int B, int S, int H, int head_dim, float eps, void* stream) {
  if (q == nullptr || k == nullptr || q_out == nullptr || k_out == nullptr) return DIT_ERR_INVALID_ARG;
  if (head_dim != 128) return DIT_ERR_UNSUPPORTED;
  if (B < 1 || S < 1 || H < 1) return DIT_ERR_SHAPE;
  if (ld_in < (int64_t)H * 128 || ld_out < (int64_t)H * 128 || (ld_in % 8) != 0 || (ld_out % 8) != 0)
    return DIT_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return DIT_ERR_ALIGNMENT;
  if ((q_scale && !aligned16(q_scale)) || (k_scale && !aligned16(k_scale)) || (rope && !aligned16(rope)))
    return DIT_ERR_ALIGNMENT;
  if (!(eps >= 0)) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  return launch_qk(reinterpret_cast<const bf16*>(q), reinterpret_cast<const bf16*>(k), ld_in,
                   reinterpret_cast<const bf16*>(q_scale), reinterpret_cast<const bf16*>(k_scale), rope,
                   reinterpret_cast<bf16*>(q_out), reinterpret_cast<bf16*>(k_out), ld_out, B, S, H, eps, 1,
                   (cudaStream_t)stream);
}

}  // extern "C"

namespace {

// splits > 1: o and lse are the partial-result arrays (split s at o + s
// o_split_stride, lse + s lse_split_stride), kv_per_split a multiple of BKV
// with every split non-empty; accumulate must be 0.
dit_status attention_launch(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v, int64_t ldq, int64_t ldk,
                            int64_t ldv, dit_bf16* o, int64_t ldo, float* lse, int B, int Sq, int Skv, int H,
                            int head_dim, float softmax_scale, int accumulate, void* stream, int splits = 1,
                            int kv_per_split = 0, int64_t o_split_stride = 0, int64_t lse_split_stride = 0) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return DIT_ERR_INVALID_ARG;
  if (head_dim != 128) return DIT_ERR_UNSUPPORTED;
  if (B < 1 || Sq < 1 || Skv < 1 || H < 1 || B > 65535 || H > 65535) return DIT_ERR_SHAPE;
  const int64_t D = (int64_t)H * 128;
  if (ldq < D || ldk < D || ldv < D || ldo < D) return DIT_ERR_SHAPE;
  if ((ldq % 8) || (ldk % 8) || (ldv % 8) || (ldo % 8)) return DIT_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DIT_ERR_ALIGNMENT;
  if (!(softmax_scale > 0)) return DIT_ERR_INVALID_ARG;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  CUtensorMap tq, tk, tv;
  if ((s = make_map_3d(&tq, q, B, Sq, D, ldq, dit::attn::BQ)) != DIT_OK) return s;
  if ((s = make_map_3d(&tk, k, B, Skv, D, ldk, dit::attn::BKV)) != DIT_OK) return s;
  if ((s = make_map_3d(&tv, v, B, Skv, D, ldv, dit::attn::BKV)) != DIT_OK) return s;
  dit::attn::Params p;
  p.o = reinterpret_cast<bf16*>(o);
  p.ldo = ldo;
  p.lse = lse;
  p.Sq = Sq;
  p.Skv = Skv;
  p.H = H;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.accumulate = accumulate;
  p.splits = splits;
  p.kv_per_split = splits > 1 ? kv_per_split : Skv;
  p.o_split_stride = o_split_stride;
  p.lse_split_stride = lse_split_stride;
  if ((int64_t)B * splits > 65535) return DIT_ERR_SHAPE;
  dim3 grid((unsigned)((Sq + 2 * dit::attn::BQ - 1) / (2 * dit::attn::BQ)), (unsigned)H, (unsigned)(B * splits));
  launch_pdl(dit::attn::attention_kernel, grid, dit::attn::NUM_THREADS, dit::attn::SMEM_BYTES, (cudaStream_t)stream, 
      tq, tk, tv, p, g_wait_limit_ns);
  return launch_status();
}

// Log-sum-exp merge of n parts, part j with row stride lds[j].
dit_status merge_launch(int n, const dit_bf16* const* o_parts, const float* const* lse_parts, const int64_t* lds,
                        dit_bf16* o, float* lse_out, int64_t ld_out, int B, int S, int H, void* stream) {
  if (o == nullptr) return DIT_ERR_INVALID_ARG;
  if (n < 1 || n > dit::kMergeMaxParts) return DIT_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || H < 1 || B > 65535 || H > 65535) return DIT_ERR_SHAPE;
  const int64_t D = (int64_t)H * 128;
  if (ld_out < D) return DIT_ERR_SHAPE;
  if ((ld_out % 8) || !aligned16(o)) return DIT_ERR_ALIGNMENT;
  dit::MergeParams p{};
  for (int j = 0; j < n; ++j) {
    if (o_parts[j] == nullptr || lse_parts[j] == nullptr) return DIT_ERR_INVALID_ARG;
    if (lds[j] < D) return DIT_ERR_SHAPE;
    if ((lds[j] % 8) || !aligned16(o_parts[j])) return DIT_ERR_ALIGNMENT;
    p.o[j] = reinterpret_cast<const bf16*>(o_parts[j]);
    p.lse[j] = lse_parts[j];
    p.ld[j] = lds[j];
  }
  p.out = reinterpret_cast<bf16*>(o);
  p.lse_out = lse_out;
  p.ld_out = ld_out;
  p.n = n;
  p.B = B;
  p.S = S;
  p.H = H;
  dit_status s = device_setup(nullptr);
  if (s != DIT_OK) return s;
  const dim3 grid((unsigned)((S + 15) / 16), (unsigned)H, (unsigned)B);
  if (n <= 2)
    launch_pdl(dit::attention_merge_kernel<2>, grid, 256, 0, (cudaStream_t)stream, p);
  else if (n <= 4)
    launch_pdl(dit::attention_merge_kernel<4>, grid, 256, 0, (cudaStream_t)stream, p);
  else
    launch_pdl(dit::attention_merge_kernel<8>, grid, 256, 0, (cudaStream_t)stream, p);
  return launch_status();
}

}  // namespace

extern "C" {

dit_status dit_attention(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v, int64_t ldq, int64_t ldk,
                         int64_t ldv, dit_bf16* o, int64_t ldo, float* lse, int B, int Sq, int Skv, int H,
                         int head_dim, float softmax_scale, void* stream) {
  return attention_launch(q, k, v, ldq, ldk, ldv, o, ldo, lse, B, Sq, Skv, H, head_dim, softmax_scale, 0, stream);
}

dit_status dit_attention_accumulate(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v, int64_t ldq,
                                    int64_t ldk, int64_t ldv, dit_bf16* o, int64_t ldo, float* lse, int B, int Sq,
                                    int Skv, int H, int head_dim, float softmax_scale, void* stream) {
  if (lse == nullptr) return DIT_ERR_INVALID_ARG;
  return attention_launch(q, k, v, ldq, ldk, ldv, o, ldo, lse, B, Sq, Skv, H, head_dim, softmax_scale, 1, stream);
}

// Key ranges of a split launch: whole key tiles per split, every split non-empty.
static void split_plan(int Skv, int n_split, int* splits, int* kv_per_split) {
  const int tiles = (Skv + dit::attn::BKV - 1) / dit::attn::BKV;
  int n = n_split < tiles ? n_split : tiles;
  if (n < 1) n = 1;
  const int per = (tiles + n - 1) / n;
  *splits = (tiles + per - 1) / per;
  *kv_per_split = per * dit::attn::BKV;
}

size_t dit_attention_split_workspace(int B, int Sq, int H, int n_split) {
  if (B < 1 || Sq < 1 || H < 1 || n_split < 1) return 0;
  const size_t n = (size_t)(n_split > dit::kAttnMaxSplits ? dit::kAttnMaxSplits : n_split);
  return n * align256((size_t)B * Sq * H * 128 * sizeof(dit_bf16)) + n * align256((size_t)B * H * Sq * sizeof(float));
}

dit_status dit_attention_split(const dit_bf16* q, const dit_bf16* k, const dit_bf16* v, int64_t ldq, int64_t ldk,
                               int64_t ldv, dit_bf16* o, int64_t ldo, float* lse, int B, int Sq, int Skv, int H,
                               int head_dim, float softmax_scale, int n_split, int accumulate, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (n_split < 1 || n_split > dit::kAttnMaxSplits) return DIT_ERR_INVALID_ARG;
  if (accumulate && lse == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || Sq < 1 || Skv < 1 || H < 1) return DIT_ERR_SHAPE;
  int splits = 1, per = 0;
  split_plan(Skv, n_split, &splits, &per);
  if (splits == 1)
    return attention_launch(q, k, v, ldq, ldk, ldv, o, ldo, lse, B, Sq, Skv, H, head_dim, softmax_scale, accumulate,
                            stream);
  if (workspace == nullptr) return DIT_ERR_WORKSPACE;
  if (workspace_bytes < dit_attention_split_workspace(B, Sq, H, splits)) return DIT_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DIT_ERR_ALIGNMENT;
  const int64_t D = (int64_t)H * 128;
  // the output is checked here because the merge, not the attention, writes it
  if (o == nullptr) return DIT_ERR_INVALID_ARG;
  if (ldo < D || B > 65535 || H > 65535) return DIT_ERR_SHAPE;
  if ((ldo % 8) != 0 || !aligned16(o)) return DIT_ERR_ALIGNMENT;
  const size_t o_bytes = align256((size_t)B * Sq * D * sizeof(dit_bf16));
  dit_bf16* o_parts = reinterpret_cast<dit_bf16*>(workspace);
  float* lse_parts = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + (size_t)splits * o_bytes);
  const size_t lse_bytes = align256((size_t)B * H * Sq * sizeof(float));
  dit_status s = attention_launch(q, k, v, ldq, ldk, ldv, o_parts, D, lse_parts, B, Sq, Skv, H, head_dim,
                                  softmax_scale, 0, stream, splits, per, (int64_t)(o_bytes / sizeof(dit_bf16)),
                                  (int64_t)(lse_bytes / sizeof(float)));
  if (s != DIT_OK) return s;
  // merge the splits (and the running result when accumulating) into o, lse
  const dit_bf16* op[dit::kMergeMaxParts];
  const float* lp[dit::kMergeMaxParts];
  int n = 0;
  if (accumulate) {
    op[n] = o;
    lp[n] = lse;
    ++n;
  }
  for (int j = 0; j < splits; ++j, ++n) {
    op[n] = o_parts + (size_t)j * (o_bytes / sizeof(dit_bf16));
    lp[n] = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(lse_parts) + (size_t)j * lse_bytes);
  }
  int64_t lds[dit::kMergeMaxParts];
  for (int j = 0; j < n; ++j) lds[j] = D;
  if (accumulate) lds[0] = ldo;  // the running result is both a part and the output
  return merge_launch(n, op, lp, lds, o, lse, ldo, B, Sq, H, stream);
}

dit_status dit_attention_merge(int n, const dit_bf16* const* o_parts, const float* const* lse_parts, int64_t ld_in,
                               dit_bf16* o, float* lse_out, int64_t ld_out, int B, int S, int H, void* stream) {
  if (o_parts == nullptr || lse_parts == nullptr) return DIT_ERR_INVALID_ARG;
  if (n < 1 || n > dit::kMergeMaxParts) return DIT_ERR_INVALID_ARG;
  int64_t lds[dit::kMergeMaxParts];
  for (int j = 0; j < n; ++j) lds[j] = ld_in;
  return merge_launch(n, o_parts, lse_parts, lds, o, lse_out, ld_out, B, S, H, stream);
}

}  // extern "C"

namespace {

dit_status gemm_validate(const dit_gemm_args* a) {
  if (a == nullptr || a->A == nullptr || a->W == nullptr || a->C == nullptr) return DIT_ERR_INVALID_ARG;
  if (a->M < 1 || a->N < 32 || a->K < 8 || (a->N % 32) != 0 || (a->K % 8) != 0) return DIT_ERR_SHAPE;
  if (a->lda < a->K || a->ldw < a->K || (a->lda % 8) || (a->ldw % 8)) return DIT_ERR_SHAPE;
  if (!aligned16(a->A) || !aligned16(a->W) || !aligned16(a->C)) return DIT_ERR_ALIGNMENT;
  const int split = a->C2 ? a->split_col : a->N;
  if (a->C2 != nullptr) {
    if (split < 0 || split > a->N || (split % 32) != 0) return DIT_ERR_SHAPE;
    if (!aligned16(a->C2) || (a->ldc2 % 8) != 0 || a->ldc2 < a->N - split) return DIT_ERR_ALIGNMENT;
  }
  if ((a->ldc % 8) != 0 || a->ldc < split) return DIT_ERR_SHAPE;
  if (a->bias && !aligned16(a->bias)) return DIT_ERR_ALIGNMENT;
  if (a->qk_cols != 0) {
    if (a->qk_cols < 0 || (a->qk_cols % 256) != 0 || a->qk_cols > split) return DIT_ERR_SHAPE;
    if (a->epi == DIT_EPI_BIAS_GATED_RESIDUAL) return DIT_ERR_INVALID_ARG;
    if ((a->q_scale && !aligned16(a->q_scale)) || (a->k_scale && !aligned16(a->k_scale)) ||
        (a->rope && !aligned16(a->rope)))
      return DIT_ERR_ALIGNMENT;
    if (a->rope && a->rope_rows < 1) return DIT_ERR_INVALID_ARG;
    if (!(a->qk_eps >= 0)) return DIT_ERR_INVALID_ARG;
  }
  switch (a->epi) {
    case DIT_EPI_NONE:
    case DIT_EPI_BIAS:
      break;
    case DIT_EPI_BIAS_GELU_COLS:
      if (a->gelu_col_begin < 0 || (a->gelu_col_begin % 32) != 0) return DIT_ERR_SHAPE;
      break;
    case DIT_EPI_BIAS_GATED_RESIDUAL:
      if (a->resid == nullptr || a->rows_per_batch < 1) return DIT_ERR_INVALID_ARG;
      if (!aligned16(a->resid) || (a->ldr % 8) != 0 || a->ldr < a->N) return DIT_ERR_ALIGNMENT;
      if (a->gate && (!aligned16(a->gate) || (a->gate_stride % 4) != 0)) return DIT_ERR_ALIGNMENT;
      if (a->C2 != nullptr) return DIT_ERR_INVALID_ARG;
      break;
    default:
      return DIT_ERR_INVALID_ARG;
  }
  return DIT_OK;
}

void gemm_epi(const dit_gemm_args* a, dit::gemm::Epi& ep) {
  ep.C = reinterpret_cast<bf16*>(a->C);
  ep.ldc = a->ldc;
  ep.C2 = reinterpret_cast<bf16*>(a->C2);
  ep.ldc2 = a->ldc2;
  ep.split_col = a->C2 ? a->split_col : a->N;
  ep.bias = reinterpret_cast<const bf16*>(a->bias);
  ep.gelu_col_begin = a->gelu_col_begin;
  ep.gate = a->gate;
  ep.gate_stride = a->gate_stride;
  ep.resid = reinterpret_cast<const bf16*>(a->resid);
  ep.ldr = a->ldr;
  ep.rows_per_batch = a->rows_per_batch > 0 ? a->rows_per_batch : a->M;
  ep.qk_cols = a->qk_cols;
  ep.qk_norm = a->qk_norm;
  ep.qk_eps = a->qk_eps;
  ep.q_scale = reinterpret_cast<const bf16*>(a->q_scale);
  ep.k_scale = reinterpret_cast<const bf16*>(a->k_scale);
  ep.rope = reinterpret_cast<const float2*>(a->rope);
  ep.rope_rows = a->rope_rows > 0 ? a->rope_rows : a->M;
  ep.w_keep = nullptr;
  ep.w_keep_bytes = 0;
}

// One job of the SM-pair kernel: tensor maps, epilogue and tile order.
dit_status pair_job(const dit_gemm_args* a, dit::gemm::pair::PairJob& j) {
  namespace P = dit::gemm::pair;
  dit_status s;
  if ((s = make_map_2d(&j.tmA, a->A, a->M, a->K, a->lda, dit::gemm::BM)) != DIT_OK) return s;
  if ((s = make_map_2d(&j.tmB, a->W, a->N, a->K, a->ldw, P::BN_CTA)) != DIT_OK) return s;
  gemm_epi(a, j.ep);
  j.M = a->M;
  j.N = a->N;
  // walk the larger operand's panels once: N-fastest when A (M x K) is the larger
  j.n_fastest = a->M > a->N ? 1 : 0;
  int dev = 0;
  if (j.n_fastest && cudaGetDevice(&dev) == cudaSuccess && g_dev[dev].keep_weights.load(std::memory_order_relaxed)) {
    // whole 128-byte lines inside the weight: the kernel returns them to normal L2 priority at the end
    const uintptr_t w0 = reinterpret_cast<uintptr_t>(a->W);
    const uintptr_t lo = (w0 + 127) & ~(uintptr_t)127;
    const uintptr_t hi = (w0 + (uintptr_t)a->N * (uintptr_t)a->ldw * 2) & ~(uintptr_t)127;
    if (hi > lo) {
      j.ep.w_keep = reinterpret_cast<const uint8_t*>(lo);
      j.ep.w_keep_bytes = (int64_t)(hi - lo);
    }
  }
  return DIT_OK;
}

dit_status pair_launch(const dit::gemm::pair::PairGroup& G, int epi, int K, int sms, cudaStream_t st) {
  namespace P = dit::gemm::pair;
  int tiles = 0;
  for (int g = 0; g < G.count; ++g)
    tiles += ((G.job[g].M + P::BM - 1) / P::BM) * ((G.job[g].N + P::BN - 1) / P::BN);
  const int clusters = tiles < sms / 2 ? tiles : sms / 2;
  const int grid = 2 * clusters;
  switch (epi) {
    case DIT_EPI_NONE:
      launch_pdl(P::gemm_pair_kernel<DIT_EPI_NONE>, grid, P::NUM_THREADS, P::SMEM_BYTES, st, G, K, g_wait_limit_ns);
      break;
    case DIT_EPI_BIAS:
      launch_pdl(P::gemm_pair_kernel<DIT_EPI_BIAS>, grid, P::NUM_THREADS, P::SMEM_BYTES, st, G, K, g_wait_limit_ns);
      break;
    case DIT_EPI_BIAS_GELU_COLS:
      launch_pdl(P::gemm_pair_kernel<DIT_EPI_BIAS_GELU_COLS>, grid, P::NUM_THREADS, P::SMEM_BYTES, st, G, K,
                 g_wait_limit_ns);
      break;
    default:
      launch_pdl(P::gemm_pair_kernel<DIT_EPI_BIAS_GATED_RESIDUAL>, grid, P::NUM_THREADS, P::SMEM_BYTES, st, G, K,
                 g_wait_limit_ns);
      break;
  }
  return launch_status();
}

}  // namespace

extern "C" {

dit_status dit_gemm_epilogue(const dit_gemm_args* a, void* stream) {
  dit_status s = gemm_validate(a);
  if (s != DIT_OK) return s;
  int sms = 0;
  if ((s = device_setup(&sms)) != DIT_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  // SM-pair kernel (256 x 256 tiles over two CTAs) once there are at least
  // two 128-row blocks; the one-CTA kernel (128 x 256 tiles) otherwise.
  if (a->M > dit::gemm::BM && sms >= 2) {
    dit::gemm::pair::PairGroup G;
    G.count = 1;
    if ((s = pair_job(a, G.job[0])) != DIT_OK) return s;
    G.job[1] = G.job[0];
    return pair_launch(G, a->epi, a->K, sms, st);
  }
  CUtensorMap tA, tB;
  if ((s = make_map_2d(&tA, a->A, a->M, a->K, a->lda, dit::gemm::BM)) != DIT_OK) return s;
  if ((s = make_map_2d(&tB, a->W, a->N, a->K, a->ldw, dit::gemm::BN)) != DIT_OK) return s;
  dit::gemm::Epi ep;
  gemm_epi(a, ep);
  const int tiles = ((a->M + dit::gemm::BM - 1) / dit::gemm::BM) * ((a->N + dit::gemm::BN - 1) / dit::gemm::BN);
  const int grid = tiles < sms ? tiles : sms;
  const int smem = dit::gemm::SMEM_BYTES;
  const int nt = dit::gemm::NUM_THREADS;
  switch (a->epi) {
    case DIT_EPI_NONE:
      dit::gemm::gemm_kernel<DIT_EPI_NONE><<<grid, nt, smem, st>>>(tA, tB, a->M, a->N, a->K, ep, g_wait_limit_ns);
      break;
    case DIT_EPI_BIAS:
      dit::gemm::gemm_kernel<DIT_EPI_BIAS><<<grid, nt, smem, st>>>(tA, tB, a->M, a->N, a->K, ep, g_wait_limit_ns);
      break;
    case DIT_EPI_BIAS_GELU_COLS:
      dit::gemm::gemm_kernel<DIT_EPI_BIAS_GELU_COLS><<<grid, nt, smem, st>>>(tA, tB, a->M, a->N, a->K, ep,
                                                                            g_wait_limit_ns);
      break;
    default:
      dit::gemm::gemm_kernel<DIT_EPI_BIAS_GATED_RESIDUAL><<<grid, nt, smem, st>>>(tA, tB, a->M, a->N, a->K, ep,
                                                                                 g_wait_limit_ns);
      break;
  }
  return launch_status();
}

dit_status dit_gemm_epilogue_grouped(const dit_gemm_args* a, const dit_gemm_args* b, void* stream) {
  dit_status s;
  if ((s = gemm_validate(a)) != DIT_OK) return s;
  if ((s = gemm_validate(b)) != DIT_OK) return s;
  if (a->epi != b->epi || a->K != b->K) return DIT_ERR_INVALID_ARG;
  int sms = 0;
  if ((s = device_setup(&sms)) != DIT_OK) return s;
  if (a->M <= dit::gemm::BM || b->M <= dit::gemm::BM || sms < 2) {
    // a job this small runs on the one-CTA kernel: two launches
    if ((s = dit_gemm_epilogue(a, stream)) != DIT_OK) return s;
    return dit_gemm_epilogue(b, stream);
  }
  dit::gemm::pair::PairGroup G;
  G.count = 2;
  if ((s = pair_job(a, G.job[0])) != DIT_OK) return s;
  if ((s = pair_job(b, G.job[1])) != DIT_OK) return s;
  return pair_launch(G, a->epi, a->K, sms, (cudaStream_t)stream);
}

}  // extern "C"

#include "blocks.inc"
