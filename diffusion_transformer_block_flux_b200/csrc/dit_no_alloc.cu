// dit_single_block_fwd_noalloc: the single-stream block forward for callers
// that are not allowed to allocate device memory.
//
// Who needs this: code that runs as a plug-in inside a host framework which
// owns every byte of device memory through its own pool (a raw cudaMalloc
// would bypass the pool's accounting and can fail or fragment it), and
// latency-critical serving loops that may not allocate once they are running
// (cudaMalloc and cudaFree can synchronise the device and stall every other
// stream).  Such callers still pass their inputs and outputs, but cannot
// hand us the intermediate workspace that dit_single_block_fwd needs.
//
// Instead, the intermediates live in one file-scope device array of fixed
// size, g_noalloc_scratch (16 MiB), which every device that loads the library
// keeps until the process exits.  Host code cannot use the array's name as a
// device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (that device must be current) and remembers it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/dit.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once
// per device).
dit_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DIT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DIT_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DIT_OK;
}

}  // namespace

extern "C" {

#if defined(__GNUC__)
__attribute__((visibility("default")))
#endif
dit_status dit_single_block_fwd_noalloc(const dit_block_cfg* cfg, const dit_single_weights* w, const dit_bf16* x,
                                        const dit_bf16* vec, const float* rope, dit_bf16* out, void* stream) {
  if (cfg == nullptr) return DIT_ERR_INVALID_ARG;
  const size_t need = dit_single_block_workspace(cfg);
  // An invalid configuration: let the workspace entry point report it, so that
  // both calls give the same status for the same bad input (its checks come
  // before any use of the workspace, and it enqueues nothing when they fail).
  if (need == 0) return dit_single_block_fwd(cfg, w, x, vec, rope, out, nullptr, 0, stream);
  if (need > kScratchBytes) return DIT_ERR_WORKSPACE;  // the block's intermediates do not fit in 16 MiB
  void* scratch = nullptr;
  dit_status s = scratch_address(&scratch);
  if (s != DIT_OK) return s;
  // Every intermediate the block reads is written earlier in the same call,
  // so the leftovers of the previous call need no clearing.
  return dit_single_block_fwd(cfg, w, x, vec, rope, out, scratch, kScratchBytes, stream);
}

}  // extern "C"
