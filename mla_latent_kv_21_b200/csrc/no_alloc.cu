// A decode entry point for callers that cannot allocate device memory.
//
// mla_decode_run needs a caller-provided workspace (the absorbed query rows,
// the per-split partial results and a small header). Some callers cannot
// obtain one at the point where they run a decode step: an inference engine
// that reserves the whole device for its own memory pool up front and forbids
// side allocations, or a latency-critical loop that cannot afford the
// device-wide synchronisation cudaMalloc / cudaFree may imply. For them,
// mla_decode_run_no_alloc uses a fixed scratch array that lives in this
// library's device image instead of a workspace.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes
// (32 MiB). Every GPU that loads the library holds it until the process exits.
// In host code the name mla_no_alloc_scratch is only a host-side stand-in, not
// a device address, so its device address is fetched once per device with
// cudaGetSymbolAddress (with that device current) and handed to the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char mla_no_alloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// A failed set-up step returns MLA_ERR_CUDA after taking its error off the
// runtime's last-error slot, so that it does not surface later as the launch
// error of an unrelated run.
mla_status_t setup_failed() {
  (void)cudaGetLastError();
  return MLA_ERR_CUDA;
}

// Resolves (once per device) the device address of the scratch array and
// clears its header so that the device status word starts at zero. The
// address is cached per device index for the life of the process, which
// assumes the device's primary context (the one the CUDA runtime uses) and no
// cudaDeviceReset between calls: a new context may place the array elsewhere.
mla_status_t scratch_for_current_device(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, mla_no_alloc_scratch) != cudaSuccess || !p) return setup_failed();
    if (cudaMemset(p, 0, 1024) != cudaSuccess) return setup_failed();
    if (cudaDeviceSynchronize() != cudaSuccess) return setup_failed();
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_run_no_alloc(mla_plan_t plan, const void* q_nope,
                                                const void* q_rope, const void* kv_cache,
                                                int64_t num_blocks, const int32_t* block_table,
                                                int32_t block_table_stride,
                                                const int32_t* seq_lens_dev, const void* w_uk,
                                                const void* w_uv, void* out, void* stream) {
  if (!plan) return MLA_ERR_INVALID_ARG;
  mla_plan_info_t info;
  mla_status_t st = mla_plan_get_info(plan, &info);
  if (st != MLA_OK) return st;
  // the FP8 cache has its own entry point (mla_decode_run_fp8), which this one
  // does not wrap
  if (mla::plan_is_fp8(plan)) return MLA_ERR_UNSUPPORTED;
  // the plan's scratch must fit in the fixed array
  if (info.workspace_bytes > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != MLA_OK) return st;
  return mla_decode_run(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                        block_table_stride, seq_lens_dev, w_uk, w_uv, out, scratch,
                        kNoAllocScratchBytes, stream);
}
