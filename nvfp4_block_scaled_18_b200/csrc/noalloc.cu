// nvfp4_rmsnorm_reorder_quantize_noalloc: the fused RMSNorm + reorder +
// quantize entry point for callers that cannot allocate device memory.
//
// The regular entry point takes a caller-owned workspace (reduction cells and
// one fp32 rinv per row).  Some callers cannot provide one: plugins embedded
// in a host framework that owns every device allocation, and real-time paths
// that must never call the allocator.  This variant keeps the
// same scratch in a file-scope device array that lives as long as the library
// is loaded, so it allocates nothing at all.
//
// Properties of the built-in scratch:
//  * capacity: NVFP4_NOALLOC_MAX_ROWS rows (M); larger M is rejected with
//    NVFP4_ERR_WORKSPACE before anything is enqueued;
//  * every GPU that loads the library holds its own copy until process exit;
//  * one array is shared by every call on a device, and it keeps whatever the
//    last call left in it: the reduction cells are cleared (cudaMemsetAsync)
//    on the call's stream at the start of each call, and calls that overlap on
//    the GPU (different streams without ordering) race on it;
//  * the first call on a device resolves the array's device address with
//    cudaGetSymbolAddress while that device is current.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4.h"

using namespace nvfp4;

namespace {

constexpr int64_t kMaxRows = NVFP4_NOALLOC_MAX_ROWS;
constexpr size_t kScratchBytes = kWsHeaderBytes + (size_t)kMaxRows * 4;

// Library-owned scratch: 256-byte reduction header + one fp32 rinv per row.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device (resolved once per device).
nvfp4_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_rmsnorm_reorder_quantize_noalloc(
    const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
    const int32_t* perm, int64_t S, const float* scale_in, nvfp4_tensor* x_aug, int* dev_status,
    void* stream) {
  if (M > kMaxRows) return NVFP4_ERR_WORKSPACE;
  // reject bad arguments before anything is enqueued (the regular entry point
  // checks them again)
  const size_t esize = dt == NVFP4_BF16 ? 2 : 4;
  if (x == nullptr || (dt != NVFP4_BF16 && dt != NVFP4_F32) || M <= 0 || K <= 0 || ldx < K || K % 16 != 0 ||
      S < 0 || S > K || S % 16 != 0 || x_aug == nullptr || x_aug->codes == nullptr || x_aug->scales == nullptr ||
      x_aug->tensor_scale == nullptr || x_aug->rows != M || x_aug->cols != K + S ||
      (gamma != nullptr && !(eps >= 0.0f)))
    return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || ((size_t)ldx * esize) % 16 != 0 ||
      (reinterpret_cast<uintptr_t>(x_aug->codes) & 15u) || (reinterpret_cast<uintptr_t>(x_aug->scales) & 15u) ||
      (gamma != nullptr && (reinterpret_cast<uintptr_t>(gamma) & 15u)))
    return NVFP4_ERR_ALIGNMENT;
  if (reorder_smem_bytes(dt, K, gamma != nullptr) > 200 * 1024 || K > 65536) return NVFP4_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  nvfp4_status st = scratch_address(&scratch);
  if (st != NVFP4_OK) return st;
  // the reduction cells must start at zero; the rinv rows are fully rewritten
  if (cudaMemsetAsync(scratch, 0, kWsHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  return nvfp4_rmsnorm_reorder_quantize(x, dt, M, K, ldx, gamma, eps, perm, S, scale_in, x_aug, scratch,
                                        kScratchBytes, dev_status, stream);
}
