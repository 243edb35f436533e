// nvfp4_linear_noalloc: the NVFP4 linear forward for callers that cannot allocate
// device memory themselves, for instance a plugin whose host application owns all
// device memory and forbids allocations on its hot path, a serving loop that must
// never enter the allocator (which can synchronise the device or fail under memory
// pressure), or a plain C caller with no memory manager of its own.
//
// Instead of a caller-provided workspace it uses one fixed scratch array in device
// global memory, defined below. Every GPU that loads this library keeps that array
// (kNoallocScratchBytes) until the process exits. All calls on a device share it:
// two calls whose kernels overlap on the GPU (different streams without ordering)
// race on it and give wrong results. Each call rewrites every byte of scratch it
// reads, so nothing has to be cleared between calls.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/qlinear.h"
#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB per device

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device (that device current) and kept.
uint8_t* scratch_on_current_device(int* status) {
  static uint8_t* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    ql::set_error_text("nvfp4_linear_noalloc: no usable current device");
    *status = QL_ERR_LAUNCH;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // leave no error pending for the caller's next check
      char msg[200];
      std::snprintf(msg, sizeof(msg), "nvfp4_linear_noalloc: cudaGetSymbolAddress failed: %s",
                    cudaGetErrorString(e));
      ql::set_error_text(msg);
      *status = QL_ERR_LAUNCH;
      return nullptr;
    }
    cache[dev] = static_cast<uint8_t*>(p);
  }
  *status = QL_OK;
  return cache[dev];
}

}  // namespace

extern "C" int nvfp4_linear_noalloc(const void* x, int64_t M, int64_t K, const uint8_t* w,
                                    const uint8_t* w_scale, int64_t N,
                                    const float* weight_scale_2, const float* input_scale,
                                    const float* bias, void* y, ql_stream_t stream) {
  if (!x || !w || !w_scale || !weight_scale_2 || !input_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  const size_t need = nvfp4_linear_workspace_size(M, K, N);
  if (need == 0) {
    ql::set_error_text("nvfp4_linear_noalloc: needs K >= 32 and K % 32 == 0");
    return QL_ERR_SHAPE;
  }
  if (need > kNoallocScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "nvfp4_linear_noalloc: this problem needs %zu bytes of scratch, more than the "
                  "%zu bytes this entry point holds; call nvfp4_linear with a workspace instead",
                  need, kNoallocScratchBytes);
    ql::set_error_text(msg);
    return QL_ERR_WORKSPACE;
  }
  // an sm_100 device first: elsewhere the scratch lookup itself would fail
  int status = ql::check_current_device(nullptr);
  if (status != QL_OK) return status;
  uint8_t* scratch = scratch_on_current_device(&status);
  if (!scratch) return status;
  return nvfp4_linear(x, M, K, w, w_scale, N, weight_scale_2, input_scale, bias, y, scratch,
                      kNoallocScratchBytes, stream);
}
