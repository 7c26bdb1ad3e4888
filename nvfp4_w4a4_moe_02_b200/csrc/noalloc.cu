// weight_qdq_noalloc: the trainer fake-quant entry point for callers that cannot allocate.
//
// weight_qdq needs a small device workspace for its per-tensor amax partials.  This variant
// keeps that scratch in a fixed array that lives in the library's own device image, so the
// caller passes only its inputs and outputs.  The array holds kNoAllocScratchFloats floats
// (16 KiB) on every GPU that loads the library, for the life of the process.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4rac.h"

namespace nvfp4 {
nvfp4_status record_host_error(nvfp4_status s, const char* msg);
void clear_host_error();
int qdq_partial_count(int64_t n_tensors);
int device_sm_count();
}  // namespace nvfp4

namespace {

constexpr int64_t kNoAllocScratchFloats = 4096;

// Shared by every call on a device; each call overwrites the partials it reads.
static __device__ __align__(256) float g_qdq_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once per device.  In
// host code the array's name only stands in for the symbol; the kernels need this address.
// The cached address belongs to the device's primary context: after cudaDeviceReset (or any
// teardown of that context) it is stale, and a later call would launch on a dangling pointer.
nvfp4_status scratch_on_current_device(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "cudaGetDevice failed: %s", cudaGetErrorString(e));
    return nvfp4::record_host_error(NVFP4_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) return nvfp4::record_host_error(NVFP4_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_qdq_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the scratch array failed: %s", cudaGetErrorString(e));
      return nvfp4::record_host_error(NVFP4_ERR_CUDA, msg);
    }
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status weight_qdq_noalloc(const uint16_t* w, int64_t n_tensors, int64_t elems_per_tensor,
                                           uint16_t* w_out, float* s_g_out, int32_t* dev_status, void* stream) {
  nvfp4::clear_host_error();
  if (!w || !w_out) return nvfp4::record_host_error(NVFP4_ERR_INVALID_ARG, "w / w_out is NULL");
  if (n_tensors <= 0 || elems_per_tensor <= 0 || elems_per_tensor % 16 != 0)
    return nvfp4::record_host_error(NVFP4_ERR_UNSUPPORTED_SHAPE,
                                    "n_tensors > 0 and elems_per_tensor % 16 == 0 required");
  if ((reinterpret_cast<uintptr_t>(w) & 15u) != 0 || (reinterpret_cast<uintptr_t>(w_out) & 15u) != 0)
    return nvfp4::record_host_error(NVFP4_ERR_ALIGNMENT, "w / w_out must be 16-byte aligned");
  const int P = nvfp4::qdq_partial_count(n_tensors);
  const int64_t need = n_tensors * (int64_t)P;
  if (need > kNoAllocScratchFloats) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "weight_qdq_noalloc: n_tensors = %lld needs %lld scratch floats, the fixed scratch holds %lld "
             "(at most 4096 tensors per call); use weight_qdq with a workspace",
             (long long)n_tensors, (long long)need, (long long)kNoAllocScratchFloats);
    return nvfp4::record_host_error(NVFP4_ERR_UNSUPPORTED_SHAPE, msg);
  }
  float* scratch = nullptr;
  nvfp4_status st = scratch_on_current_device(&scratch);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // every partial the qdq kernel reads is written by the amax kernel first: nothing to clear
  cudaError_t e = nvfp4::launch_amax(w, n_tensors, 1, elems_per_tensor, elems_per_tensor, scratch, P, dev_status, s);
  if (e == cudaSuccess)
    e = nvfp4::launch_qdq(w, n_tensors, elems_per_tensor, w_out, scratch, P, s_g_out, dev_status,
                          nvfp4::device_sm_count(), s);
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "weight_qdq_noalloc launch: %s", cudaGetErrorString(e));
    return nvfp4::record_host_error(NVFP4_ERR_CUDA, msg);
  }
  return NVFP4_OK;
}
