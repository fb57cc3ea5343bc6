// verify_attn_forward_static: the split + reduce call for callers that cannot
// allocate device memory, using a workspace that is part of the library
// image instead of one the caller provides.
//
// Some callers cannot call cudaMalloc when they need this call: a serving
// loop that has to stay allocation-free once its CUDA graphs are warm, an
// embedding runtime that owns the device heap and forbids other allocators,
// or a plugin that only receives tensors it may read and write. They still
// pass their inputs and outputs; the scratch the split kernel needs for its
// partial states comes from the array below.
//
// The array is file-scope `static __device__` storage of a fixed size, so
// every GPU on which the library is used holds it until the process exits.
// In host code its name is only a host-side stand-in, never a device
// address: the address is obtained once per device with
// cudaGetSymbolAddress, with that device current, and that pointer is what
// the kernels receive.
#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_attn.h"
#include "verify_attn_internal.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_workspace[VERIFY_ATTN_STATIC_WS_BYTES];

void* g_static_ptr[kMaxDevices] = {nullptr};

// Set-up, once per device: resolve the device address of the array.
int static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  if (!g_static_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return VERIFY_ATTN_CUDA_ERROR;
    }
    g_static_ptr[dev] = ptr;
  }
  *out = g_static_ptr[dev];
  return VERIFY_ATTN_OK;
}

}  // namespace

extern "C" int verify_attn_forward_static(const verify_attn_plan_t* plan, const verify_attn_args* args,
                                          uint32_t* status, verify_attn_stream_t stream) {
  if (!plan || !args) return VERIFY_ATTN_EINVAL;
  if (plan->ws_bytes > (int64_t)VERIFY_ATTN_STATIC_WS_BYTES) return VERIFY_ATTN_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  int rc = static_workspace(&ws);
  if (rc) return rc;
  const size_t ws_bytes = VERIFY_ATTN_STATIC_WS_BYTES;
  // The array keeps the previous call's contents: clear the status word, the
  // only part that must start at zero (every partial state the reduce reads
  // is written by the same call's split kernel).
  rc = verify_attn_workspace_init(plan, ws, ws_bytes, stream);
  if (rc) return rc;
  rc = verify_attn_run(plan, args, ws, ws_bytes, stream);
  if (rc) return rc;
  rc = verify_attn_reduce(plan, args, ws, ws_bytes, stream);
  if (rc) return rc;
  if (status &&
      cudaMemcpyAsync(status, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}
