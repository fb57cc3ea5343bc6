// Internal interface of the KV relocation kernel (verify_defrag.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace va {

struct DefragParams {
  uint16_t* kv_pool;
  int64_t kv_stride, pool_slots;
  int32_t* kv_indices;
  const int32_t* kv_indptr;
  const int32_t* dst_begin;
  int32_t batch, budget;
  uint32_t* status;          // or null
};

// Grid sized for max_total positions (any total is processed, grid-stride).
cudaError_t launch_defrag(const DefragParams& p, int64_t max_total, cudaStream_t stream);

}  // namespace va
