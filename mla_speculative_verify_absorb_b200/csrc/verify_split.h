// Launch interface of the split and reduce kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace va {

struct SplitParams {
  const uint16_t* q_latent;
  int64_t ql_tok, ql_head;
  const uint16_t* q_rope;
  int64_t qr_tok, qr_head;
  const uint16_t* kv_pool;
  int64_t kv_stride;
  const int32_t* kv_indices;
  const int32_t* kv_indptr;
  const int32_t* qo_indptr;
  const uint64_t* tree_anc;
  int32_t batch, num_heads, max_tree, num_clusters;
  int64_t max_kv_per_req, pool_slots;
  float scale_log2;          // sm_scale * log2(e): scores are kept in log2 units
  int32_t num_slots;
  uint32_t* status;          // workspace status word
  float4* meta;              // [num_slots, 128] {m, l, count, 0}
  float* partial;            // [num_slots, 128, 512]
  const uint16_t* stage;     // [stage_rows, 576] gathered KV rows (verify_gather.cu)
  int64_t stage_rows;
};

// KV gather into the staging rows of the workspace.
struct GatherParams {
  const uint16_t* kv_pool;
  int64_t kv_stride;
  const int32_t* kv_indices;
  const int32_t* kv_indptr;
  const int32_t* qo_indptr;
  int32_t batch, max_tree;
  int64_t max_kv_per_req, pool_slots;
  uint32_t* status;
  uint16_t* stage;
  int64_t stage_tiles;       // capacity of `stage` in key tiles
};

struct ReduceParams {
  const int32_t* kv_indptr;
  const int32_t* qo_indptr;
  const uint64_t* tree_anc;
  int32_t batch, num_heads, max_tree, num_clusters;
  int64_t max_kv_per_req;
  int32_t row_tiles_per_req, num_slots;
  uint32_t* status;
  const float4* meta;
  const float* partial;
  uint16_t* out;
  int64_t out_tok, out_head;
  float* lse;
  int32_t* visible_count;
};

int split_smem_bytes();
cudaError_t split_max_active_clusters(int* n);
cudaError_t launch_split(const SplitParams& p, cudaStream_t stream);
cudaError_t launch_gather(const GatherParams& p, int grid, cudaStream_t stream);
cudaError_t launch_reduce(const ReduceParams& p, cudaStream_t stream);
cudaError_t launch_tree_mask(const int32_t* parents, const int32_t* qo_indptr, int32_t batch, uint64_t* anc,
                             uint32_t* status, cudaStream_t stream);

}  // namespace va
