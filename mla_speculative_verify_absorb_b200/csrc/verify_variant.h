// Internal interface of the split-verify variant's kernels: the masked
// tree-block attention (verify_tree_block.cu), the two-state LSE merge and
// the stacked R-state merge of KV-sequence shards (verify_merge.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace va {

struct TreeBlockParams {
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
  int32_t batch, num_heads, max_tree;
  int64_t max_kv_per_req, pool_slots;
  float scale_log2;          // sm_scale * log2(e)
  int32_t exclude_self;      // 1: the node's own key is left to the dense pass
  uint16_t* out;             // bf16 [sumT, H, 512] normalised tree-block output, or
  float* out_f32;            // fp32 [sumT, H, 512] contiguous (used when non-null)
  int64_t out_tok, out_head;
  float* lse;                // [sumT, H], natural log; -inf for an empty key set
  uint64_t* self_anc;        // or null: receives 1 << t for every node t
  int32_t* visible_count;    // or null: prefix + tree keys this pair of passes attends
  uint32_t* status;
};

struct MergeParams {
  const uint16_t* o_a;
  int64_t a_tok, a_head;
  const float* lse_a;        // [tokens, H]
  const void* o_b;           // bf16, or fp32 when b_f32
  int64_t b_tok, b_head;
  int32_t b_f32;
  const float* lse_b;
  uint16_t* out;             // may alias o_a or o_b
  int64_t out_tok, out_head;
  float* lse;                // or null
  int64_t max_tokens;
  const int32_t* num_tokens; // or null: device-side token count (<= max_tokens)
  int32_t num_heads;
};

struct MergeStackedParams {
  const uint16_t* o;         // bf16 [R, max_tokens, H, 512] contiguous
  const float* lse;          // [R, max_tokens, H]
  int32_t num_states;        // R >= 1
  uint16_t* out;             // bf16 [tokens, H, 512], strides in elements
  int64_t out_tok, out_head;
  float* lse_out;            // or null
  int64_t max_tokens;
  const int32_t* num_tokens; // or null
  int32_t num_heads;
};

cudaError_t launch_merge_stacked(const MergeStackedParams& p, cudaStream_t stream);
cudaError_t launch_tree_block(const TreeBlockParams& p, int64_t max_tokens, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);

}  // namespace va
