// Host side of the C ABI declared in include/verify_attn.h: plan, argument
// checks, launches, the tree-mask helper, status and error strings.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "verify_attn.h"
#include "verify_attn_internal.h"
#include "verify_split.h"
#include "verify_defrag.h"
#include "verify_variant.h"

namespace {

constexpr int64_t kAlign = 256;

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool row_stride_ok(int64_t s) { return s > 0 && (s % 8) == 0; }

int check_plan(const verify_attn_plan_t* plan) {
  if (!plan || plan->version != VERIFY_ATTN_PLAN_VERSION || plan->num_clusters < 1 || plan->num_slots < 1)
    return VERIFY_ATTN_EINVAL;
  return VERIFY_ATTN_OK;
}

int check_args(const verify_attn_plan_t* plan, const verify_attn_args* a, const void* ws, size_t ws_bytes,
               bool need_out) {
  int rc = check_plan(plan);
  if (rc) return rc;
  if (!a || !ws) return VERIFY_ATTN_EINVAL;
  if ((int64_t)ws_bytes < plan->ws_bytes) return VERIFY_ATTN_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return VERIFY_ATTN_EINVAL;
  if (a->batch < 1 || a->batch > plan->max_batch) return VERIFY_ATTN_EINVAL;
  if (!a->q_latent || !a->q_rope || !a->kv_pool || !a->kv_indices || !a->kv_indptr || !a->qo_indptr ||
      !a->tree_anc)
    return VERIFY_ATTN_EINVAL;
  if (!aligned16(a->q_latent) || !aligned16(a->q_rope) || !aligned16(a->kv_pool)) return VERIFY_ATTN_EINVAL;
  if (!row_stride_ok(a->q_latent_stride_tok) || !row_stride_ok(a->q_latent_stride_head) ||
      !row_stride_ok(a->q_rope_stride_tok) || !row_stride_ok(a->q_rope_stride_head) ||
      !row_stride_ok(a->kv_row_stride) || a->kv_row_stride < va::kDQK)
    return VERIFY_ATTN_EINVAL;
  if (need_out) {
    if (!a->out || !aligned16(a->out)) return VERIFY_ATTN_EINVAL;
    if (!row_stride_ok(a->out_stride_tok) || !row_stride_ok(a->out_stride_head)) return VERIFY_ATTN_EINVAL;
  }
  return VERIFY_ATTN_OK;
}

}  // namespace

extern "C" {

int verify_attn_plan(const verify_attn_params* params, verify_attn_plan_t* plan, size_t* ws_bytes) {
  if (!params || !plan || !ws_bytes) return VERIFY_ATTN_EINVAL;
  const verify_attn_params& q = *params;
  if (q.d_latent != VERIFY_ATTN_D_LATENT || q.d_rope != VERIFY_ATTN_D_ROPE) return VERIFY_ATTN_UNSUPPORTED;
  if (q.max_tree < 1 || q.num_heads < 1 || q.max_batch < 1) return VERIFY_ATTN_EINVAL;
  if (q.max_tree > VERIFY_ATTN_MAX_TREE || q.num_heads > VERIFY_ATTN_MAX_HEADS) return VERIFY_ATTN_UNSUPPORTED;
  if (q.max_kv_per_req < q.max_tree || q.max_kv_per_req > INT32_MAX) return VERIFY_ATTN_EINVAL;
  if (q.max_total_kv < q.max_tree || q.max_total_kv > INT32_MAX) return VERIFY_ATTN_EINVAL;
  if (q.pool_slots < 1 || q.pool_slots > INT32_MAX) return VERIFY_ATTN_EINVAL;
  if (!(q.sm_scale > 0.f) || !isfinite(q.sm_scale)) return VERIFY_ATTN_EINVAL;

  // Persistent CTA pairs: half the SMs, or fewer if the device cannot keep
  // that many clusters of two resident at once (so there is never a second wave).
  int num_sms = q.num_sms;
  int64_t resident = INT32_MAX;
  if (num_sms == 0) {
    int dev = 0, active = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        va::split_max_active_clusters(&active) != cudaSuccess) {
      cudaGetLastError();
      return VERIFY_ATTN_CUDA_ERROR;
    }
    if (active >= 1) resident = active;
  }
  if (num_sms < 2) return VERIFY_ATTN_EINVAL;

  const int64_t row_tiles = ((int64_t)q.max_tree * q.num_heads + va::kRowsPerTile - 1) / va::kRowsPerTile;
  const int64_t key_tiles_req = (q.max_kv_per_req + va::kKeysPerTile - 1) / va::kKeysPerTile;
  const int64_t key_tiles_total = (q.max_total_kv + va::kKeysPerTile - 1) / va::kKeysPerTile + q.max_batch;
  int64_t units = (int64_t)q.max_batch * row_tiles * key_tiles_req;
  if (row_tiles * key_tiles_total < units) units = row_tiles * key_tiles_total;
  int64_t clusters = num_sms / 2;
  if (resident < clusters) clusters = resident;
  if (units < clusters) clusters = units;
  if (clusters < 1) clusters = 1;
  const int64_t slots = clusters + (int64_t)q.max_batch * row_tiles;
  if (slots > INT32_MAX) return VERIFY_ATTN_UNSUPPORTED;
  // Staging rows: every request padded to whole key tiles (TMA row
  // coordinates are 32-bit).
  const int64_t stage_rows = key_tiles_total * va::kKeysPerTile;
  if (stage_rows > INT32_MAX) return VERIFY_ATTN_UNSUPPORTED;

  memset(plan, 0, sizeof(*plan));
  plan->version = VERIFY_ATTN_PLAN_VERSION;
  plan->num_heads = q.num_heads;
  plan->max_batch = q.max_batch;
  plan->max_tree = q.max_tree;
  plan->max_kv_per_req = q.max_kv_per_req;
  plan->max_total_kv = q.max_total_kv;
  plan->pool_slots = q.pool_slots;
  plan->sm_scale = q.sm_scale;
  plan->num_clusters = (int32_t)clusters;
  plan->rows_per_tile = va::kRowsPerTile;
  plan->keys_per_tile = va::kKeysPerTile;
  plan->row_tiles_per_req = (int32_t)row_tiles;
  plan->num_slots = (int32_t)slots;
  plan->ws_meta_offset = va::kWsHeaderBytes;
  plan->ws_partial_offset = round_up(plan->ws_meta_offset + slots * va::kRowsPerTile * 16, kAlign);
  plan->ws_stage_offset = round_up(plan->ws_partial_offset + slots * va::kRowsPerTile * va::kDLatent * 4, 1024);
  plan->stage_rows = stage_rows;
  plan->ws_bytes = plan->ws_stage_offset + stage_rows * va::kDQK * 2;
  plan->split_smem_bytes = va::split_smem_bytes();
  *ws_bytes = (size_t)plan->ws_bytes;
  return VERIFY_ATTN_OK;
}

int verify_attn_workspace_init(const verify_attn_plan_t* plan, void* ws, size_t ws_bytes,
                               verify_attn_stream_t stream) {
  int rc = check_plan(plan);
  if (rc) return rc;
  if (!ws) return VERIFY_ATTN_EINVAL;
  if ((int64_t)ws_bytes < plan->ws_bytes) return VERIFY_ATTN_WORKSPACE_TOO_SMALL;
  if (cudaMemsetAsync(ws, 0, va::kWsHeaderBytes, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

namespace {

void fill_split(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws, va::SplitParams& p) {
  p.q_latent = a->q_latent;
  p.ql_tok = a->q_latent_stride_tok;
  p.ql_head = a->q_latent_stride_head;
  p.q_rope = a->q_rope;
  p.qr_tok = a->q_rope_stride_tok;
  p.qr_head = a->q_rope_stride_head;
  p.kv_pool = a->kv_pool;
  p.kv_stride = a->kv_row_stride;
  p.kv_indices = a->kv_indices;
  p.kv_indptr = a->kv_indptr;
  p.qo_indptr = a->qo_indptr;
  p.tree_anc = a->tree_anc;
  p.batch = a->batch;
  p.num_heads = plan->num_heads;
  p.max_tree = plan->max_tree;
  p.num_clusters = plan->num_clusters;
  p.max_kv_per_req = plan->max_kv_per_req;
  p.pool_slots = plan->pool_slots;
  p.scale_log2 = plan->sm_scale * 1.4426950408889634f;
  p.num_slots = plan->num_slots;
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.status = reinterpret_cast<uint32_t*>(base);
  p.meta = reinterpret_cast<float4*>(base + plan->ws_meta_offset);
  p.partial = reinterpret_cast<float*>(base + plan->ws_partial_offset);
  p.stage = reinterpret_cast<const uint16_t*>(base + plan->ws_stage_offset);
  p.stage_rows = plan->stage_rows;
}

cudaError_t launch_gather_for(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws,
                              cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  va::GatherParams gp;
  gp.kv_pool = a->kv_pool;
  gp.kv_stride = a->kv_row_stride;
  gp.kv_indices = a->kv_indices;
  gp.kv_indptr = a->kv_indptr;
  gp.qo_indptr = a->qo_indptr;
  gp.batch = a->batch;
  gp.max_tree = plan->max_tree;
  gp.max_kv_per_req = plan->max_kv_per_req;
  gp.pool_slots = plan->pool_slots;
  gp.status = reinterpret_cast<uint32_t*>(base);
  gp.stage = reinterpret_cast<uint16_t*>(base + plan->ws_stage_offset);
  // A grid of a few CTAs per SM loops over the key tiles of the call.
  const int64_t tiles = plan->stage_rows / va::kKeysPerTile;
  gp.stage_tiles = tiles;
  const int64_t grid = tiles < (int64_t)plan->num_clusters * 8 ? tiles : (int64_t)plan->num_clusters * 8;
  return va::launch_gather(gp, (int)grid, stream);
}

}  // namespace

int verify_attn_gather(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws, size_t ws_bytes,
                       verify_attn_stream_t stream) {
  int rc = check_args(plan, a, ws, ws_bytes, false);
  if (rc) return rc;
  if (launch_gather_for(plan, a, ws, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_split(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws, size_t ws_bytes,
                      verify_attn_stream_t stream) {
  int rc = check_args(plan, a, ws, ws_bytes, false);
  if (rc) return rc;
  va::SplitParams p;
  fill_split(plan, a, ws, p);
  if (va::launch_split(p, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_run(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws, size_t ws_bytes,
                    verify_attn_stream_t stream) {
  int rc = check_args(plan, a, ws, ws_bytes, false);
  if (rc) return rc;
  va::SplitParams p;
  fill_split(plan, a, ws, p);
  if (launch_gather_for(plan, a, ws, (cudaStream_t)stream) != cudaSuccess ||
      va::launch_split(p, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_reduce(const verify_attn_plan_t* plan, const verify_attn_args* a, void* ws, size_t ws_bytes,
                       verify_attn_stream_t stream) {
  int rc = check_args(plan, a, ws, ws_bytes, true);
  if (rc) return rc;
  va::ReduceParams p;
  p.kv_indptr = a->kv_indptr;
  p.qo_indptr = a->qo_indptr;
  p.tree_anc = a->tree_anc;
  p.batch = a->batch;
  p.num_heads = plan->num_heads;
  p.max_tree = plan->max_tree;
  p.num_clusters = plan->num_clusters;
  p.max_kv_per_req = plan->max_kv_per_req;
  p.row_tiles_per_req = plan->row_tiles_per_req;
  p.num_slots = plan->num_slots;
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.status = reinterpret_cast<uint32_t*>(base);
  p.meta = reinterpret_cast<const float4*>(base + plan->ws_meta_offset);
  p.partial = reinterpret_cast<const float*>(base + plan->ws_partial_offset);
  p.out = a->out;
  p.out_tok = a->out_stride_tok;
  p.out_head = a->out_stride_head;
  p.lse = a->lse;
  p.visible_count = a->visible_count;
  if (va::launch_reduce(p, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_build_tree_mask(const int32_t* parents_h, int32_t T, uint64_t* anc_h) {
  if (!parents_h || !anc_h) return VERIFY_ATTN_EINVAL;
  if (T < 1 || T > VERIFY_ATTN_MAX_TREE) return VERIFY_ATTN_EINVAL;
  if (parents_h[0] != -1) return VERIFY_ATTN_EINVAL;
  for (int32_t i = 1; i < T; ++i)
    if (parents_h[i] < 0 || parents_h[i] >= i) return VERIFY_ATTN_EINVAL;
  // Parents precede children, so one forward pass suffices: a node's mask is
  // its parent's mask plus its own bit.
  uint64_t tmp[VERIFY_ATTN_MAX_TREE];
  tmp[0] = 1ull;
  for (int32_t i = 1; i < T; ++i) tmp[i] = tmp[parents_h[i]] | (1ull << i);
  memcpy(anc_h, tmp, sizeof(uint64_t) * (size_t)T);
  return VERIFY_ATTN_OK;
}

int verify_attn_build_tree_mask_device(const int32_t* parents, const int32_t* qo_indptr, int32_t batch,
                                       uint64_t* anc, uint32_t* status, verify_attn_stream_t stream) {
  if (!parents || !qo_indptr || !anc || batch < 1) return VERIFY_ATTN_EINVAL;
  if (va::launch_tree_mask(parents, qo_indptr, batch, anc, status, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_tree_block(const verify_attn_plan_t* plan, const verify_attn_args* a, int exclude_self,
                           uint64_t* self_anc, float* out_f32, void* ws, size_t ws_bytes,
                           verify_attn_stream_t stream) {
  int rc = check_args(plan, a, ws, ws_bytes, out_f32 == nullptr);
  if (rc) return rc;
  if (!a->lse || (out_f32 && !aligned16(out_f32))) return VERIFY_ATTN_EINVAL;
  va::TreeBlockParams p;
  p.q_latent = a->q_latent;
  p.ql_tok = a->q_latent_stride_tok;
  p.ql_head = a->q_latent_stride_head;
  p.q_rope = a->q_rope;
  p.qr_tok = a->q_rope_stride_tok;
  p.qr_head = a->q_rope_stride_head;
  p.kv_pool = a->kv_pool;
  p.kv_stride = a->kv_row_stride;
  p.kv_indices = a->kv_indices;
  p.kv_indptr = a->kv_indptr;
  p.qo_indptr = a->qo_indptr;
  p.tree_anc = a->tree_anc;
  p.batch = a->batch;
  p.num_heads = plan->num_heads;
  p.max_tree = plan->max_tree;
  p.max_kv_per_req = plan->max_kv_per_req;
  p.pool_slots = plan->pool_slots;
  p.scale_log2 = plan->sm_scale * 1.4426950408889634f;
  p.exclude_self = exclude_self ? 1 : 0;
  p.out = a->out;
  p.out_f32 = out_f32;
  p.out_tok = a->out_stride_tok;
  p.out_head = a->out_stride_head;
  p.lse = a->lse;
  p.self_anc = self_anc;
  p.visible_count = a->visible_count;
  p.status = static_cast<uint32_t*>(ws);
  const int64_t max_tokens = (int64_t)plan->max_batch * plan->max_tree;
  if (va::launch_tree_block(p, max_tokens, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_merge_states(const verify_attn_merge_args* a, verify_attn_stream_t stream) {
  if (!a || !a->o_a || !a->o_b || !a->out || !a->lse_a || !a->lse_b) return VERIFY_ATTN_EINVAL;
  if (a->num_heads < 1 || a->num_heads > VERIFY_ATTN_MAX_HEADS || a->max_tokens < 0) return VERIFY_ATTN_EINVAL;
  if (!aligned16(a->o_a) || !aligned16(a->o_b) || !aligned16(a->out)) return VERIFY_ATTN_EINVAL;
  if (!row_stride_ok(a->o_a_stride_tok) || !row_stride_ok(a->o_a_stride_head) || !row_stride_ok(a->o_b_stride_tok) ||
      !row_stride_ok(a->o_b_stride_head) || !row_stride_ok(a->out_stride_tok) || !row_stride_ok(a->out_stride_head))
    return VERIFY_ATTN_EINVAL;
  va::MergeParams p;
  p.o_a = a->o_a;
  p.a_tok = a->o_a_stride_tok;
  p.a_head = a->o_a_stride_head;
  p.lse_a = a->lse_a;
  p.o_b = a->o_b;
  p.b_tok = a->o_b_stride_tok;
  p.b_head = a->o_b_stride_head;
  p.lse_b = a->lse_b;
  p.b_f32 = a->o_b_f32 ? 1 : 0;
  p.out = a->out;
  p.out_tok = a->out_stride_tok;
  p.out_head = a->out_stride_head;
  p.lse = a->lse;
  p.max_tokens = a->max_tokens;
  p.num_tokens = a->num_tokens;
  p.num_heads = a->num_heads;
  if (a->max_tokens == 0) return VERIFY_ATTN_OK;
  if (va::launch_merge(p, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_merge_stacked(const verify_attn_merge_stacked_args* a, verify_attn_stream_t stream) {
  if (!a || !a->o || !a->lse_states || !a->out) return VERIFY_ATTN_EINVAL;
  if (a->num_states < 1 || a->num_states > 1024 || a->num_heads < 1 || a->num_heads > VERIFY_ATTN_MAX_HEADS ||
      a->max_tokens < 0)
    return VERIFY_ATTN_EINVAL;
  if (!aligned16(a->o) || !aligned16(a->out) || !row_stride_ok(a->out_stride_tok) ||
      !row_stride_ok(a->out_stride_head))
    return VERIFY_ATTN_EINVAL;
  if (a->max_tokens == 0) return VERIFY_ATTN_OK;
  va::MergeStackedParams p;
  p.o = a->o;
  p.lse = a->lse_states;
  p.num_states = a->num_states;
  p.out = a->out;
  p.out_tok = a->out_stride_tok;
  p.out_head = a->out_stride_head;
  p.lse_out = a->lse;
  p.max_tokens = a->max_tokens;
  p.num_tokens = a->num_tokens;
  p.num_heads = a->num_heads;
  if (va::launch_merge_stacked(p, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_defrag(const verify_attn_defrag_args* a, verify_attn_stream_t stream) {
  if (!a || !a->kv_pool || !a->kv_indices || !a->kv_indptr || !a->dst_begin) return VERIFY_ATTN_EINVAL;
  if (a->batch < 1 || a->budget < 0 || a->pool_slots < 1 || a->pool_slots > INT32_MAX) return VERIFY_ATTN_EINVAL;
  if (!aligned16(a->kv_pool) || !row_stride_ok(a->kv_row_stride) || a->kv_row_stride < va::kDQK)
    return VERIFY_ATTN_EINVAL;
  if (a->max_total_kv < 0 || a->max_total_kv > INT32_MAX) return VERIFY_ATTN_EINVAL;
  va::DefragParams p;
  p.kv_pool = a->kv_pool;
  p.kv_stride = a->kv_row_stride;
  p.pool_slots = a->pool_slots;
  p.kv_indices = a->kv_indices;
  p.kv_indptr = a->kv_indptr;
  p.dst_begin = a->dst_begin;
  p.batch = a->batch;
  p.budget = a->budget;
  p.status = a->status;
  if (va::launch_defrag(p, a->max_total_kv, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  return VERIFY_ATTN_OK;
}

int verify_attn_status(const void* ws, verify_attn_stream_t stream, uint32_t* detail_h) {
  if (!ws) return VERIFY_ATTN_EINVAL;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess ||
      cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return VERIFY_ATTN_CUDA_ERROR;
  }
  if (detail_h) *detail_h = word;
  if (word & va::kStatusTimeout) return VERIFY_ATTN_DEVICE_TIMEOUT;
  if (word) return VERIFY_ATTN_DEVICE_BAD_INPUT;
  return VERIFY_ATTN_OK;
}

const char* verify_attn_strerror(int code) {
  switch (code) {
    case VERIFY_ATTN_OK: return "ok";
    case VERIFY_ATTN_EINVAL: return "invalid argument (pointer, size, stride, alignment or tree)";
    case VERIFY_ATTN_UNSUPPORTED: return "unsupported configuration (dims must be 512+64, tree <= 64 nodes)";
    case VERIFY_ATTN_WORKSPACE_TOO_SMALL: return "workspace smaller than the plan requires";
    case VERIFY_ATTN_CUDA_ERROR: return "CUDA launch or runtime error";
    case VERIFY_ATTN_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case VERIFY_ATTN_DEVICE_BAD_INPUT: return "device lengths, slots or tree masks outside the plan were skipped";
    default: return "unknown verify_attn error";
  }
}

}  // extern "C"
