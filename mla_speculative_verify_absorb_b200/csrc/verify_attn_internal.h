// Internal definitions shared by the host code and the kernels of the
// verify-attention library: tile sizes, the workspace status bits and the
// work schedule that the split kernel and the reduce kernel must agree on.
#pragma once

#include <stdint.h>

#include "verify_attn.h"

#if defined(__CUDACC__)
#define VA_HD __host__ __device__ __forceinline__
#else
#define VA_HD inline
#endif

namespace va {

constexpr int kDLatent = VERIFY_ATTN_D_LATENT;   // 512: c_kv / value width
constexpr int kDRope = VERIFY_ATTN_D_ROPE;       // 64: rope width
constexpr int kDQK = kDLatent + kDRope;          // 576: score contraction width
constexpr int kRowsPerTile = 128;                // query rows per CTA pair (64 per CTA)
constexpr int kRowsPerCta = 64;
constexpr int kKeysPerTile = 256;                // KV positions per work unit (128 per CTA for QK)
constexpr int kWsHeaderBytes = 256;              // status word + diagnostics at ws offset 0
constexpr int kMaxTree = VERIFY_ATTN_MAX_TREE;    // 64: one uint64 mask word per query

// Status bits written (atomicOr) into the first word of the workspace.
constexpr uint32_t kStatusTimeout = 1u << 0;      // a bounded wait expired
constexpr uint32_t kStatusBadLengths = 1u << 1;   // T_b / N_b outside the plan
constexpr uint32_t kStatusBadSlot = 1u << 2;      // kv_indices entry outside the pool
constexpr uint32_t kStatusBadTree = 1u << 3;      // tree_anc has a bit at or beyond T_b, or misses self

// Work units: for every request b, its query rows (t-major, h-minor:
// row = t*H + h) are cut into row tiles of kRowsPerTile, its KV positions
// into key tiles of kKeysPerTile. Unit (g, kt) pairs global row tile g with
// key tile kt of g's request; units are numbered g-major. Cluster c of G
// takes units [floor(c*U/G), floor((c+1)*U/G)). The partial state that
// cluster c leaves for row tile g goes to slot g + c, which is unique because
// the (g, c) pairs that meet form a monotone staircase.
struct Request {
  int32_t q_begin, T;       // tokens [q_begin, q_begin + T)
  int32_t kv_begin, N;      // KV positions [kv_begin, kv_begin + N)
  int32_t row_tiles, key_tiles;
  bool valid;
};

VA_HD Request load_request(const int32_t* qo_indptr, const int32_t* kv_indptr, int b, int H,
                           int max_tree, int64_t max_kv_per_req) {
  Request r;
  r.q_begin = qo_indptr[b];
  r.T = qo_indptr[b + 1] - r.q_begin;
  r.kv_begin = kv_indptr[b];
  r.N = kv_indptr[b + 1] - r.kv_begin;
  r.valid = r.T >= 1 && r.T <= max_tree && r.N >= r.T && (int64_t)r.N <= max_kv_per_req;
  if (r.valid) {
    r.row_tiles = (r.T * H + kRowsPerTile - 1) / kRowsPerTile;
    r.key_tiles = (r.N + kKeysPerTile - 1) / kKeysPerTile;
  } else {
    r.row_tiles = 0;
    r.key_tiles = 0;
  }
  return r;
}

VA_HD int64_t unit_start(int64_t c, int64_t U, int64_t G) { return (c * U) / G; }

// Last cluster whose range starts at or before unit u (U >= 1).
VA_HD int64_t cluster_of_unit(int64_t u, int64_t U, int64_t G) { return ((u + 1) * G - 1) / U; }

}  // namespace va
