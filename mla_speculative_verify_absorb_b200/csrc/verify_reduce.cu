// Reduce kernel: LSE merge of the split kernel's partial states.
//
// For every query row the split kernel left one partial state (m, l, O,
// count) per CTA pair that covered part of the row's KV range (page "The
// Verify Kernel Breakthrough", section "The Message in Context": NSPLIT
// partials plus a reduce; page "The Architecture Detective", section "The
// Split Verify Design": merge by log-sum-exp). With m in log2 units:
//     m* = max m_s over states with l_s > 0,   w_s = 2^(m_s - m*),
//     out = sum w_s O_s / sum w_s l_s,         lse = ln 2 * (m* + log2 sum w_s l_s),
//     visible = sum count_s.
// One warp merges one row: lane i owns value columns {4i..4i+3} + 128k, so
// each partial row (2 KB) and each bf16 output row is read/written with
// fully coalesced 16-byte / 8-byte accesses. The kernel is HBM-bound.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

constexpr int kReduceWarps = 8;
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerBlock = kReduceWarps * kRowsPerWarp;          // 16
constexpr int kBlocksPerTile = kRowsPerTile / kRowsPerBlock;        // 8

__global__ void __launch_bounds__(kReduceWarps * 32) verify_reduce_kernel(const ReduceParams p) {
  const int64_t g_target = blockIdx.x / kBlocksPerTile;
  const int chunk = blockIdx.x % kBlocksPerTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = p.num_clusters;

  // Total units of the call, and the request / first unit of row tile g_target.
  int64_t U = 0;
  for (int b = 0; b < p.batch; ++b) {
    Request r = load_request(p.qo_indptr, p.kv_indptr, b, p.num_heads, p.max_tree, p.max_kv_per_req);
    U += (int64_t)r.row_tiles * r.key_tiles;
    if (blockIdx.x == 0 && threadIdx.x == 0 && !r.valid) atomicOr(p.status, kStatusBadLengths);
  }
  if (U == 0) return;
  int64_t g = 0, ustart = 0;
  Request req;
  int rt = -1;
  for (int b = 0; b < p.batch && rt < 0; ++b) {
    Request r = load_request(p.qo_indptr, p.kv_indptr, b, p.num_heads, p.max_tree, p.max_kv_per_req);
    if (g_target < g + r.row_tiles) {
      req = r;
      rt = (int)(g_target - g);
      ustart += (int64_t)rt * r.key_tiles;
    } else {
      g += r.row_tiles;
      ustart += (int64_t)r.row_tiles * r.key_tiles;
    }
  }
  if (rt < 0) return;   // beyond the call's row tiles

  const int64_t c_lo = cluster_of_unit(ustart, U, G);
  const int64_t c_hi = cluster_of_unit(ustart + req.key_tiles - 1, U, G);
  const int64_t rows = (int64_t)req.T * p.num_heads;

  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int tile_row = chunk * kRowsPerBlock + warp * kRowsPerWarp + i;
    const int64_t gr = (int64_t)rt * kRowsPerTile + tile_row;
    if (gr >= rows) break;
    const int64_t t = gr / p.num_heads, h = gr % p.num_heads;

    float m_star = -CUDART_INF_F;
    for (int64_t c = c_lo; c <= c_hi; ++c) {
      if (unit_start(c, U, G) == unit_start(c + 1, U, G)) continue;   // cluster without work
      const float4 mt = p.meta[(g_target + c) * kRowsPerTile + tile_row];
      if (mt.y > 0.f) m_star = fmaxf(m_star, mt.x);
    }
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
    float l_star = 0.f, count = 0.f;
    for (int64_t c = c_lo; c <= c_hi; ++c) {
      if (unit_start(c, U, G) == unit_start(c + 1, U, G)) continue;
      const int64_t srow = (g_target + c) * kRowsPerTile + tile_row;
      const float4 mt = p.meta[srow];
      count += mt.z;
      if (!(mt.y > 0.f)) continue;
      const float w = exp2f(mt.x - m_star);
      l_star += w * mt.y;
      const float4* src = reinterpret_cast<const float4*>(p.partial + srow * kDLatent);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 o = src[lane + 32 * k];
        acc[4 * k + 0] += w * o.x;
        acc[4 * k + 1] += w * o.y;
        acc[4 * k + 2] += w * o.z;
        acc[4 * k + 3] += w * o.w;
      }
    }
    const float inv = l_star > 0.f ? 1.f / l_star : 0.f;
    uint16_t* dst = p.out + (int64_t)(req.q_begin + t) * p.out_tok + h * p.out_head;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc[4 * k + 0] * inv, acc[4 * k + 1] * inv);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc[4 * k + 2] * inv, acc[4 * k + 3] * inv);
      uint2 v;
      v.x = *reinterpret_cast<uint32_t*>(&lo);
      v.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(dst + 4 * (lane + 32 * k)) = v;
    }
    if (lane == 0) {
      if (p.lse) {
        const float lse2 = l_star > 0.f ? m_star + log2f(l_star) : -CUDART_INF_F;
        p.lse[(int64_t)(req.q_begin + t) * p.num_heads + h] = lse2 * 0.69314718055994530942f;
      }
      if (h == 0) {
        if (p.visible_count) p.visible_count[req.q_begin + t] = (int32_t)count;
        const uint64_t anc = p.tree_anc[req.q_begin + t];
        const bool self = (anc >> t) & 1ull;
        const bool beyond = req.T < 64 && (anc >> req.T) != 0ull;
        if (!self || beyond) atomicOr(p.status, kStatusBadTree);
      }
    }
  }
}

}  // namespace

cudaError_t launch_reduce(const ReduceParams& p, cudaStream_t stream) {
  const int64_t tiles = (int64_t)p.row_tiles_per_req * p.batch;
  verify_reduce_kernel<<<dim3((unsigned)(tiles * kBlocksPerTile)), dim3(kReduceWarps * 32), 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
