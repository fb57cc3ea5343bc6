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
// One warp merges one row. The lanes first read the row's (m, l, count)
// headers of all covering pairs at once (lane k: pair c_lo + k) and combine
// them with shuffles; then lane i accumulates value columns {4i..4i+3} + 128k
// of the weighted partial rows (2 KB each, coalesced 16-byte loads, four
// pairs' rows in flight) and writes the bf16 output row with 8-byte stores.
// The kernel is bound by the latency of those two dependent reads, so it
// runs one warp per row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

constexpr int kReduceWarps = 8;
constexpr int kRowsPerBlock = kReduceWarps;                         // one row per warp
constexpr int kBlocksPerTile = kRowsPerTile / kRowsPerBlock;        // 16

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

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
  const int n = (int)(c_hi - c_lo + 1);
  const int64_t rows = (int64_t)req.T * p.num_heads;
  const int tile_row = chunk * kRowsPerBlock + warp;
  const int64_t gr = (int64_t)rt * kRowsPerTile + tile_row;
  if (gr >= rows) return;
  const int64_t t = gr / p.num_heads, h = gr % p.num_heads;
  const int64_t row0 = (g_target + c_lo) * kRowsPerTile + tile_row;   // slot row of pair c_lo

  // Headers: lane k holds pair c_lo + k (more than 32 covering pairs are
  // read in further chunks); a pair without work or without visible keys
  // has l = 0 and contributes nothing.
  auto header = [&](int k) -> float4 {
    if (k < n && unit_start(c_lo + k, U, G) != unit_start(c_lo + k + 1, U, G))
      return p.meta[row0 + (int64_t)k * kRowsPerTile];
    return make_float4(-CUDART_INF_F, 0.f, 0.f, 0.f);
  };
  const float4 mt0 = header(lane);
  float m_star = mt0.y > 0.f ? mt0.x : -CUDART_INF_F;
  for (int k0 = 32; k0 < n; k0 += 32) {
    const float4 mt = header(k0 + lane);
    if (mt.y > 0.f) m_star = fmaxf(m_star, mt.x);
  }
  m_star = warp_max(m_star);
  const float w_mine = mt0.y > 0.f ? exp2f(mt0.x - m_star) : 0.f;   // weight of pair lane
  float l_part = w_mine * mt0.y, c_part = mt0.z;
  for (int k0 = 32; k0 < n; k0 += 32) {
    const float4 mt = header(k0 + lane);
    c_part += mt.z;
    if (mt.y > 0.f) l_part += exp2f(mt.x - m_star) * mt.y;
  }
  const float l_star = warp_sum(l_part);
  const float count = warp_sum(c_part);

  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int k0 = 0; k0 < n; k0 += 4) {
    float w[4];
    float4 o[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + q;
      float wk;
      if (k < 32) {
        wk = __shfl_sync(0xffffffffu, w_mine, k & 31);
      } else {   // more than 32 covering pairs: recompute this pair's weight
        const float4 mt = header(k);
        wk = mt.y > 0.f ? exp2f(mt.x - m_star) : 0.f;
      }
      w[q] = k < n ? wk : 0.f;
      const float4* src = reinterpret_cast<const float4*>(p.partial + (row0 + (int64_t)k * kRowsPerTile) * kDLatent);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[q][e] = w[q] > 0.f ? src[lane + 32 * e] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[4 * e + 0] += w[q] * o[q][e].x;
        acc[4 * e + 1] += w[q] * o[q][e].y;
        acc[4 * e + 2] += w[q] * o[q][e].z;
        acc[4 * e + 3] += w[q] * o[q][e].w;
      }
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

}  // namespace

cudaError_t launch_reduce(const ReduceParams& p, cudaStream_t stream) {
  const int64_t tiles = (int64_t)p.row_tiles_per_req * p.batch;
  verify_reduce_kernel<<<dim3((unsigned)(tiles * kBlocksPerTile)), dim3(kReduceWarps * 32), 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
