// KV gather kernel of the verify attention: copies the latent rows that a
// call's requests reference (kv_indices into the page_size=1 pool) into a
// contiguous staging area of the workspace, so that the split kernel can load
// every K and V tile with plain tiled TMA copies.
//
// Page "The Execution Phase", section "The Core Design": the KV of a request
// lives in scattered pool slots and every query row tile reads all of it; the
// pages gather it inside the attention kernel with 128-bit loads. On B200 a
// single gather pass costs one read and one write of the call's KV at HBM
// speed, after which the many re-reads by the row tiles come from L2 through
// the TMA engine instead of the load/store units.
//
// Staging layout: request b owns rows [256 * KT_b, 256 * (KT_b + key_tiles_b))
// where KT_b is the number of 256-key tiles of the requests before it; row
// 256 * KT_b + j holds pool[kv_indices[kv_indptr[b] + j], 0:576] for j < N_b and
// zeros for the padding up to the tile boundary. Slots outside the pool are
// written as zero rows and flagged in the status word.
#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

constexpr int kGatherThreads = 256;   // 8 warps; warp w copies rows 32w .. 32w+31 of a tile
constexpr int kRowVecs = kDQK * 2 / 16;   // 72 16-byte vectors per 576-wide bf16 row

__global__ void __launch_bounds__(kGatherThreads) verify_gather_kernel(const GatherParams p) {
  __shared__ int32_t s_total;
  __shared__ int32_t s_req[3];   // request, its first tile, its KV begin
  __shared__ int32_t s_n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    int32_t total = 0;
    for (int b = 0; b < p.batch; ++b)
      total += load_request(p.qo_indptr, p.kv_indptr, b, 1, p.max_tree, p.max_kv_per_req).key_tiles;
    // Lengths whose sum exceeds the plan would run past the staging rows:
    // copy what fits and report it (the split kernel reads zeros beyond).
    if (total > p.stage_tiles) {
      atomicOr(p.status, kStatusBadLengths);
      total = (int32_t)p.stage_tiles;
    }
    s_total = total;
  }
  __syncthreads();
  const int32_t total = s_total;

  for (int32_t gt = blockIdx.x; gt < total; gt += gridDim.x) {
    if (threadIdx.x == 0) {
      int32_t base = 0;
      for (int b = 0; b < p.batch; ++b) {
        const Request r = load_request(p.qo_indptr, p.kv_indptr, b, 1, p.max_tree, p.max_kv_per_req);
        if (gt < base + r.key_tiles) {
          s_req[0] = b;
          s_req[1] = gt - base;
          s_req[2] = r.kv_begin;
          s_n = r.N;
          break;
        }
        base += r.key_tiles;
      }
    }
    __syncthreads();
    const int32_t kt = s_req[1], kv_begin = s_req[2], N = s_n;
    __syncthreads();   // s_req is rewritten by the next iteration

    // Each lane first reads the slot of one of the warp's 32 rows.
    const int32_t j_lane = kt * kKeysPerTile + warp * 32 + lane;
    int32_t slot = -1;
    if (j_lane < N) {
      slot = p.kv_indices[kv_begin + j_lane];
      if (slot < 0 || (int64_t)slot >= p.pool_slots) {
        atomicOr(p.status, kStatusBadSlot);
        slot = -1;
      }
    }
    int4* dst_tile = reinterpret_cast<int4*>(p.stage + ((int64_t)gt * kKeysPerTile + warp * 32) * kDQK);
#pragma unroll 1
    for (int r0 = 0; r0 < 32; r0 += 4) {
      int4 v[4][3];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int32_t s = __shfl_sync(0xffffffffu, slot, r0 + q);
        const int4* src = reinterpret_cast<const int4*>(p.kv_pool + (int64_t)(s < 0 ? 0 : s) * p.kv_stride);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const int e = lane + 32 * c;
          v[q][c] = make_int4(0, 0, 0, 0);
          if (s >= 0 && e < kRowVecs) v[q][c] = __ldcs(src + e);   // read once: stream past L2
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int4* dst = dst_tile + (int64_t)(r0 + q) * kRowVecs;
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const int e = lane + 32 * c;
          if (e < kRowVecs) dst[e] = v[q][c];
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_gather(const GatherParams& p, int grid, cudaStream_t stream) {
  if (grid < 1) grid = 1;
  verify_gather_kernel<<<grid, kGatherThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
