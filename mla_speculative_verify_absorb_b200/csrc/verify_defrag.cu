// KV relocation (Tier 1 defragmentation) for the page_size=1 latent pool.
//
// Page "The Execution Phase", section "Tier 0 KV Defragmentation": the
// allocator patch (Tier 0) makes new allocations ascending; Tier 1, live
// relocation of a request's fragmented slots under a copy budget, was
// deferred on the pages and no algorithm is given. This kernel implements
// the plainest reading: for request b and n_b = min(N_b, budget), KV position
// j < n_b moves to slot dst_begin[b] + j (its 576-wide latent row is copied
// there unless it already is) and kv_indices is rewritten to that slot, so a
// request's leading KV becomes one contiguous run while attention sees the
// same rows. The caller's allocator guarantees that destination runs hold no
// slot that another position still references.
//
// One warp per chunk of 32 consecutive KV positions (grid-stride): lane l
// finds the request of position q0 + l (binary search in kv_indptr), checks
// the slots and reads kv_indices coalesced; the warp then copies the chunk's
// moved rows four at a time (12 16-byte loads in flight per lane) and lane l
// rewrites its index. HBM-bound: 2 x 1152 bytes per moved position plus 8
// bytes of index traffic per position.
#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_attn_internal.h"
#include "verify_defrag.h"

namespace va {
namespace {

constexpr int kDefragWarps = 8;
constexpr int kRowVecs16 = kDQK * 2 / 16;   // 72 16-byte vectors per latent row

__global__ void __launch_bounds__(kDefragWarps * 32) verify_defrag_kernel(const DefragParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kDefragWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kDefragWarps;
  const int64_t total = p.kv_indptr[p.batch];
  uint32_t bits = 0;
  for (int64_t q0 = warp0 * 32; q0 < total; q0 += nwarps * 32) {
    const int64_t q = q0 + lane;
    int32_t src = -1;    // slot to copy from, -1: nothing to copy
    int64_t dst = -1;    // new slot of position q, -1: index unchanged
    if (q < total) {
      int lo = 0, hi = p.batch;   // request b with kv_indptr[b] <= q < kv_indptr[b + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.kv_indptr[mid] <= q) lo = mid; else hi = mid;
      }
      const int64_t k0 = p.kv_indptr[lo], k1 = p.kv_indptr[lo + 1];
      const int64_t j = q - k0;
      const int64_t n = (k1 - k0) < (int64_t)p.budget ? (k1 - k0) : (int64_t)p.budget;
      if (k1 < k0 || j < 0) {
        bits |= kStatusBadLengths;
      } else if (j < n) {
        const int64_t d0 = p.dst_begin[lo];
        const int32_t s = p.kv_indices[q];
        if (d0 < 0 || d0 + n > p.pool_slots) {
          bits |= kStatusBadLengths;
        } else if (s < 0 || (int64_t)s >= p.pool_slots) {
          bits |= kStatusBadSlot;
        } else {
          dst = d0 + j;
          if ((int64_t)s != dst) src = s;
        }
      }
    }
    if (__ballot_sync(0xffffffffu, src >= 0)) {
#pragma unroll 1
      for (int r0 = 0; r0 < 32; r0 += 4) {
        int4 v[4][3];
        int32_t rs[4];
        int64_t rd[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          rs[r] = __shfl_sync(0xffffffffu, src, r0 + r);
          rd[r] = __shfl_sync(0xffffffffu, dst, r0 + r);
          if (rs[r] < 0) continue;
          const int4* from = reinterpret_cast<const int4*>(p.kv_pool + (int64_t)rs[r] * p.kv_stride);
#pragma unroll
          for (int c = 0; c < 3; ++c)
            if (lane + 32 * c < kRowVecs16) v[r][c] = __ldcs(from + lane + 32 * c);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (rs[r] < 0) continue;
          int4* to = reinterpret_cast<int4*>(p.kv_pool + rd[r] * p.kv_stride);
#pragma unroll
          for (int c = 0; c < 3; ++c)
            if (lane + 32 * c < kRowVecs16) to[lane + 32 * c] = v[r][c];
        }
      }
    }
    if (dst >= 0) p.kv_indices[q] = (int32_t)dst;
  }
  if (bits && p.status) atomicOr(p.status, bits);
}

}  // namespace

cudaError_t launch_defrag(const DefragParams& p, int64_t max_total, cudaStream_t stream) {
  const int64_t chunks = (max_total + 31) / 32;
  int64_t blocks = (chunks + kDefragWarps - 1) / kDefragWarps;
  if (blocks > 148 * 16) blocks = 148 * 16;   // grid-stride beyond that
  if (blocks < 1) blocks = 1;
  verify_defrag_kernel<<<(unsigned)blocks, kDefragWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
