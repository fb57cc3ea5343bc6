// Device-side ancestor-or-self masks for a whole batch of draft trees.
//
// The pages build the tree and its mask on the CPU every decode step (page
// "The Execution Phase", section "The Methodology": 1.8 ms tree build, 0.18 ms
// mask build); doing it on the device keeps the step inside one captured
// graph. One warp per request: lane i (and i + 32) walks from node i up to the
// root, setting bit j for every node j on the way (node i included). A
// malformed tree (root not -1, or a parent not strictly before its child)
// sets the status bit and leaves only the self bits, so no walk can loop.
#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

__global__ void __launch_bounds__(32) tree_mask_kernel(const int32_t* __restrict__ parents,
                                                       const int32_t* __restrict__ qo_indptr, uint64_t* anc,
                                                       uint32_t* status) {
  const int b = blockIdx.x;
  const int32_t q0 = qo_indptr[b];
  const int32_t T = qo_indptr[b + 1] - q0;
  if (T < 1 || T > kMaxTree) {
    if (threadIdx.x == 0 && status && T != 0) atomicOr(status, kStatusBadTree);
    return;
  }
  // The whole tree is valid iff every node's parent precedes it (root: -1).
  bool ok = true;
  for (int i = threadIdx.x; i < T; i += 32) {
    const int32_t par = parents[q0 + i];
    ok = ok && (i == 0 ? par == -1 : (par >= 0 && par < i));
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && threadIdx.x == 0 && status) atomicOr(status, kStatusBadTree);
  for (int i = threadIdx.x; i < T; i += 32) {
    uint64_t bits = 1ull << i;
    if (ok) {
      int32_t j = parents[q0 + i];
      while (j >= 0) {            // strictly decreasing, so at most i steps
        bits |= 1ull << j;
        j = parents[q0 + j];
      }
    }
    anc[q0 + i] = bits;
  }
}

}  // namespace

cudaError_t launch_tree_mask(const int32_t* parents, const int32_t* qo_indptr, int32_t batch, uint64_t* anc,
                             uint32_t* status, cudaStream_t stream) {
  tree_mask_kernel<<<dim3((unsigned)batch), dim3(32), 0, stream>>>(parents, qo_indptr, anc, status);
  return cudaGetLastError();
}

}  // namespace va
