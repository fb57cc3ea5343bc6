// Two-state log-sum-exp merge of the split-verify variant.
//
// Page "The Architecture Detective", section "The Split Verify Design": the
// dense-prefix result and the tree-block result of a query row are combined
// by their log-sum-exps. With states (o_a, lse_a) and (o_b, lse_b) over
// disjoint key sets, m = max(lse_a, lse_b), w_x = exp(lse_x - m):
//   out = (w_a o_a + w_b o_b) / (w_a + w_b),   lse = m + ln(w_a + w_b).
// A state with lse = -inf (no key) has weight 0; two empty states give
// out = 0 and lse = -inf. o_a is bf16; o_b is bf16 or fp32. One warp per (token, head) row; lane l handles the
// bf16 pairs l, l+32, ..., l+224 of the 512-wide rows. Each lane reads its
// pairs before writing them, so `out` may alias either input.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "verify_attn_internal.h"
#include "verify_variant.h"

namespace va {
namespace {

constexpr int kMergeWarps = 8;

__device__ __forceinline__ float2 bf2(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}

__global__ void __launch_bounds__(kMergeWarps * 32) verify_merge_kernel(const MergeParams p) {
  const int lane = threadIdx.x & 31;
  int64_t tokens = p.max_tokens;
  if (p.num_tokens) {
    const int64_t d = *p.num_tokens;
    tokens = d < 0 ? 0 : (d < tokens ? d : tokens);
  }
  const int64_t rows = tokens * p.num_heads;
  for (int64_t row = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5); row < rows;
       row += (int64_t)gridDim.x * kMergeWarps) {
    const int64_t g = row / p.num_heads, h = row % p.num_heads;
    const float la = p.lse_a[row], lb = p.lse_b[row];
    const float m = fmaxf(la, lb);
    const bool empty = !(m > -CUDART_INF_F);
    const float wa = empty ? 0.f : expf(la - m);
    const float wb = empty ? 0.f : expf(lb - m);
    const float s = wa + wb;
    const float inv = s > 0.f ? 1.f / s : 0.f;
    const uint32_t* a = reinterpret_cast<const uint32_t*>(p.o_a + g * p.a_tok + h * p.a_head);
    uint32_t* o = reinterpret_cast<uint32_t*>(p.out + g * p.out_tok + h * p.out_head);
    uint32_t va_[8];
    float2 vb_[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      va_[j] = wa > 0.f ? a[lane + 32 * j] : 0u;
      vb_[j] = make_float2(0.f, 0.f);
    }
    if (wb > 0.f) {
      if (p.b_f32) {
        const float2* b = reinterpret_cast<const float2*>(static_cast<const float*>(p.o_b) + g * p.b_tok + h * p.b_head);
#pragma unroll
        for (int j = 0; j < 8; ++j) vb_[j] = b[lane + 32 * j];
      } else {
        const uint32_t* b = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.o_b) + g * p.b_tok +
                                                              h * p.b_head);
#pragma unroll
        for (int j = 0; j < 8; ++j) vb_[j] = bf2(b[lane + 32 * j]);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 x = bf2(va_[j]), y = vb_[j];
      __nv_bfloat162 r = __floats2bfloat162_rn((wa * x.x + wb * y.x) * inv, (wa * x.y + wb * y.y) * inv);
      o[lane + 32 * j] = *reinterpret_cast<uint32_t*>(&r);
    }
    if (lane == 0 && p.lse) p.lse[row] = s > 0.f ? m + logf(s) : -CUDART_INF_F;
  }
}

// R states stacked along a leading axis (the KV-sequence shards of one call,
// gathered from the ranks): m = max_r lse_r, w_r = exp(lse_r - m),
// out = sum_r w_r o_r / sum_r w_r, lse = m + ln sum_r w_r, rounded to bf16
// once. Lane r (< R, in chunks of 32) holds state r's weight; the rows are
// accumulated in fp32 in the order r = 0, 1, ....
__global__ void __launch_bounds__(kMergeWarps * 32) verify_merge_stacked_kernel(const MergeStackedParams p) {
  const int lane = threadIdx.x & 31;
  int64_t tokens = p.max_tokens;
  if (p.num_tokens) {
    const int64_t d = *p.num_tokens;
    tokens = d < 0 ? 0 : (d < tokens ? d : tokens);
  }
  const int64_t rows = tokens * p.num_heads;
  const int64_t state_rows = p.max_tokens * p.num_heads;
  for (int64_t row = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5); row < rows;
       row += (int64_t)gridDim.x * kMergeWarps) {
    float m = -CUDART_INF_F;
    for (int r = lane; r < p.num_states; r += 32) m = fmaxf(m, p.lse[(int64_t)r * state_rows + row]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const bool empty = !(m > -CUDART_INF_F);
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    float wsum = 0.f;
    for (int r0 = 0; r0 < p.num_states; r0 += 32) {
      const int r_mine = r0 + lane;
      const float w_mine =
          (!empty && r_mine < p.num_states) ? expf(p.lse[(int64_t)r_mine * state_rows + row] - m) : 0.f;
      const int n = p.num_states - r0 < 32 ? p.num_states - r0 : 32;
      for (int k = 0; k < n; ++k) {
        const float w = __shfl_sync(0xffffffffu, w_mine, k);
        if (!(w > 0.f)) continue;   // uniform: every lane holds the same w
        wsum += w;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(p.o + ((int64_t)(r0 + k) * state_rows + row) * kDLatent);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 x = bf2(src[lane + 32 * j]);
          acc[2 * j] = fmaf(w, x.x, acc[2 * j]);
          acc[2 * j + 1] = fmaf(w, x.y, acc[2 * j + 1]);
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const int64_t g = row / p.num_heads, h = row % p.num_heads;
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + g * p.out_tok + h * p.out_head);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * j] * inv, acc[2 * j + 1] * inv);
      dst[lane + 32 * j] = *reinterpret_cast<uint32_t*>(&b);
    }
    if (lane == 0 && p.lse_out) p.lse_out[row] = wsum > 0.f ? m + logf(wsum) : -CUDART_INF_F;
  }
}

}  // namespace

cudaError_t launch_merge_stacked(const MergeStackedParams& p, cudaStream_t stream) {
  const int64_t rows = p.max_tokens * p.num_heads;
  int64_t grid = (rows + kMergeWarps - 1) / kMergeWarps;
  if (grid > 148 * 8) grid = 148 * 8;
  if (grid < 1) grid = 1;
  verify_merge_stacked_kernel<<<(unsigned)grid, kMergeWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  const int64_t rows = p.max_tokens * p.num_heads;
  int64_t grid = (rows + kMergeWarps - 1) / kMergeWarps;
  if (grid > 148 * 8) grid = 148 * 8;
  if (grid < 1) grid = 1;
  verify_merge_kernel<<<(unsigned)grid, kMergeWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
