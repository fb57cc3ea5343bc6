// Masked tree-block attention of the split-verify variant.
//
// Page "The Architecture Detective", section "The Split Verify Design": the
// verify attention can be taken apart into dense attention of every query
// over the shared prefix, a tiny masked attention of the tree tokens over the
// tree block, and a log-sum-exp merge of the two results. This kernel is the
// tree-block part: query row (t, h) attends the tree keys L_b + j whose bit j
// is set in its ancestor-or-self mask (with `exclude_self`, the node's own
// key is left to the dense pass), and writes the normalised output (fp32, so
// that the merge rounds to bf16 once, or bf16) and the natural-log LSE of
// that key set.
//
// One CTA per (tree token, group of eight heads), grid-stride: it gathers the
// token's visible tree rows (at most 64 x 1152 B) into shared memory, and
// each of its eight warps takes one head. A warp holds the 576-wide query in
// registers (lane l: bf16 pairs l, l+32, ...), forms each score with a warp
// sum, keeps the scores of keys l and l+32 in lane l, and accumulates the
// 512-wide output in fp32 (lane l: pairs l, l+32, ..., l+224). The work is a
// few hundred MFLOP per call, on CUDA cores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "verify_attn_internal.h"
#include "verify_variant.h"

namespace va {
namespace {

constexpr int kTbWarps = 8;
constexpr int kRowWords = kDQK / 2;          // 288 bf16 pairs per latent row
constexpr int kRowVec = kDQK * 2 / 16;       // 72 16-byte vectors per latent row
constexpr int kTbSmem = kMaxTree * kDQK * 2; // 73 728 B: the visible tree rows

__device__ __forceinline__ float2 bf2(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__global__ void __launch_bounds__(kTbWarps * 32) verify_tree_block_kernel(const TreeBlockParams p) {
  extern __shared__ __align__(16) uint8_t tb_smem[];
  uint32_t* rows = reinterpret_cast<uint32_t*>(tb_smem);   // row k: kRowWords words
  __shared__ int32_t s_key[kMaxTree];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t total = p.qo_indptr[p.batch];

  const int head_groups = (p.num_heads + kTbWarps - 1) / kTbWarps;
  const int64_t items = (int64_t)total * head_groups;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int32_t g = (int32_t)(it / head_groups);
    const int hg = (int)(it % head_groups);
    int lo = 0, hi = p.batch;   // request b with qo_indptr[b] <= g < qo_indptr[b + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.qo_indptr[mid] <= g) lo = mid; else hi = mid;
    }
    const Request r = load_request(p.qo_indptr, p.kv_indptr, lo, 1, p.max_tree, p.max_kv_per_req);
    if (!r.valid) {   // uniform across the CTA
      if (threadIdx.x == 0 && hg == 0) atomicOr(p.status, kStatusBadLengths);
      continue;
    }
    const int t = g - r.q_begin;
    const int64_t L = (int64_t)r.N - r.T;
    const uint64_t anc = p.tree_anc[g];
    const uint64_t in_tree = r.T >= 64 ? ~0ull : ((1ull << r.T) - 1ull);
    const uint64_t self = 1ull << t;
    uint64_t bits = anc & in_tree;
    if (p.exclude_self) bits &= ~self;
    const int n = __popcll(bits);
    if (threadIdx.x == 0 && hg == 0) {
      if ((anc & ~in_tree) != 0ull || (anc & self) == 0ull) atomicOr(p.status, kStatusBadTree);
      if (p.self_anc) p.self_anc[g] = self;
      if (p.visible_count) p.visible_count[g] = (int32_t)(L + n + (p.exclude_self ? 1 : 0));
    }
    if (threadIdx.x < kMaxTree && ((bits >> threadIdx.x) & 1ull))
      s_key[__popcll(bits & ((1ull << threadIdx.x) - 1ull))] = threadIdx.x;
    __syncthreads();

    // Gather the n visible tree rows; a slot outside the pool gives a zero row.
    for (int k = warp; k < n; k += kTbWarps) {
      const int32_t slot = p.kv_indices[r.kv_begin + L + s_key[k]];
      const bool ok = slot >= 0 && (int64_t)slot < p.pool_slots;
      if (!ok && lane == 0 && hg == 0) atomicOr(p.status, kStatusBadSlot);
      const int4* src = reinterpret_cast<const int4*>(p.kv_pool + (int64_t)(ok ? slot : 0) * p.kv_stride);
      int4* dst = reinterpret_cast<int4*>(tb_smem + (size_t)k * kDQK * 2);
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const int e = lane + 32 * c;
        if (e < kRowVec) dst[e] = ok ? src[e] : make_int4(0, 0, 0, 0);
      }
    }
    __syncthreads();

    const int h = hg * kTbWarps + warp;
    if (h < p.num_heads) {
      const uint32_t* ql = reinterpret_cast<const uint32_t*>(p.q_latent + (int64_t)g * p.ql_tok + (int64_t)h * p.ql_head);
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(p.q_rope + (int64_t)g * p.qr_tok + (int64_t)h * p.qr_head);
      float2 q[9];
#pragma unroll
      for (int i = 0; i < 9; ++i) {
        const int w = lane + 32 * i;   // pairs 0..255 latent, 256..287 rope
        q[i] = bf2(w < kDLatent / 2 ? ql[w] : qr[w - kDLatent / 2]);
      }
      float s0 = -CUDART_INF_F, s1 = -CUDART_INF_F;   // scores of keys lane, lane + 32 (log2 domain)
      for (int k = 0; k < n; ++k) {
        const uint32_t* row = rows + k * kRowWords;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 9; ++i) {
          const float2 kf = bf2(row[lane + 32 * i]);
          acc = fmaf(q[i].x, kf.x, acc);
          acc = fmaf(q[i].y, kf.y, acc);
        }
        const float s = warp_sum(acc) * p.scale_log2;
        if (lane == (k & 31)) {
          if (k < 32) s0 = s; else s1 = s;
        }
      }
      const float m = warp_max(fmaxf(s0, s1));
      const float p0 = lane < n ? exp2f(s0 - m) : 0.f;
      const float p1 = lane + 32 < n ? exp2f(s1 - m) : 0.f;
      const float l = warp_sum(p0 + p1);

      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = 0.f;
      for (int k = 0; k < n; ++k) {
        const float pk = __shfl_sync(0xffffffffu, k < 32 ? p0 : p1, k & 31);
        const uint32_t* row = rows + k * kRowWords;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 v = bf2(row[lane + 32 * j]);
          o[2 * j] = fmaf(pk, v.x, o[2 * j]);
          o[2 * j + 1] = fmaf(pk, v.y, o[2 * j + 1]);
        }
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (p.out_f32) {
        float2* dst = reinterpret_cast<float2*>(p.out_f32 + ((int64_t)g * p.num_heads + h) * kDLatent);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[lane + 32 * j] = make_float2(o[2 * j] * inv, o[2 * j + 1] * inv);
      } else {
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (int64_t)g * p.out_tok + (int64_t)h * p.out_head);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          __nv_bfloat162 b = __floats2bfloat162_rn(o[2 * j] * inv, o[2 * j + 1] * inv);
          dst[lane + 32 * j] = *reinterpret_cast<uint32_t*>(&b);
        }
      }
      if (lane == 0)
        p.lse[(int64_t)g * p.num_heads + h] = n > 0 ? (m + log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
    }
    __syncthreads();   // rows and s_key are rewritten for the next token
  }
}

}  // namespace

cudaError_t launch_tree_block(const TreeBlockParams& p, int64_t max_tokens, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(verify_tree_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTbSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = 1;
  }
  const int64_t items = max_tokens * ((p.num_heads + kTbWarps - 1) / kTbWarps);
  int64_t grid = items < 148 * 4 ? items : 148 * 4;
  if (grid < 1) grid = 1;
  verify_tree_block_kernel<<<(unsigned)grid, kTbWarps * 32, kTbSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
