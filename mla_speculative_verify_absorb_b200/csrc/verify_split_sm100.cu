// Split kernel of the MLA-absorb tree-verify attention for B200 (sm_100a).
//
// What it computes (page "The Execution Phase", section "The Transition:
// From Planning to Execution": MLA-absorb attention with a custom tree mask;
// section "The Core Design": KV tile loaded once for all heads): for a tile
// of 128 query rows (token, head) of one request and a run of KV tiles of
// 128 positions, the fp32 partial state
//     m = running max of the scaled scores (log2 units),
//     l = sum 2^(s - m),  O = sum 2^(s - m) * c_kv,  count = visible keys,
// written per (row tile, CTA pair) for the LSE-merge reduce (page "The
// Verify Kernel Breakthrough", section "The Message in Context": KV-split
// partials plus reduce).
//
// How (B200-specific; the pages' sm_120 kernel is prior art, not the plan):
//  * A cluster of two CTAs on two SMs shares one 128-row tile: each CTA
//    holds 64 rows of Q in shared memory and the pair issues
//    tcgen05.mma.cta_group::2 with M = 128, so every SM keeps all 128 tensor
//    memory lanes busy with only 64 rows. In that mode a CTA's accumulator of
//    N columns takes N/2 TMEM columns (lanes 0-63: columns [0, N/2) of its 64
//    rows, lanes 64-127: columns [N/2, N)), which is what lets the 512-wide
//    fp32 output accumulator (256 TMEM columns) sit beside two score buffers.
//  * S = Q K^T: M = 128 rows, N = 128 keys (each CTA gathers 64 of them),
//    K = 576 in nine 64-wide chunks. O += P V: M = 128, N = 256 value columns
//    per instruction (each CTA gathers 128 of them), K = keys; V is the first
//    512 columns of the same latent rows, staged MN-major.
//  * Scattered pool rows are gathered with 16-byte cp.async into 128-byte
//    swizzled stages of 8 KB by two producer warps; one thread of the leader
//    CTA issues all MMAs; four softmax warps per CTA read S from TMEM, apply
//    scale and the ancestor mask, keep the online softmax (the O rescale is
//    skipped unless the row max grows by more than 2^8), write bf16 P into
//    shared memory and finally dump O to the workspace.
//  * Persistent grid: cluster c of G takes an equal share of the call's
//    (row tile, key tile) units, so work is balanced whatever the mix of
//    request lengths, and at most G + #row tiles partial states are written.
//  * Every wait is bounded; on expiry the kernel records it in the status
//    word, unwinds both CTAs and frees its tensor memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"
#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

using namespace ptx;

constexpr int kThreads = 448;          // 4 softmax + 6 KV loader + Q loader + relay + 2 MMA warps
constexpr int kSoftmaxThreads = 128;
constexpr int kKvWarp0 = 4;
constexpr int kNumKvWarps = 6;
constexpr int kQWarp = 10;
constexpr int kRelayWarp = 11;
constexpr int kRelayBatch = 4;          // peer stages forwarded per release-arrive instruction
constexpr int kMmaWarp = 12;           // issues the score MMAs; also owns the TMEM allocation
constexpr int kPvWarp = 13;            // issues the value MMAs

constexpr int kStageBytes = 8192;
constexpr int kNumStages = 14;
constexpr int kQBlocks = kDQK / 64;    // 9 chunks of 64 columns
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQBlocks * 8192;   // 2 buffers x 2 key blocks x 8 KB
constexpr int kOffRing = kOffP + 4 * 8192;
constexpr int kOffCtrl = kOffRing + kNumStages * kStageBytes;

// TMEM columns (per CTA; 2x2 layout of the pair MMA).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;        // S buffers: 64 columns each
constexpr uint32_t kColO = 128;       // O: two 128-column halves (value columns [0,256) and [256,512))

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, true);

constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Ctrl {
  uint64_t ring_full[kNumStages];   // leader: 32 loader-lane arrivals + 1 relay arrival per stage
  uint64_t peer_full[kNumStages];   // peer: 32 loader-lane arrivals, relayed to the leader
  uint64_t ring_empty[kNumStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t o_free;
  uint64_t mma_final;
  uint64_t xchg;          // softmax-thread exchange of row maxima and sums (128 arrivals)
  uint32_t tmem_base;
  int32_t abort_flag;
  float red_max[2][kSoftmaxThreads];
  float red_l[2][kSoftmaxThreads];
  float red_c[2][kSoftmaxThreads];
};

constexpr int kSmemBytes = kOffCtrl + (int)sizeof(Ctrl) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "split kernel shared memory exceeds the sm_100 limit");

struct Segment {
  Request req;
  int32_t b, rt, kt0, n;
  int64_t g;
};

__device__ __forceinline__ Request request_of(const SplitParams& p, int b) {
  return load_request(p.qo_indptr, p.kv_indptr, b, p.num_heads, p.max_tree, p.max_kv_per_req);
}

__device__ int64_t total_units(const SplitParams& p) {
  int64_t U = 0;
  for (int b = 0; b < p.batch; ++b) {
    Request r = request_of(p, b);
    U += (int64_t)r.row_tiles * r.key_tiles;
  }
  return U;
}

// Segment (maximal run of units on one row tile) that starts at unit u.
__device__ bool find_segment(const SplitParams& p, int64_t u, int64_t u_end, Segment& s) {
  if (u >= u_end) return false;
  int64_t acc = 0, g = 0;
  for (int b = 0; b < p.batch; ++b) {
    Request r = request_of(p, b);
    int64_t ub = (int64_t)r.row_tiles * r.key_tiles;
    if (u < acc + ub) {
      int64_t local = u - acc;
      s.req = r;
      s.b = b;
      s.rt = (int32_t)(local / r.key_tiles);
      s.kt0 = (int32_t)(local % r.key_tiles);
      s.g = g + s.rt;
      int64_t left = u_end - u;
      s.n = (int32_t)((int64_t)(r.key_tiles - s.kt0) < left ? (r.key_tiles - s.kt0) : left);
      return true;
    }
    acc += ub;
    g += r.row_tiles;
  }
  return false;
}

__device__ void give_up(Ctrl* ctrl, const SplitParams& p, uint32_t rank) {
  atomicOr(p.status, kStatusTimeout);
  const uint32_t local = smem_addr(&ctrl->abort_flag);
  st_cluster_u32(map_to_rank(local, rank), 1u);
  st_cluster_u32(map_to_rank(local, rank ^ 1u), 1u);
}

// Bounded wait by one thread for the completion of the phase with `parity`.
// Returns false when the limit expires (both CTAs are then told to unwind)
// or when the pair is already unwinding.
__device__ bool wait_one(uint32_t bar, uint32_t parity, Ctrl* ctrl, const SplitParams& p, uint32_t rank) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*(volatile int32_t*)&ctrl->abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      give_up(ctrl, p, rank);
      return false;
    }
  }
}

// The same wait taken by all 32 lanes of a warp together: every lane
// acquires the barrier itself and all lanes return the same answer, so the
// warp never splits on a timeout.
__device__ bool wait_warp(uint32_t bar, uint32_t parity, Ctrl* ctrl, const SplitParams& p, uint32_t rank) {
  const bool lane0 = (threadIdx.x & 31) == 0;
  uint64_t t0 = 0;
  for (int iter = 0;; ++iter) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    int stop = 0;
    if (lane0) {
      const uint64_t now = globaltimer();
      if (iter == 0) t0 = now;
      if (*(volatile int32_t*)&ctrl->abort_flag) {
        stop = 1;
      } else if (now - t0 > kWaitLimitNs) {
        give_up(ctrl, p, rank);
        stop = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, stop, 0)) return false;
  }
}

__device__ __forceinline__ uint64_t low_bits(int64_t k) {
  return k <= 0 ? 0ull : (k >= 64 ? ~0ull : ((1ull << k) - 1ull));
}

// Visibility of KV positions key0 .. key0+63 of a request (bit e <-> key0+e):
// prefix positions (< L) always, tree position L+i iff bit i of anc, nothing
// at or beyond N.
__device__ __forceinline__ uint64_t visible_bits(int64_t key0, int64_t L, int64_t N, uint64_t anc) {
  uint64_t v = low_bits(L - key0);
  int64_t d = key0 - L;
  uint64_t tree;
  if (d >= 0)
    tree = d >= 64 ? 0ull : (anc >> d);
  else
    tree = -d >= 64 ? 0ull : (anc << (-d));
  return (v | tree) & low_bits(N - key0);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ----------------------------------------------------------------------------- producers

// Stage order of one segment of n tiles, shared by the loaders, the relay and
// the MMA issuer: K(0), then for i = 1..n-1: K(i), V(i-1), then V(n-1). K(i)
// is 9 stages (64-column blocks of the 576 score columns), V(i) 8 stages
// (4 key chunks of 32 x 2 output halves), so a segment has 17n stages.
constexpr int kStagesK = kQBlocks;    // 9
constexpr int kStagesV = 8;
constexpr int kStagesPerTile = kStagesK + kStagesV;

struct StageDesc {
  int32_t tile;    // tile index within the segment
  int32_t is_v;    // 0: K stage, 1: V stage
  int32_t idx;     // K: column block 0..8; V: kc*2 + dh
};

__device__ __forceinline__ StageDesc describe_stage(uint32_t p, int n) {
  StageDesc d;
  if (p < (uint32_t)kStagesK) {
    d.tile = 0; d.is_v = 0; d.idx = (int)p;
    return d;
  }
  const uint32_t q = p - kStagesK;
  const uint32_t blk = q / kStagesPerTile, r = q % kStagesPerTile;
  if (blk < (uint32_t)(n - 1)) {
    if (r < (uint32_t)kStagesK) { d.tile = (int)blk + 1; d.is_v = 0; d.idx = (int)r; }
    else { d.tile = (int)blk; d.is_v = 1; d.idx = (int)r - kStagesK; }
  } else {
    d.tile = n - 1; d.is_v = 1; d.idx = (int)(q - (uint32_t)(n - 1) * kStagesPerTile);
  }
  return d;
}

// Walks the cluster's segments forward to find the segment of stage st.
struct StageCursor {
  const SplitParams& p;
  int64_t u, u1;
  Segment seg;
  uint32_t base = 0;   // first global stage of seg
  bool valid = false;

  __device__ StageCursor(const SplitParams& p_, int64_t u0, int64_t u1_) : p(p_), u(u0), u1(u1_) {
    valid = find_segment(p, u, u1, seg);
  }
  // Position seg so that base <= st < base + 17 n; false once past the end.
  __device__ bool seek(uint32_t st) {
    while (valid && st >= base + (uint32_t)kStagesPerTile * seg.n) {
      base += (uint32_t)kStagesPerTile * seg.n;
      u += seg.n;
      valid = find_segment(p, u, u1, seg);
    }
    return valid;
  }
};

// Warps 4-9: gather the K and V stages of every tile with 16-byte cp.async.
// Loader warp w fills global stages w, w+6, w+12, ...; each lane copies 16
// chunks of 16 bytes (4 keys x 128 B per warp instruction) into the
// 128-byte-swizzled stage and the hardware arrives on the CTA-local full
// barrier once they land (leader: ring_full, peer: peer_full, relayed). The
// pool slots of the warp's next stage are fetched while the current stage is
// issued. Rows past the request or with a slot outside the pool are zero.
struct KvLoader {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank;
  int warp, lane;

  __device__ KvLoader(const SplitParams& p_, Ctrl* c, uint8_t* s, uint32_t r, int w)
      : p(p_), ctrl(c), smem(s), rank(r), warp(w) {
    lane = threadIdx.x & 31;
  }

  // Lane group g = lane / 8 copies a run of consecutive keys of the stage
  // (K: 16 keys, V: 8 keys); lane & 7 selects the 16-byte chunk of the 128-byte
  // row. One warp instruction therefore still moves four whole 128-byte rows,
  // and each lane fetches the slots of its run with a few vector loads.
  __device__ __forceinline__ void load_slots(const Segment& s, const StageDesc& d, int32_t (&sl)[16]) {
    const int g = lane >> 3;
    const int64_t kt = s.kt0 + d.tile;
    const int n = d.is_v ? 8 : 16;
    const int64_t pos0 = d.is_v ? kt * kKeysPerTile + (d.idx >> 1) * 32 + 8 * g
                                : kt * kKeysPerTile + rank * 64 + 16 * g;
    const int32_t* src = p.kv_indices + s.req.kv_begin + pos0;
    if (pos0 + n <= s.req.N && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0)) {
      const int4* v4 = reinterpret_cast<const int4*>(src);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (4 * q >= n) break;
        const int4 v = __ldg(v4 + q);
        sl[4 * q + 0] = v.x;
        sl[4 * q + 1] = v.y;
        sl[4 * q + 2] = v.z;
        sl[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j >= n) break;
        sl[j] = pos0 + j < s.req.N ? __ldg(src + j) : -1;
      }
    }
  }

  __device__ __forceinline__ void issue(const StageDesc& d, const int32_t (&sl)[16], uint32_t stage) {
    const uint32_t base = smem_addr(smem + kOffRing + stage * kStageBytes);
    const int ch = lane & 7, g = lane >> 3;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      int key, col, slot_j;
      uint32_t dst;
      if (!d.is_v) {
        key = 16 * g + j;
        slot_j = sl[j];
        col = d.idx * 64 + ch * 8;
        dst = base + key * 128 + ((ch ^ (key & 7)) << 4);
      } else {
        const int blk = j >> 3, dh = d.idx & 1;
        key = 8 * g + (j & 7);
        slot_j = sl[j & 7];
        col = dh * 256 + (int)rank * 128 + blk * 64 + ch * 8;
        dst = base + blk * 4096 + key * 128 + ((ch ^ (key & 7)) << 4);
      }
      const bool ok = slot_j >= 0 && (int64_t)slot_j < p.pool_slots;
      if (slot_j >= 0 && !ok) atomicOr(p.status, kStatusBadSlot);
      const uint16_t* gsrc = p.kv_pool + (ok ? (int64_t)slot_j * p.kv_stride + col : 0);
      cp_async_16(dst, gsrc, ok ? 16u : 0u);
    }
  }

  __device__ void run(int64_t u0, int64_t u1) {
    StageCursor cur(p, u0, u1), nxt(p, u0, u1);
    uint32_t st = (uint32_t)warp;
    if (!cur.seek(st)) return;
    StageDesc d = describe_stage(st - cur.base, cur.seg.n);
    int32_t sl[16], sl_next[16];
    load_slots(cur.seg, d, sl);
    uint64_t* local_full = rank == 0 ? ctrl->ring_full : ctrl->peer_full;
    while (true) {
      const uint32_t st_next = st + kNumKvWarps;
      const bool has_next = nxt.seek(st_next);
      StageDesc dn;
      if (has_next) {
        dn = describe_stage(st_next - nxt.base, nxt.seg.n);
        load_slots(nxt.seg, dn, sl_next);
      }
      const uint32_t stage = st % kNumStages, use = st / kNumStages;
      if (use >= 1 && !wait_warp(smem_addr(&ctrl->ring_empty[stage]), (use - 1) & 1u, ctrl, p, rank)) return;
      issue(d, sl, stage);
      cp_async_arrive_noinc(smem_addr(&local_full[stage]));
      if (!has_next) return;
      st = st_next;
      d = dn;
#pragma unroll
      for (int j = 0; j < 16; ++j) sl[j] = sl_next[j];
    }
  }
};

// Warp 11 of the peer CTA: forwards the completion of its stages to the
// leader's ring_full after making the cp.async-written bytes visible to the
// tensor core (async proxy). A remote release-arrive costs hundreds of
// cycles, so lanes 0..kRelayBatch-1 each take one stage of a batch and arrive
// in the same instruction.
struct Relay {
  const SplitParams& p;
  Ctrl* ctrl;
  uint32_t rank;

  __device__ Relay(const SplitParams& p_, Ctrl* c, uint32_t r) : p(p_), ctrl(c), rank(r) {}

  __device__ void run(int64_t u0, int64_t u1) {
    uint32_t total = 0;
    Segment s;
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n) total += (uint32_t)kStagesPerTile * s.n;
    const int lane = threadIdx.x & 31;
    for (uint32_t st0 = 0; st0 < total; st0 += kRelayBatch) {
      const uint32_t st = st0 + (uint32_t)lane;
      const bool mine = lane < kRelayBatch && st < total;
      bool ok = true;
      if (mine) ok = wait_one(smem_addr(&ctrl->peer_full[st % kNumStages]), (st / kNumStages) & 1u, ctrl, p, rank);
      if (!__all_sync(0xffffffffu, ok)) return;
      if (mine) {
        fence_proxy_async_smem();
        mbar_arrive_cluster(map_to_rank(smem_addr(&ctrl->ring_full[st % kNumStages]), 0));
      }
      __syncwarp();
    }
  }
};

// Warp 5: loads the CTA's 64 query rows of each segment's row tile into the
// swizzled Q buffer with 16-byte cp.async (after the previous segment's last
// score MMA released it), then announces them on the leader's q_full.
struct QLoader {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank;
  int lane;

  __device__ QLoader(const SplitParams& p_, Ctrl* c, uint8_t* s, uint32_t r) : p(p_), ctrl(c), smem(s), rank(r) {
    lane = threadIdx.x & 31;
  }

  __device__ void load_row(const Segment& s, int row) {
    const int64_t rows = (int64_t)s.req.T * p.num_heads;
    const int64_t gr = (int64_t)s.rt * kRowsPerTile + rank * kRowsPerCta + row;
    const bool valid = gr < rows;
    const int64_t t = valid ? gr / p.num_heads : 0, h = valid ? gr % p.num_heads : 0;
    const uint16_t* ql = p.q_latent + (s.req.q_begin + t) * p.ql_tok + h * p.ql_head;
    const uint16_t* qr = p.q_rope + (s.req.q_begin + t) * p.qr_tok + h * p.qr_head;
    const uint32_t base = smem_addr(smem + kOffQ) + row * 128;
    const uint32_t nbytes = valid ? 16u : 0u;
#pragma unroll 8
    for (int c = 0; c < 64; ++c)
      cp_async_16(base + (c >> 3) * 8192 + (((c & 7) ^ (row & 7)) << 4), ql + c * 8, nbytes);
#pragma unroll
    for (int c = 0; c < 8; ++c) cp_async_16(base + 8 * 8192 + ((c ^ (row & 7)) << 4), qr + c * 8, nbytes);
  }

  __device__ void run(int64_t u0, int64_t u1) {
    Segment s;
    int si = 0;
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n, ++si) {
      if (si > 0 && !wait_warp(smem_addr(&ctrl->q_empty), (si - 1) & 1, ctrl, p, rank)) return;
      load_row(s, lane);
      load_row(s, lane + 32);
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_addr(&ctrl->q_full), 0));
    }
  }
};

// ----------------------------------------------------------------------------- MMA issuer

// Global stage index (within a segment starting at `base` with n tiles) of
// stage k of K(i) or of V(i); the inverse of describe_stage.
__device__ __forceinline__ uint32_t k_stage(uint32_t base, int i, int kb) {
  return base + (i == 0 ? (uint32_t)kb : (uint32_t)(kStagesK + (i - 1) * kStagesPerTile + kb));
}
__device__ __forceinline__ uint32_t v_stage(uint32_t base, int n, int i, int v) {
  return base + (i < n - 1 ? (uint32_t)(2 * kStagesK + i * kStagesPerTile + v)
                           : (uint32_t)(kStagesK + (n - 1) * kStagesPerTile + v));
}

// Shared helpers of the two MMA-issuing threads (leader CTA only). Each
// thread's tcgen05.commit blocks it for a few hundred cycles, so score and
// value MMAs come from two threads in different warps: one thread's commits
// overlap the other's MMAs.
struct IssuerBase {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank, tmem;

  __device__ IssuerBase(const SplitParams& p_, Ctrl* c, uint8_t* s, uint32_t r, uint32_t t)
      : p(p_), ctrl(c), smem(s), rank(r), tmem(t) {}

  __device__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    if (!wait_one(smem_addr(bar), parity, ctrl, p, rank)) return false;
    tc_fence_after();
    return true;
  }
  __device__ bool wait_stage(uint32_t st) {
    if (!wait_bar(&ctrl->ring_full[st % kNumStages], (st / kNumStages) & 1u)) return false;
    fence_proxy_async_smem();   // cp.async-written bytes -> tensor-core reads
    return true;
  }
  __device__ void commit_both(uint64_t* bar) { mma_commit_2sm_mc(smem_addr(bar), (uint16_t)0x3); }
  __device__ uint64_t stage_desc(uint32_t st, uint32_t lbo) const {
    return sdesc_sw128(smem_addr(smem + kOffRing + (st % kNumStages) * kStageBytes), lbo, 1024);
  }
};

// S = Q K^T for every tile: nine K stages of four M=128, N=128, K=16 MMAs.
struct QkIssuer : IssuerBase {
  using IssuerBase::IssuerBase;

  __device__ void run(int64_t u0, int64_t u1) {
    Segment s;
    int si = 0;
    int64_t j = 0;
    uint32_t base = 0;
    const uint64_t qd = sdesc_sw128(smem_addr(smem + kOffQ), 16, 1024);
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n, ++si) {
      if (!wait_bar(&ctrl->q_full, si & 1)) return;
      for (int i = 0; i < s.n; ++i, ++j) {
        // S buffer j&1 is free once the softmax of tile j-2 has signalled its P.
        if (j >= 2 && !wait_bar(&ctrl->p_full[j & 1], (uint32_t)((j - 2) >> 1) & 1u)) return;
        const uint32_t d = tmem + kColS0 + (uint32_t)(j & 1) * 64;
        for (int kb = 0; kb < kQBlocks; ++kb) {
          const uint32_t st = k_stage(base, i, kb);
          if (!wait_stage(st)) return;
          const uint64_t bd = stage_desc(st, 16);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_2sm_bf16(d, qd + (uint64_t)((kb * 8192 + k * 32) >> 4), bd + (uint64_t)((k * 32) >> 4), kIdescQK,
                         (kb | k) != 0);
          commit_both(&ctrl->ring_empty[st % kNumStages]);
        }
        if (i == s.n - 1) commit_both(&ctrl->q_empty);
        commit_both(&ctrl->s_full[j & 1]);
      }
      base += (uint32_t)kStagesPerTile * s.n;
    }
  }
};

// O += P V for every tile: eight V stages of two M=128, N=256, K=16 MMAs.
struct PvIssuer : IssuerBase {
  using IssuerBase::IssuerBase;

  __device__ void run(int64_t u0, int64_t u1) {
    Segment s;
    int si = 0;
    int64_t j = 0;
    uint32_t base = 0;
    const uint64_t pd0 = sdesc_sw128(smem_addr(smem + kOffP), 16, 1024);
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n, ++si) {
      for (int i = 0; i < s.n; ++i, ++j) {
        if (!wait_bar(&ctrl->p_full[j & 1], (uint32_t)(j >> 1) & 1u)) return;
        if (i == 0 && si > 0 && !wait_bar(&ctrl->o_free, (si - 1) & 1)) return;
        const uint64_t pd = pd0 + (uint64_t)(((uint32_t)(j & 1) * 16384) >> 4);
        for (int v = 0; v < kStagesV; ++v) {
          const int kc = v >> 1, dh = v & 1;
          const uint32_t st = v_stage(base, s.n, i, v);
          if (!wait_stage(st)) return;
          const uint64_t bd = stage_desc(st, 4096);
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int key16 = kc * 2 + ks;   // 16-key step within the tile
            mma_2sm_bf16(tmem + kColO + dh * 128, pd + (uint64_t)(((key16 >> 2) * 8192 + (key16 & 3) * 32) >> 4),
                         bd + (uint64_t)((ks * 2048) >> 4), kIdescPV, !(i == 0 && kc == 0 && ks == 0));
          }
          commit_both(&ctrl->ring_empty[st % kNumStages]);
        }
        commit_both(&ctrl->pv_done[j & 1]);
      }
      base += (uint32_t)kStagesPerTile * s.n;
    }
  }
};

// ----------------------------------------------------------------------------- softmax / epilogue

struct Softmax {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank, tmem;
  int tid, warp, row, half;
  int64_t cluster;
  uint32_t xphase = 0;

  __device__ Softmax(const SplitParams& p_, Ctrl* c, uint8_t* s, uint32_t r, uint32_t t, int64_t cl)
      : p(p_), ctrl(c), smem(s), rank(r), tmem(t), cluster(cl) {
    tid = threadIdx.x;
    warp = tid >> 5;
    row = tid & 63;
    half = tid >> 6;
  }

  __device__ uint32_t lane_addr(uint32_t col) const { return tmem + ((uint32_t)(warp * 32) << 16) + col; }

  __device__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    if (!wait_warp(smem_addr(bar), parity, ctrl, p, rank)) return false;
    tc_fence_after();
    return true;
  }

  // Swap a value with the thread holding the other half of the same row
  // (tid ^ 64, in warp w ^ 2) through shared memory and the xchg barrier.
  __device__ bool exchange(float* buf, float mine, float& theirs) {
    buf[tid] = mine;
    mbar_arrive_local(smem_addr(&ctrl->xchg));
    if (!wait_warp(smem_addr(&ctrl->xchg), xphase & 1u, ctrl, p, rank)) return false;
    ++xphase;
    theirs = *(volatile float*)&buf[tid ^ 64];
    return true;
  }

  __device__ void signal_leader(uint64_t* bar) {
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive_cluster(map_to_rank(smem_addr(bar), 0));
  }

  __device__ void rescale_o(float alpha) {
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
      uint32_t r[32];
      tmem_ld32(lane_addr(kColO + c), r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
      tmem_st32(lane_addr(kColO + c), r);
    }
    tmem_wait_st();
  }

  __device__ bool run(int64_t u0, int64_t u1) {
    Segment s;
    int si = 0;
    int64_t j = 0;
    const float scale = p.scale_log2;
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n, ++si) {
      const int64_t rows = (int64_t)s.req.T * p.num_heads;
      const int tile_row = rank * kRowsPerCta + row;
      const int64_t gr = (int64_t)s.rt * kRowsPerTile + tile_row;
      const bool valid_row = gr < rows;
      const int64_t t = valid_row ? gr / p.num_heads : 0;
      const uint64_t anc = valid_row ? p.tree_anc[s.req.q_begin + t] : 0ull;
      const int64_t N = s.req.N, L = s.req.N - s.req.T;
      float m_run = -CUDART_INF_F, l_run = 0.f, cnt = 0.f;

      for (int i = 0; i < s.n; ++i, ++j) {
        const int64_t kt = s.kt0 + i;
        if (!wait_bar(&ctrl->s_full[j & 1], (uint32_t)(j >> 1) & 1u)) return false;
        uint32_t v[64];
        {
          uint32_t a[32], b[32];
          tmem_ld32(lane_addr(kColS0 + (uint32_t)(j & 1) * 64), a);
          tmem_ld32(lane_addr(kColS0 + (uint32_t)(j & 1) * 64 + 32), b);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            v[e] = a[e];
            v[32 + e] = b[e];
          }
        }
        const uint64_t vis = valid_row ? visible_bits(kt * kKeysPerTile + half * 64, L, N, anc) : 0ull;
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float x = ((vis >> e) & 1ull) ? __uint_as_float(v[e]) * scale : -CUDART_INF_F;
          v[e] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
        float mx_other;
        if (!exchange(ctrl->red_max[xphase & 1], mx, mx_other)) return false;
        const float m_tile = fmaxf(mx, mx_other);

        float alpha = 1.f;
        bool rescale = false;
        if (i == 0) {
          m_run = m_tile;
        } else if (m_tile > m_run + kRescaleThreshold) {
          alpha = exp2f(m_run - m_tile);
          m_run = m_tile;
          rescale = true;
        }
        const float m_use = (m_run == -CUDART_INF_F) ? 0.f : m_run;

        // P buffer j&1 was last read by the PV of tile j-2.
        if (j >= 2 && !wait_bar(&ctrl->pv_done[j & 1], (uint32_t)((j - 2) >> 1) & 1u)) return false;
        float lsum = 0.f;
        const uint32_t prow = smem_addr(smem + kOffP) + (uint32_t)(j & 1) * 16384 + half * 8192 + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = exp2f(__uint_as_float(v[c * 8 + 2 * e]) - m_use);
            const float p1 = exp2f(__uint_as_float(v[c * 8 + 2 * e + 1]) - m_use);
            lsum += p0 + p1;
            w[e] = pack_bf16x2(p0, p1);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + ((c ^ (row & 7)) << 4)), "r"(w[0]),
                       "r"(w[1]), "r"(w[2]), "r"(w[3])
                       : "memory");
        }
        l_run = l_run * alpha + lsum;
        cnt += (float)__popcll(vis);

        if (__any_sync(0xffffffffu, rescale)) {
          // O is stable once the PV of tile j-1 has completed. The whole warp
          // takes part (tcgen05.ld/st are warp-collective); rows that keep
          // their max scale by 1.
          if (!wait_bar(&ctrl->pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u)) return false;
          rescale_o(alpha);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        signal_leader(&ctrl->p_full[j & 1]);
      }

      // Epilogue: O of the segment is final once its last PV completed.
      if (!wait_bar(&ctrl->pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u)) return false;
      float l_other, c_other;
      if (!exchange(ctrl->red_l[xphase & 1], l_run, l_other)) return false;
      if (!exchange(ctrl->red_c[xphase & 1], cnt, c_other)) return false;
      const float l_tot = l_run + l_other;
      const float c_tot = cnt + c_other;
      const int64_t slot = s.g + cluster;
      float* dst = p.partial + ((slot * kRowsPerTile + tile_row) * kDLatent);
      // tcgen05.ld is warp-collective: every lane loads, only rows of the
      // request store.
#pragma unroll 1
      for (int dh = 0; dh < 2; ++dh) {
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t r[32];
          tmem_ld32(lane_addr(kColO + dh * 128 + c), r);
          tmem_wait_ld();
          if (valid_row) {
            float4* o4 = reinterpret_cast<float4*>(dst + dh * 256 + half * 128 + c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o4[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                  __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
          }
        }
      }
      if (valid_row && half == 0) p.meta[slot * kRowsPerTile + tile_row] = make_float4(m_run, l_tot, c_tot, 0.f);
      tc_fence_before();
      signal_leader(&ctrl->o_free);
    }
    return true;
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    verify_split_kernel(const SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kOffCtrl);
  const uint32_t rank = cluster_ctarank();
  const int64_t cluster = blockIdx.x >> 1;
  const int64_t G = p.num_clusters;
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumStages; ++s) {
      mbar_init(smem_addr(&ctrl->ring_full[s]), 32 + 1);   // the stage's loader warp lanes + the peer's relay
      mbar_init(smem_addr(&ctrl->peer_full[s]), 32);       // the peer's loader warp lanes
      mbar_init(smem_addr(&ctrl->ring_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&ctrl->s_full[b]), 1);
      mbar_init(smem_addr(&ctrl->p_full[b]), 8);       // 4 softmax warps x 2 CTAs
      mbar_init(smem_addr(&ctrl->pv_done[b]), 1);
    }
    mbar_init(smem_addr(&ctrl->q_full), 2);         // one Q loader warp per CTA
    mbar_init(smem_addr(&ctrl->q_empty), 1);
    mbar_init(smem_addr(&ctrl->o_free), 8);
    mbar_init(smem_addr(&ctrl->mma_final), 2);      // one commit from each issuing thread
    mbar_init(smem_addr(&ctrl->xchg), kSoftmaxThreads);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_2sm(smem_addr(&ctrl->tmem_base), kTmemCols);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  const int64_t U = total_units(p);
  const int64_t u0 = U > 0 ? unit_start(cluster, U, G) : 0;
  const int64_t u1 = U > 0 ? unit_start(cluster + 1, U, G) : 0;

  if (warp < 4) {
    Softmax sm(p, ctrl, smem, rank, tmem, cluster);
    sm.run(u0, u1);
  } else if (warp >= kKvWarp0 && warp < kKvWarp0 + kNumKvWarps) {
    KvLoader ld(p, ctrl, smem, rank, warp - kKvWarp0);
    ld.run(u0, u1);
    cp_async_wait<0>();
  } else if (warp == kRelayWarp) {
    if (rank == 1) {
      Relay rl(p, ctrl, rank);
      rl.run(u0, u1);
    }
    __syncwarp();
  } else if (warp == kQWarp) {
    QLoader ql(p, ctrl, smem, rank);
    ql.run(u0, u1);
    cp_async_wait<0>();
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    if (rank == 0 && (threadIdx.x & 31) == 0) {
      if (warp == kMmaWarp) {
        QkIssuer is(p, ctrl, smem, rank, tmem);
        is.run(u0, u1);
      } else {
        PvIssuer is(p, ctrl, smem, rank, tmem);
        is.run(u0, u1);
      }
      // Everything this thread issued completes before this arrives in both CTAs.
      mma_commit_2sm_mc(smem_addr(&ctrl->mma_final), (uint16_t)0x3);
    }
    __syncwarp();
  }

  // Both CTAs: all tensor-core work targeting this CTA's TMEM must be done
  // before the memory is released.
  if (warp == kMmaWarp && (threadIdx.x & 31) == 0) wait_one(smem_addr(&ctrl->mma_final), 0, ctrl, p, rank);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

}  // namespace

int split_smem_bytes() { return kSmemBytes; }

static cudaError_t configure_split() {
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(verify_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = 1;
  }
  return cudaSuccess;
}

// Clusters of two that can be resident at once on the current device.
cudaError_t split_max_active_clusters(int* n) {
  cudaError_t e = configure_split();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 1024, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  return cudaOccupancyMaxActiveClusters(n, verify_split_kernel, &cfg);
}

cudaError_t launch_split(const SplitParams& p, cudaStream_t stream) {
  cudaError_t e = configure_split();
  if (e != cudaSuccess) return e;
  verify_split_kernel<<<dim3(2 * p.num_clusters), dim3(kThreads), kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace va
