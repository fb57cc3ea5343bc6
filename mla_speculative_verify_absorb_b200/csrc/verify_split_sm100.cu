// Split kernel of the MLA-absorb tree-verify attention for B200 (sm_100a).
//
// What it computes (page "The Execution Phase", section "The Transition:
// From Planning to Execution": MLA-absorb attention with a custom tree mask;
// section "The Core Design": KV tile loaded once for all heads): for a tile
// of 128 query rows (token, head) of one request and a run of KV tiles of
// 256 positions, the fp32 partial state
//     m = running max of the scaled scores (log2 units),
//     l = sum 2^(s - m),  O = sum 2^(s - m) * c_kv,  count = visible keys,
// written per (row tile, CTA pair) for the LSE-merge reduce (page "The
// Verify Kernel Breakthrough", section "The Message in Context": KV-split
// partials plus reduce).
//
// How (B200-specific; the pages' sm_120 kernel is prior art, not the plan):
//  * The KV rows of the call were first copied, in key order, into a
//    contiguous staging area (verify_gather.cu), so every K and V stage is
//    a box of a 2-D or 3-D tensor map over those rows and moves with tiled
//    TMA copies (two adjacent stages with one copy where the ring allows):
//    no load/store-unit work per key and no per-key slot lookups here.
//  * A cluster of two CTAs on two SMs shares one 128-row tile: each CTA
//    holds 64 rows of Q in shared memory and the pair issues
//    tcgen05.mma.cta_group::2 with M = 128. In that mode a CTA's accumulator
//    of N columns takes N/2 TMEM columns (lanes 0-63: columns [0, N/2) of its
//    64 rows, lanes 64-127: columns [N/2, N)), which is what lets the 512-wide
//    fp32 output accumulator (256 TMEM columns) sit beside two 256-key score
//    buffers (128 columns each).
//  * S = Q K^T: M = 128 rows, N = 256 keys (each CTA loads 128 of them),
//    K = 576 in nine 64-wide blocks. O += P V: M = 128, N = 256 value columns
//    per instruction, K = keys; CTA r supplies value columns [256 r, 256 r +
//    256), so each CTA loads half of every V row. Both contractions run at
//    N = 256, the shape at which the pair's tensor cores stay saturated.
//  * Two warps per CTA issue the TMA copies into a ring of 16 KB stages,
//    taking alternate stages (bulk copies issued by one thread complete one
//    after another, so a single issuing thread cannot keep enough bytes in
//    flight), counting both CTAs' bytes on the leader's barrier
//    (cta_group::2); one warp of the leader issues every MMA of the pair.
//    These warps run converged, with one elected lane executing each copy,
//    MMA and commit, so the operands stay warp-uniform; four softmax
//    warps per CTA read S from TMEM, apply scale and the ancestor mask, keep
//    the online softmax (the O rescale is skipped unless the row max grows
//    by more than 2^8), write bf16 P into shared memory and finally dump O
//    to the workspace.
//  * Persistent grid: cluster c of G takes an equal share of the call's
//    (row tile, key tile) units, so work is balanced whatever the mix of
//    request lengths, and at most G + #row tiles partial states are written.
//  * Every wait is bounded; on expiry the kernel records it in the status
//    word, unwinds both CTAs and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"
#include "verify_attn_internal.h"
#include "verify_split.h"

namespace va {
namespace {

using namespace ptx;

constexpr int kThreads = 256;          // 4 softmax + 2 TMA producers + Q loader + MMA warps
constexpr int kSoftmaxThreads = 128;
constexpr int kProdWarp = 4;           // warps 4 and 7 issue the K/V TMA copies of their CTA
constexpr int kProdWarp2 = 7;
constexpr int kProducers = 2;
constexpr int kQWarp = 5;
constexpr int kMmaWarp = 6;            // issues all MMAs; also owns the TMEM allocation

constexpr int kStageBytes = 16384;
constexpr int kNumStages = 7;
constexpr int kQBlocks = kDQK / 64;    // 9 blocks of 64 columns
constexpr int kOffQ = 0;               // 9 x [64 rows x 128 B]
constexpr int kOffP = kOffQ + kQBlocks * 8192;   // 4 key blocks x [64 rows x 128 B]
constexpr int kOffRing = kOffP + 4 * 8192;
constexpr int kOffCtrl = kOffRing + kNumStages * kStageBytes;
static_assert(kOffRing % 1024 == 0 && kOffP % 1024 == 0, "swizzled buffers need 1 KB alignment");

// TMEM columns (per CTA; 2x2 layout of the pair MMA).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;        // S buffers: 128 columns each
constexpr uint32_t kColO = 256;       // O: two 128-column halves (MMA dh = 0, 1)

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 256, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, true);

constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainNs = 200000ull;    // after an abort: time for copies in flight to land

struct Ctrl {
  uint64_t ring_full[kNumStages];   // leader: expect_tx by its producer, bytes of both CTAs
  uint64_t ring_empty[kNumStages];  // both CTAs: the consuming MMAs' commit
  uint64_t s_full[2];
  uint64_t s_free[2];               // leader: 4 softmax warps x 2 CTAs have read S
  uint64_t p_full;                  // leader: 4 softmax warps x 2 CTAs have written P
  uint64_t pv_done;
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t o_free;
  uint64_t mma_final;
  uint64_t xchg;          // softmax-thread exchange of row maxima and sums (128 arrivals)
  uint32_t tmem_base;
  int32_t abort_flag;
  float red[2][kSoftmaxThreads];
};

constexpr int kSmemBytes = kOffCtrl + (int)sizeof(Ctrl) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "split kernel shared memory exceeds the sm_100 limit");

struct Segment {
  Request req;
  int32_t b, rt, kt0, n;
  int32_t kt_base;   // first staging tile of the request
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
  int32_t kt_base = 0;
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
      s.kt_base = kt_base;
      int64_t left = u_end - u;
      s.n = (int32_t)((int64_t)(r.key_tiles - s.kt0) < left ? (r.key_tiles - s.kt0) : left);
      return true;
    }
    acc += ub;
    g += r.row_tiles;
    kt_base += r.key_tiles;
  }
  return false;
}

// Records an expired wait: the status bit, and for the first one in the
// workspace the barrier (its byte offset in Ctrl), the phase parity waited
// for, and the CTA rank and warp that waited.
__device__ void give_up(Ctrl* ctrl, const SplitParams& p, uint32_t rank, uint32_t bar, uint32_t parity) {
  atomicOr(p.status, kStatusTimeout);
  if (atomicCAS(p.status + 1, 0u, 1u) == 0u) {
    p.status[2] = bar - smem_addr(ctrl);
    p.status[3] = parity | (rank << 4) | ((threadIdx.x >> 5) << 8);
  }
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
      give_up(ctrl, p, rank, bar, parity);
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
        give_up(ctrl, p, rank, bar, parity);
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

// Stage order of one segment of n tiles, shared by the producers and the MMA
// issuer: K(0), then for i = 1..n-1: K(i), V(i-1), then V(n-1). K(i) is 9
// stages (one 64-column block of the 576 score columns for the CTA's 128
// keys), V(i) 8 stages (64 keys x two 64-column blocks of the CTA's value
// columns; stage v covers keys 64 (v >> 1) .. +63 and blocks 2 (v & 1), +1),
// so a segment has 17 n stages.
constexpr int kStagesK = kQBlocks;    // 9
constexpr int kStagesV = 8;

// Warps 4 and 7 of each CTA: both walk the cluster's stages in order and
// each loads every other one into the ring with tiled TMA copies from the
// staging rows. K stage of block kb: box [128 keys x 64 columns] at column 64 kb, keys 128 r .. of the
// tile (CTA r). V stage: one box of a 3-D view of the same rows, [2 column
// blocks x 64 keys x 64 columns], value columns 256 r + 128 h .. + 127. The leader's warp announces both CTAs' bytes on
// its ring_full barrier; the peer's copies count their bytes there too.
// Two consecutive K blocks of a tile travel as one 32 KB copy when their
// ring slots are adjacent (no wrap); the producers and the issuer take the
// same decision from the stage index.
__device__ __forceinline__ int k_blocks_at(int kb, uint32_t st) {
  return (kb + 1 < kStagesK && (int)(st % kNumStages) + 1 < kNumStages) ? 2 : 1;
}
// Likewise the two V stages of one 64-key quarter (value halves h = 0, 1).
__device__ __forceinline__ int v_stages_at(int v, uint32_t st) {
  return ((v & 1) == 0 && (int)(st % kNumStages) + 1 < kNumStages) ? 2 : 1;
}

struct Producer {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank;
  const CUtensorMap* tm_k;    // [128 keys x 64 columns] boxes
  const CUtensorMap* tm_k2;   // [2 blocks x 128 keys x 64 columns] boxes
  const CUtensorMap* tm_v;    // [2 blocks x 64 keys x 64 columns] boxes
  const CUtensorMap* tm_v2;   // [4 blocks x 64 keys x 64 columns] boxes
  uint32_t which;      // this warp takes the copies op with op % kProducers == which
  uint32_t st = 0, op = 0;
  bool alive = true;
  uint64_t policy = l2_policy_evict_last();   // every K/V tile is re-read by all row tiles

  __device__ bool mine() const { return alive && op % kProducers == which; }

  // The n (1 or 2) slots of stages st..st+n-1: wait (whole warp) until the
  // MMAs of the last slot's previous use completed (stages are released in
  // order, so the earlier slot is free too), then (leader) announce the bytes
  // both CTAs will land on the first slot's full barrier and complete the
  // other slot's phase with a plain arrival.
  __device__ bool acquire(int n, uint32_t& dst, uint32_t& bar) {
    const uint32_t last = st + (uint32_t)n - 1;
    const uint32_t use = last / kNumStages;
    if (use >= 1) {
      const uint32_t e = smem_addr(&ctrl->ring_empty[last % kNumStages]), par = (use - 1) & 1u;
      bool ok = false;
      for (int spin = 0; spin < 1024 && !ok; ++spin) ok = __all_sync(0xffffffffu, mbar_test_wait_cta(e, par));
      if (!ok && !wait_warp(e, par, ctrl, p, rank)) return alive = false;
    }
    const uint32_t stage = st % kNumStages;
    const uint32_t full = smem_addr(&ctrl->ring_full[stage]);
    if (rank == 0) {
      mbar_arrive_expect_tx_local_elect(full, (uint32_t)n * 2u * kStageBytes);
      if (n == 2) mbar_arrive_local_elect(smem_addr(&ctrl->ring_full[stage + 1]));
    }
    bar = map_to_rank(full, 0);
    dst = smem_addr(smem + kOffRing + stage * kStageBytes);
    return true;
  }
  __device__ void load_k(int32_t row0) {
    for (int kb = 0; kb < kStagesK; ++op) {
      const int n = k_blocks_at(kb, st);
      uint32_t dst, bar;
      if (mine() && acquire(n, dst, bar)) {
        if (n == 2)
          tma_load_3d_2sm_elect(dst, tm_k2, 0, row0 + 128 * (int32_t)rank, kb, bar, policy);
        else
          tma_load_2d_2sm_elect(dst, tm_k, 64 * kb, row0 + 128 * (int32_t)rank, bar, policy);
      }
      st += (uint32_t)n;
      kb += n;
    }
  }
  __device__ void load_v(int32_t row0) {
    for (int v = 0; v < kStagesV; ++op) {
      const int n = v_stages_at(v, st);
      uint32_t dst, bar;
      if (mine() && acquire(n, dst, bar)) {
        // Stage (quarter q, half h): blocks 4 r + 2 h, +1 of keys 64 q ..;
        // a pair of stages is the four blocks 4 r .. 4 r + 3.
        const int32_t key = row0 + 64 * (v >> 1);
        if (n == 2)
          tma_load_3d_2sm_elect(dst, tm_v2, 0, key, 4 * (int32_t)rank, bar, policy);
        else
          tma_load_3d_2sm_elect(dst, tm_v, 0, key, 4 * (int32_t)rank + 2 * (v & 1), bar, policy);
      }
      st += (uint32_t)n;
      v += n;
    }
  }

  __device__ void run(int64_t u0, int64_t u1) {
    Segment s;
    for (int64_t u = u0; alive && find_segment(p, u, u1, s); u += s.n) {
      const int32_t row0 = (s.kt_base + s.kt0) * kKeysPerTile;
      load_k(row0);
      for (int i = 1; i < s.n; ++i) {
        load_k(row0 + i * kKeysPerTile);
        load_v(row0 + (i - 1) * kKeysPerTile);
      }
      load_v(row0 + (s.n - 1) * kKeysPerTile);
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

// ----------------------------------------------------------------------------- MMA issuers

// The MMA issuer: warp 6 of the leader CTA issues every tcgen05.mma of the
// pair, in ring order, so the two SMs' tensor cores always see one
// instruction stream (two issuing threads interleaving pair MMAs were seen
// to hang the pair). For each stage: K stage of tile i -> four M=128, N=256,
// K=16 score MMAs into S buffer (j & 1); V stage -> four value MMAs into one
// half of O. Before the first K stage of a tile it waits until the softmax
// warps have read S of tile j-2 from that buffer (and at a segment start for
// the segment's Q); before the first V stage of a tile, for P of that tile
// (and at a segment start for the previous segment's O to be stored). Each
// stage is released to the producers by a commit once its MMAs complete.
struct Issuer {
  const SplitParams& p;
  Ctrl* ctrl;
  uint8_t* smem;
  uint32_t rank, tmem;
  uint32_t st = 0;
  uint64_t qd = 0, pd = 0;

  __device__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    if (!wait_warp(smem_addr(bar), parity, ctrl, p, rank)) return false;
    tc_fence_after();
    return true;
  }
  // A ring stage is usually landed or about to: poll it without sleeping
  // before falling back to the bounded wait.
  __device__ bool wait_stage(uint32_t& saddr) {
    const uint32_t stage = st % kNumStages, parity = (st / kNumStages) & 1u;
    const uint32_t bar = smem_addr(&ctrl->ring_full[stage]);
    bool ok = false;
    for (int spin = 0; spin < 4096 && !ok; ++spin) ok = __all_sync(0xffffffffu, mbar_test_wait_cta(bar, parity));
    if (!ok && !wait_warp(bar, parity, ctrl, p, rank)) return false;
    saddr = smem_addr(smem + kOffRing + stage * kStageBytes);
    return true;
  }
  __device__ void release_stage() {
    mma_commit_2sm_mc_elect(smem_addr(&ctrl->ring_empty[st % kNumStages]), (uint16_t)0x3);
    ++st;
  }
  __device__ void commit_both(uint64_t* bar) { mma_commit_2sm_mc_elect(smem_addr(bar), (uint16_t)0x3); }

  // S(j) = Q K(j)^T from the nine K stages of tile j.
  __device__ bool score(int64_t j, bool last_of_segment) {
    // S buffer j&1 is free once the softmax warps have read S of tile j-2.
    if (j >= 2 && !wait_bar(&ctrl->s_free[j & 1], (uint32_t)((j - 2) >> 1) & 1u)) return false;
    const uint32_t dt = tmem + kColS0 + (uint32_t)(j & 1) * 128;
    for (int kb0 = 0; kb0 < kStagesK;) {
      const int n = k_blocks_at(kb0, st);   // a two-block copy lands on its first stage's barrier
      uint32_t saddr;
      if (!wait_stage(saddr)) return false;
      for (int b = 0; b < n; ++b) {
        const int kb = kb0 + b;
        const uint64_t bd = sdesc_sw128(saddr + (uint32_t)b * kStageBytes, 16, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_2sm_bf16_elect(dt, qd + (uint64_t)((kb * 8192 + k * 32) >> 4), bd + (uint64_t)((k * 32) >> 4),
                             kIdescQK, (kb | k) != 0);
        release_stage();
      }
      kb0 += n;
    }
    if (last_of_segment) commit_both(&ctrl->q_empty);
    commit_both(&ctrl->s_full[j & 1]);
    return true;
  }
  // O += P(j) V(j) from the eight V stages of tile j.
  __device__ bool value(int64_t j, bool first_of_segment, int si) {
    if (!wait_bar(&ctrl->p_full, (uint32_t)(j & 1))) return false;
    if (first_of_segment && si > 0 && !wait_bar(&ctrl->o_free, (si - 1) & 1)) return false;
    for (int v0 = 0; v0 < kStagesV;) {
      const int n = v_stages_at(v0, st);   // a two-stage copy lands on its first stage's barrier
      uint32_t saddr;
      if (!wait_stage(saddr)) return false;
      for (int b = 0; b < n; ++b) {
        const int v = v0 + b, kq = v >> 1, dh = v & 1;
        const uint64_t bd = sdesc_sw128(saddr + (uint32_t)b * kStageBytes, 8192, 1024);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_2sm_bf16_elect(tmem + kColO + dh * 128, pd + (uint64_t)((kq * 8192 + ks * 32) >> 4),
                             bd + (uint64_t)((ks * 2048) >> 4), kIdescPV, !(first_of_segment && kq == 0 && ks == 0));
        release_stage();
      }
      v0 += n;
    }
    commit_both(&ctrl->pv_done);
    return true;
  }

  __device__ void run(int64_t u0, int64_t u1) {
    Segment s;
    int si = 0;
    int64_t j = 0;   // global index of the segment's first tile
    qd = sdesc_sw128(smem_addr(smem + kOffQ), 16, 1024);
    pd = sdesc_sw128(smem_addr(smem + kOffP), 16, 1024);
    for (int64_t u = u0; find_segment(p, u, u1, s); u += s.n, ++si, j += s.n) {
      if (!wait_bar(&ctrl->q_full, si & 1)) return;
      if (!score(j, s.n == 1)) return;
      for (int i = 1; i < s.n; ++i) {
        if (!score(j + i, i == s.n - 1)) return;
        if (!value(j + i - 1, i == 1, si)) return;
      }
      if (!value(j + s.n - 1, s.n == 1, si)) return;
    }
  }
};

// ----------------------------------------------------------------------------- softmax / epilogue

// Warps 0-3 of both CTAs. Thread (row, half) owns TMEM lane 64 half + row:
// keys [128 half, 128 half + 128) of every score tile and value columns
// [256 half, 256 half + 256) of O (MMA dh gives columns 128 dh .. of that run).
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
  __device__ bool exchange(float mine, float& theirs) {
    float* buf = ctrl->red[xphase & 1];
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
        const int64_t key0 = (int64_t)(s.kt0 + i) * kKeysPerTile + half * 128;
        if (!wait_bar(&ctrl->s_full[j & 1], (uint32_t)(j >> 1) & 1u)) return false;
        uint32_t v[128];
        {
          const uint32_t col = kColS0 + (uint32_t)(j & 1) * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(lane_addr(col + 32 * c), *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
          tmem_wait_ld();
        }
        // S of this tile is in registers: the buffer can take tile j+2.
        tc_fence_before();
        signal_leader(&ctrl->s_free[j & 1]);

        const uint64_t vis0 = valid_row ? visible_bits(key0, L, N, anc) : 0ull;
        const uint64_t vis1 = valid_row ? visible_bits(key0 + 64, L, N, anc) : 0ull;
        // Row max of the raw scores (the scale is positive, so it commutes
        // with max), over eight independent chains; masked keys become -inf.
        // Tiles inside the prefix are fully visible for the whole warp.
        float mk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = -CUDART_INF_F;
        if (__all_sync(0xffffffffu, (vis0 & vis1) == ~0ull)) {
#pragma unroll
          for (int e = 0; e < 128; ++e) mk[e & 7] = fmaxf(mk[e & 7], __uint_as_float(v[e]));
        } else {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            const uint64_t vis = e < 64 ? vis0 : vis1;
            const float x = ((vis >> (e & 63)) & 1ull) ? __uint_as_float(v[e]) : -CUDART_INF_F;
            v[e] = __float_as_uint(x);
            mk[e & 7] = fmaxf(mk[e & 7], x);
          }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])),
                               fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7])));
        float mx_other;
        if (!exchange(mx, mx_other)) return false;
        const float m_tile = fmaxf(mx, mx_other) * scale;

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

        // p = 2^(s * scale - m): one packed FMA per two keys, then the
        // exponentials; the row sum over four packed chains.
        const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(-m_use, -m_use);
        float2 sum2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) sum2[k] = make_float2(0.f, 0.f);
        uint32_t w[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float2 a = __ffma2_rn(make_float2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2, nm2);
          const float2 pe = make_float2(exp2f(a.x), exp2f(a.y));
          sum2[e & 3] = __fadd2_rn(sum2[e & 3], pe);
          w[e] = pack_bf16x2(pe.x, pe.y);
        }
        const float2 s01 = __fadd2_rn(sum2[0], sum2[1]), s23 = __fadd2_rn(sum2[2], sum2[3]);
        const float lsum = (s01.x + s01.y) + (s23.x + s23.y);
        l_run = l_run * alpha + lsum;
        cnt += (float)(__popcll(vis0) + __popcll(vis1));

        // P (single buffer) and O are free once the PV of tile j-1 completed.
        if (j >= 1 && !wait_bar(&ctrl->pv_done, (uint32_t)((j - 1) & 1))) return false;
        const uint32_t prow = smem_addr(smem + kOffP) + (uint32_t)half * 16384 + row * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + (c >> 3) * 8192 +
                                                                         (((c & 7) ^ (row & 7)) << 4)),
                       "r"(w[4 * c]), "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                       : "memory");
        }
        // The whole warp takes part (tcgen05.ld/st are warp-collective); rows
        // that keep their max scale by 1.
        if (__any_sync(0xffffffffu, rescale)) rescale_o(alpha);
        fence_proxy_async_smem();
        tc_fence_before();
        signal_leader(&ctrl->p_full);
      }

      // Epilogue: O of the segment is final once its last PV completed.
      if (!wait_bar(&ctrl->pv_done, (uint32_t)((j - 1) & 1))) return false;
      float l_other, c_other;
      if (!exchange(l_run, l_other)) return false;
      if (!exchange(cnt, c_other)) return false;
      const float l_tot = l_run + l_other;
      const float c_tot = cnt + c_other;
      const int64_t slot = s.g + cluster;
      float* dst = p.partial + ((slot * kRowsPerTile + tile_row) * kDLatent) + half * 256;
      // tcgen05.ld is warp-collective: every lane loads, only rows of the
      // request store.
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr(kColO + c), r);
        tmem_wait_ld();
        if (valid_row) {
          float4* o4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            o4[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
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
    verify_split_kernel(const SplitParams p, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_k2, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_v2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kOffCtrl);
  const uint32_t rank = cluster_ctarank();
  const int64_t cluster = blockIdx.x >> 1;
  const int64_t G = p.num_clusters;
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumStages; ++s) {
      mbar_init(smem_addr(&ctrl->ring_full[s]), 1);   // the leader's expect_tx arrival
      mbar_init(smem_addr(&ctrl->ring_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&ctrl->s_full[b]), 1);
      mbar_init(smem_addr(&ctrl->s_free[b]), 8);      // 4 softmax warps x 2 CTAs
    }
    mbar_init(smem_addr(&ctrl->p_full), 8);
    mbar_init(smem_addr(&ctrl->pv_done), 1);
    mbar_init(smem_addr(&ctrl->q_full), 2);         // one Q loader warp per CTA
    mbar_init(smem_addr(&ctrl->q_empty), 1);
    mbar_init(smem_addr(&ctrl->o_free), 8);
    mbar_init(smem_addr(&ctrl->mma_final), 1);      // the issuing thread's last commit
    mbar_init(smem_addr(&ctrl->xchg), kSoftmaxThreads);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProdWarp && (threadIdx.x & 31) == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_k2);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_v2);
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
  } else if (warp == kProdWarp || warp == kProdWarp2) {
    Producer pr{p, ctrl, smem, rank, &tm_k, &tm_k2, &tm_v, &tm_v2, warp == kProdWarp ? 0u : 1u};
    pr.run(u0, u1);
    // After an abort, copies issued before it may still be in flight:
    // give them time to land before the CTA can exit.
    if ((threadIdx.x & 31) == 0 && *(volatile int32_t*)&ctrl->abort_flag) {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < kDrainNs) {
      }
    }
    __syncwarp();
  } else if (warp == kQWarp) {
    QLoader ql(p, ctrl, smem, rank);
    ql.run(u0, u1);
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    if (rank == 0) {
      Issuer is{p, ctrl, smem, rank, tmem};
      is.run(u0, u1);
      // Everything the warp issued completes before this arrives in both CTAs.
      mma_commit_2sm_mc_elect(smem_addr(&ctrl->mma_final), (uint16_t)0x3);
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Tensor map over the staging rows: [stage_rows rows, 576 bf16 columns], row
// stride 1152 bytes, boxes of 64 columns x `box_rows` rows with the 128-byte
// swizzle that the tensor-core operand descriptors expect.
cudaError_t encode_stage_map(const SplitParams& p, uint32_t box_rows, CUtensorMap* map) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return e != cudaSuccess ? e : cudaErrorNotSupported;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)p.stage_rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p.stage), dims, strides, box,
                      estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D view of the staging rows: (64 columns of a block, key row, 64-column
// block index) with strides (2 B, 1152 B, 128 B). A box [2 blocks x 64 keys x
// 64 columns] lands as two 8 KB blocks of 64 swizzled 128-byte rows (a V
// stage, the MN-major operand of the value MMA), [4 blocks x 64 keys x 64
// columns] as two consecutive V stages, and [2 blocks x 128 keys x 64
// columns] as two consecutive K stages.
cudaError_t encode_stage_blocks_map(const SplitParams& p, uint32_t box_keys, uint32_t box_blocks, CUtensorMap* map) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return e != cudaSuccess ? e : cudaErrorNotSupported;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  const cuuint64_t dims[3] = {64, (cuuint64_t)p.stage_rows, (cuuint64_t)(kDQK / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)kDQK * 2, 128};
  const cuuint32_t box[3] = {64, box_keys, box_blocks};
  const cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(p.stage), dims, strides, box,
                      estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
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
  CUtensorMap tm_k, tm_k2, tm_v, tm_v2;
  e = encode_stage_map(p, 128, &tm_k);
  if (e != cudaSuccess) return e;
  e = encode_stage_blocks_map(p, 128, 2, &tm_k2);
  if (e != cudaSuccess) return e;
  e = encode_stage_blocks_map(p, 64, 2, &tm_v);
  if (e != cudaSuccess) return e;
  e = encode_stage_blocks_map(p, 64, 4, &tm_v2);
  if (e != cudaSuccess) return e;
  verify_split_kernel<<<dim3(2 * p.num_clusters), dim3(kThreads), kSmemBytes, stream>>>(p, tm_k, tm_k2, tm_v, tm_v2);
  return cudaGetLastError();
}

}  // namespace va
