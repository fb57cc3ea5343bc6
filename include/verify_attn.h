/*
 * verify_attn.h -- C ABI of the B200 (sm_100a) MLA-absorb tree-verify attention.
 *
 * The operation ("MLA-absorb attention with a custom tree mask": page "The
 * Execution Phase: From Plan to 3-6x Decode Speedup on Blackwell Consumer
 * GPUs", section "The Transition: From Planning to Execution", item 3):
 *
 *   For request b with T_b tree nodes and a prefix of L_b tokens, its KV
 *   sequence has N_b = L_b + T_b positions: the prefix in order, then the tree
 *   nodes in node order (tree node i is position L_b + i). Position j lives
 *   in pool row kv_pool[kv_indices[kv_indptr[b] + j]] (a page_size=1 pool:
 *   page "The Verify Kernel Breakthrough", section "The Message in Context").
 *   Every head of every tree node t attends
 *     - every prefix position j < L_b, and
 *     - tree position L_b + i iff bit i of tree_anc[qo_indptr[b] + t] is set
 *       (ancestor-or-self mask; page "The Architecture Detective", section
 *       "The Split Verify Design": dense prefix, masked tree block),
 *   with scores  s_j = sm_scale * (q_latent[t,h,:] . c_kv[j,:] + q_rope[t,h,:] . k_rope[j,:])
 *   and values c_kv[j, 0:512] (one latent row per token serves all heads:
 *   page "The Execution Phase", section "The Core Design"), and writes
 *     out[t,h,:] = softmax_j(s_j) . c_kv,   lse[t,h] = ln sum_j exp(s_j).
 *
 * Work split (page "The Verify Kernel Breakthrough", section "The Message in
 * Context": KV-split flash-decode with partial+reduce): verify_attn_run
 * writes fp32 partial states (m, l, O) per KV split into the caller's
 * workspace; verify_attn_reduce merges them (LSE merge) into out/lse.
 *
 * Capture safety (page "The Execution Phase", section "Making the Kernel
 * CUDA Graph Capture-Safe"): the library never allocates, never
 * synchronises and never reads device data on the host inside run/reduce.
 * The launch shape depends only on the plan, so a call can be captured into
 * a CUDA graph and replayed while the per-request lengths in the device
 * indptr arrays change, as long as they stay within the plan's maxima.
 *
 * Conventions for every function below:
 *   - Pointers are DEVICE pointers unless the name ends in _h (host).
 *   - The caller owns all memory; the library keeps no pointer after return.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Strides are in elements. Every bf16 row (one token and head of q, one
 *     pool slot, one output row) must start on a 16-byte boundary: base
 *     pointers 16-byte aligned, strides multiples of 8 elements.
 *   - Return 0 on success or a negative VERIFY_ATTN_E* code; nothing is
 *     launched when an argument check fails.
 */
#ifndef VERIFY_ATTN_H
#define VERIFY_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *verify_attn_stream_t;

#define VERIFY_ATTN_OK 0
#define VERIFY_ATTN_EINVAL (-1)               /* bad pointer, size, stride, alignment or tree */
#define VERIFY_ATTN_UNSUPPORTED (-2)          /* d_latent != 512, d_rope != 64, tree > 64 nodes, too many heads */
#define VERIFY_ATTN_WORKSPACE_TOO_SMALL (-3)  /* ws_bytes below what the plan needs */
#define VERIFY_ATTN_CUDA_ERROR (-4)           /* a CUDA launch or runtime call failed */
#define VERIFY_ATTN_DEVICE_TIMEOUT (-5)       /* a bounded device-side wait gave up */
#define VERIFY_ATTN_DEVICE_BAD_INPUT (-6)     /* device lengths/slots outside the plan; the bad part was skipped */

#define VERIFY_ATTN_D_LATENT 512
#define VERIFY_ATTN_D_ROPE 64
#define VERIFY_ATTN_MAX_TREE 64
#define VERIFY_ATTN_MAX_HEADS 1024
#define VERIFY_ATTN_PLAN_VERSION 2

/* Problem maxima a plan is made for (host struct, copied into the plan). */
typedef struct {
    int32_t max_batch;       /* >= 1: most requests per call */
    int32_t num_heads;       /* H, 1..VERIFY_ATTN_MAX_HEADS */
    int32_t max_tree;        /* most tree nodes per request, 1..64 */
    int32_t d_latent;        /* must be 512 */
    int32_t d_rope;          /* must be 64 */
    int32_t num_sms;         /* SMs to plan for; 0 = ask the current device */
    int64_t max_kv_per_req;  /* most KV positions (prefix + tree) per request, >= max_tree */
    int64_t max_total_kv;    /* most KV positions summed over a call's requests */
    int64_t pool_slots;      /* rows in kv_pool; every kv_indices entry must be below this */
    float sm_scale;          /* softmax scale applied to the 576-wide dot product, finite and > 0 */
    int32_t reserved;
} verify_attn_params;

/* Launch plan: plain data, filled by verify_attn_plan, read by run/reduce.
 * Callers may copy it but should not edit it. */
typedef struct {
    int32_t version;            /* VERIFY_ATTN_PLAN_VERSION */
    int32_t num_heads;
    int32_t max_batch;
    int32_t max_tree;
    int64_t max_kv_per_req;
    int64_t max_total_kv;
    int64_t pool_slots;
    float sm_scale;
    int32_t num_clusters;       /* persistent CTA pairs of the split kernel */
    int32_t rows_per_tile;      /* (token, head) query rows per CTA pair: 128 */
    int32_t keys_per_tile;      /* KV positions per work unit: 256 */
    int32_t row_tiles_per_req;  /* ceil(max_tree * num_heads / rows_per_tile) */
    int32_t num_slots;          /* partial-state slots in the workspace */
    int64_t ws_meta_offset;     /* bytes: float4 {m, l, count, 0} per slot row */
    int64_t ws_partial_offset;  /* bytes: fp32 O[512] per slot row */
    int64_t ws_bytes;           /* total workspace bytes */
    int32_t split_smem_bytes;   /* dynamic shared memory of the split kernel */
    int32_t reserved0;
    int64_t ws_stage_offset;    /* bytes: gathered KV rows, bf16 [stage_rows, 576] */
    int64_t stage_rows;         /* keys_per_tile * (ceil(max_total_kv / keys_per_tile) + max_batch) */
    int32_t reserved[2];
} verify_attn_plan_t;

/* Per-call arguments (device pointers). */
typedef struct {
    const uint16_t *q_latent;   /* bf16 [sumT, H, 512] */
    int64_t q_latent_stride_tok, q_latent_stride_head;
    const uint16_t *q_rope;     /* bf16 [sumT, H, 64] */
    int64_t q_rope_stride_tok, q_rope_stride_head;
    const uint16_t *kv_pool;    /* bf16 [pool_slots, >=576]: c_kv in 0..511, k_rope in 512..575 */
    int64_t kv_row_stride;
    const int32_t *kv_indices;  /* [sum N_b] pool slots: prefix positions, then tree nodes */
    const int32_t *kv_indptr;   /* [batch+1] offsets into kv_indices; N_b = diff */
    const int32_t *qo_indptr;   /* [batch+1] offsets into tokens; T_b = diff, 1..max_tree */
    const uint64_t *tree_anc;   /* [sumT] ancestor-or-self bitmask over the request's tree nodes */
    int32_t batch;              /* 1..max_batch (host value, fixed for a captured graph) */
    int32_t reserved0;
    uint16_t *out;              /* bf16 [sumT, H, 512] */
    int64_t out_stride_tok, out_stride_head;
    float *lse;                 /* [sumT, H] natural-log LSE, or NULL */
    int32_t *visible_count;     /* [sumT] keys each node attended, or NULL */
} verify_attn_args;

/*
 * Validate the maxima and fill *plan and *ws_bytes (host only; queries the
 * current device's SM count when params->num_sms is 0, nothing else).
 * Returns VERIFY_ATTN_EINVAL / VERIFY_ATTN_UNSUPPORTED on bad maxima.
 */
int verify_attn_plan(const verify_attn_params *params, verify_attn_plan_t *plan, size_t *ws_bytes);

/*
 * Zero the workspace's device status word (cudaMemsetAsync on `stream`).
 * Call once after allocating a workspace and after reading a non-zero status.
 */
int verify_attn_workspace_init(const verify_attn_plan_t *plan, void *ws, size_t ws_bytes,
                               verify_attn_stream_t stream);

/*
 * Gather + split kernels. The gather copies the latent rows the requests
 * reference (kv_pool rows through kv_indices) into the staging rows of ws,
 * each request padded with zero rows to a multiple of keys_per_tile; then
 * every persistent CTA pair takes an equal share of the (query-row tile, KV
 * tile) units of the call, loads its tiles from the staging rows with TMA,
 * runs both contractions on the tensor cores and writes one fp32 partial
 * state (m, l, O) per (row tile, pair) into ws. Asynchronous on `stream`,
 * capture-safe (two kernel launches, tensor maps encoded on the host from the
 * ws pointer). Device-side length or slot errors set the status word and
 * skip the offending work (a slot outside the pool reads as a zero row).
 */
int verify_attn_run(const verify_attn_plan_t *plan, const verify_attn_args *args, void *ws,
                    size_t ws_bytes, verify_attn_stream_t stream);

/*
 * The two halves of verify_attn_run, for callers that time or schedule them
 * separately: verify_attn_gather copies the referenced latent rows into the
 * staging rows of ws; verify_attn_split runs the split kernel on them and
 * must follow a verify_attn_gather with the same plan, args and ws on the
 * same stream. Same arguments, checks and return codes as verify_attn_run.
 */
int verify_attn_gather(const verify_attn_plan_t *plan, const verify_attn_args *args, void *ws,
                       size_t ws_bytes, verify_attn_stream_t stream);
int verify_attn_split(const verify_attn_plan_t *plan, const verify_attn_args *args, void *ws,
                      size_t ws_bytes, verify_attn_stream_t stream);

/*
 * Reduce kernel: LSE-merges every row's partial states from ws into
 * args->out (bf16, round to nearest even), args->lse (natural log) and
 * args->visible_count. Must follow verify_attn_run on the same stream with
 * the same plan, args and ws. Asynchronous, capture-safe.
 */
int verify_attn_reduce(const verify_attn_plan_t *plan, const verify_attn_args *args, void *ws,
                       size_t ws_bytes, verify_attn_stream_t stream);

/*
 * Host helper: ancestor-or-self masks of one tree from its parent array
 * (parents_h[0] == -1 is the root, 0 <= parents_h[i] < i otherwise). Bit j of
 * anc_h[i] is set iff node j is node i or one of its ancestors. T in 1..64.
 * Returns VERIFY_ATTN_EINVAL for a malformed tree (anc_h untouched then).
 */
int verify_attn_build_tree_mask(const int32_t *parents_h, int32_t T, uint64_t *anc_h);

/*
 * Device version of verify_attn_build_tree_mask for a whole batch, so the
 * mask build can run inside the same captured graph as the attention (the
 * pages build the mask on the CPU every step: page "The Execution Phase",
 * section "The Methodology"). parents: [sumT] request-local parent ids
 * (root -1, otherwise 0 <= parent < node), qo_indptr: [batch+1], anc: [sumT]
 * output. A request whose tree is malformed gets only its self bits and sets
 * the tree bit of *status (a device status word such as the workspace's
 * first word, or NULL). One warp per request; asynchronous, capture-safe.
 */
int verify_attn_build_tree_mask_device(const int32_t *parents, const int32_t *qo_indptr, int32_t batch,
                                       uint64_t *anc, uint32_t *status, verify_attn_stream_t stream);

/*
 * Read the workspace's device status word: copies it to the host on
 * `stream` and synchronises that stream (not capture-safe; call after the
 * work you want to check). Returns VERIFY_ATTN_OK, VERIFY_ATTN_DEVICE_TIMEOUT,
 * VERIFY_ATTN_DEVICE_BAD_INPUT or VERIFY_ATTN_CUDA_ERROR; *detail_h (may be
 * NULL) receives the raw status bits: 1 a bounded wait expired, 2 lengths
 * outside the plan, 4 a slot outside the pool, 8 a tree mask with a bit at or
 * beyond T or without its own bit. After an expired wait, words 1-3 of the
 * workspace (uint32) record the first one: 1, the barrier's byte offset in the
 * split kernel's control block, and parity | rank << 4 | warp << 8.
 */
int verify_attn_status(const void *ws, verify_attn_stream_t stream, uint32_t *detail_h);

/* Static string for a return code. */
const char *verify_attn_strerror(int code);

/*
 * KV relocation (Tier 1 defragmentation, the step the pages deferred: live
 * relocation of a request's fragmented page_size=1 slots into contiguous ones
 * under a copy budget; page "The Execution Phase", section "Tier 0 KV
 * Defragmentation"). For request b and n_b = min(N_b, budget), KV position
 * j < n_b moves to slot dst_begin[b] + j: its 576-wide latent row is copied
 * there (skipped when already there; row padding beyond 576 is not touched)
 * and kv_indices[kv_indptr[b] + j] is rewritten. Attention over the result
 * sees exactly the same rows.
 *
 * Caller guarantees (not checked, a violation races): no destination slot is
 * referenced by any other position of the call, and destination runs of
 * different requests do not overlap. Checked on the device: each source slot
 * in [0, pool_slots) (else bit 4 of *status, position skipped) and each run
 * inside the pool (else bit 2, request skipped). Asynchronous on `stream`,
 * capture-safe, allocates nothing.
 */
typedef struct {
    uint16_t *kv_pool;          /* bf16 [pool_slots, >=576]; read and written */
    int64_t kv_row_stride;      /* elements between pool rows, >= 576, multiple of 8 */
    int64_t pool_slots;
    int32_t *kv_indices;        /* [sum N_b] slots, rewritten in place */
    const int32_t *kv_indptr;   /* [batch+1] */
    const int32_t *dst_begin;   /* [batch] first slot of each request's destination run */
    int32_t batch;              /* >= 1 */
    int32_t budget;             /* leading positions of each request to place, >= 0 */
    int64_t max_total_kv;       /* host bound on sum N_b, sizes the grid (any sum is processed) */
    uint32_t *status;           /* device word receiving error bits, or NULL */
} verify_attn_defrag_args;

int verify_attn_defrag(const verify_attn_defrag_args *args, verify_attn_stream_t stream);

/*
 * Split-verify variant (page "The Architecture Detective", section "The
 * Split Verify Design": dense attention over the prefix, a tiny masked
 * attention over the tree block, and an LSE merge of the two). The fused
 * path (verify_attn_run + verify_attn_reduce) computes the same result in
 * one pass; the variant is composed from three calls on one stream:
 *
 *   1. verify_attn_tree_block(plan, args_t, 1, self_anc, ...): tree keys that
 *      are strict ancestors of each node -> args_t->out (o_t), args_t->lse
 *      (lse_t); writes self_anc[t] = 1 << t and, if given, visible_count;
 *   2. verify_attn_run + verify_attn_reduce with tree_anc = self_anc: the
 *      prefix keys plus the node's own key -> (o_p, lse_p);
 *   3. verify_attn_merge_states: (o_p, lse_p) + (o_t, lse_t) -> out, lse.
 *
 * verify_attn_tree_block: same argument struct and checks as
 * verify_attn_reduce. The tree-block output goes to out_f32 (fp32
 * [sumT, H, 512] contiguous, 16-byte aligned) when that is non-NULL, else to
 * args->out (bf16, strides as given). The composition uses fp32 so that the
 * final output is rounded to bf16 once. args->lse (REQUIRED here) receives the
 * natural-log LSE of the tree-block key set (-inf and a zero row when the set
 * is empty).
 * exclude_self = 0 attends every key of the node's ancestor-or-self mask;
 * 1 leaves the node's own key to the dense pass. self_anc (device uint64
 * [sumT]) is optional. args->visible_count, if given, receives
 * L_b + |tree keys attended| (+1 with exclude_self). Status bits as for the
 * fused path (2 lengths, 4 slot, 8 tree), in the workspace's status word;
 * the workspace is otherwise untouched. Asynchronous, capture-safe.
 */
int verify_attn_tree_block(const verify_attn_plan_t *plan, const verify_attn_args *args, int exclude_self,
                           uint64_t *self_anc, float *out_f32, void *workspace, size_t workspace_bytes,
                           verify_attn_stream_t stream);

/*
 * Two-state LSE merge. Rows are (token, head) with token < min(max_tokens,
 * *num_tokens) (num_tokens may be NULL: max_tokens rows). o_a, out: bf16
 * [tokens, H, 512]; o_b: bf16, or fp32 when o_b_f32 = 1; all with the given
 * strides in elements (multiples of 8, 16-byte aligned bases); lse_a, lse_b,
 * lse: fp32 [tokens, H] contiguous,
 * natural log. out may alias o_a or o_b; lse may be NULL. A state with
 * lse = -inf has weight 0; two such states give a zero row and -inf.
 */
typedef struct {
    const uint16_t *o_a;
    int64_t o_a_stride_tok, o_a_stride_head;
    const float *lse_a;
    const void *o_b;
    int64_t o_b_stride_tok, o_b_stride_head;
    const float *lse_b;
    int32_t o_b_f32;             /* 0: o_b is bf16, 1: fp32 */
    uint16_t *out;
    int64_t out_stride_tok, out_stride_head;
    float *lse;
    int64_t max_tokens;
    const int32_t *num_tokens;   /* device int32, or NULL */
    int32_t num_heads;
} verify_attn_merge_args;

int verify_attn_merge_states(const verify_attn_merge_args *args, verify_attn_stream_t stream);

/*
 * Stacked R-state LSE merge, the combine step of KV-sequence sharding: each
 * of R ranks attends a disjoint part of every row's visible keys (its
 * prefix chunk; the last rank also takes the tree block) and returns
 * (o_r, lse_r); the R states are gathered along a leading axis and merged
 * (page "The Breakthrough", section "The Message in Context": KV-split
 * partials combined by a reduce; page "The Architecture Detective",
 * section "The Split Verify Design": LSE merge). With m = max_r lse_r and
 * w_r = exp(lse_r - m): out = sum_r w_r o_r / sum_r w_r, lse = m + ln sum_r w_r.
 * States with lse = -inf have weight 0; all empty gives a zero row and -inf.
 *
 * o: bf16 [R, max_tokens, H, 512] contiguous, 16-byte aligned; lse_states:
 * fp32 [R, max_tokens, H]; out: bf16 [tokens, H, 512] with the given strides
 * (multiples of 8 elements); lse: fp32 [tokens, H] or NULL. Rows are tokens <
 * min(max_tokens, *num_tokens) (num_tokens may be NULL). out must not alias o.
 */
typedef struct {
    const uint16_t *o;
    const float *lse_states;
    int32_t num_states;          /* R, 1..1024 */
    int32_t num_heads;
    uint16_t *out;
    int64_t out_stride_tok, out_stride_head;
    float *lse;
    int64_t max_tokens;
    const int32_t *num_tokens;   /* device int32, or NULL */
} verify_attn_merge_stacked_args;

int verify_attn_merge_stacked(const verify_attn_merge_stacked_args *args, verify_attn_stream_t stream);

/* Size of the library-owned workspace used by verify_attn_forward_static. */
#define VERIFY_ATTN_STATIC_WS_BYTES (128u << 20)

/*
 * verify_attn_forward_static -- run + reduce without any allocation.
 *
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory when they run the verify step: a serving loop
 * that must stay allocation-free after warm-up, a runtime that owns the device
 * heap and forbids other allocators, or a plugin that only receives the
 * tensors it may read and write. Such a caller passes its inputs and outputs
 * as for verify_attn_run / verify_attn_reduce; the scratch those kernels need
 * comes from a fixed array of VERIFY_ATTN_STATIC_WS_BYTES (128 MiB) inside the
 * library, which every GPU that uses the library keeps until the process
 * exits.
 *
 * - Plans whose ws_bytes exceed VERIFY_ATTN_STATIC_WS_BYTES are rejected with
 *   VERIFY_ATTN_WORKSPACE_TOO_SMALL before anything is launched.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture on the device.
 * - Every call shares the one array, which keeps the previous call's
 *   contents; the call clears the status word itself. Calls that overlap on
 *   the GPU (other streams, other host threads) race on it.
 * - status: a caller-owned device uint32 that receives the status word at
 *   the end of the call (same bits as verify_attn_status), or NULL.
 * - No cudaMalloc, cudaFree or other allocating routine is called.
 * Returns the same codes as verify_attn_run / verify_attn_reduce.
 */
int verify_attn_forward_static(const verify_attn_plan_t *plan, const verify_attn_args *args, uint32_t *status,
                               verify_attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VERIFY_ATTN_H */
