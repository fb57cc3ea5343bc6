/*
 * CPU oracle for MLA-absorb tree-verify attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this file's library. The product path (the CUDA library and its
 * Python binding) never calls into it, and the two share no code.
 *
 * Plain, slow, float64. Every bf16 input is widened exactly to double; no
 * blocking, no fusion, no reordering beyond what each definition states.
 *
 * What is computed, and where it comes from:
 *
 *  - The operation is "MLA-absorb attention with a custom tree mask"
 *    (page "The Execution Phase: From Plan to 3-6x Decode Speedup on
 *    Blackwell Consumer GPUs", section "The Transition: From Planning to
 *    Execution", item 3). All heads read the same latent row of a token
 *    (same page, section "The Core Design: A Streaming Flash Attention
 *    Kernel": one latent read serves every head), so there is one KV head.
 *  - Score of query (token r, head h) against key position j of its request:
 *        s_j = scale * ( q_latent[r,h,:] . c_kv[slot_j,:]  +  q_rope[r,h,:] . k_rope[slot_j,:] )
 *    and the value of key j is its latent c_kv[slot_j, 0:512]. The latent
 *    and rope widths (512, 64) and the scale 192^-0.5 are the workload's
 *    given constants.
 *  - Visibility: tree node t of a request with prefix length L sees every
 *    prefix position 0..L-1 and the tree positions L+i whose node i is an
 *    ancestor of t or t itself (page "The Architecture Detective", section
 *    "The Split Verify Design": the tree queries attend the whole prefix
 *    densely, only the tree block carries the custom mask). Tree node i is
 *    stored at KV position L+i (prefix first, then tree nodes in node order).
 *  - Output: softmax over the visible scores, applied to the visible values;
 *    lse = max + ln(sum exp(s - max)).
 *  - Partial states and their merge: the split kernel of the pages writes
 *    partial results per KV split and a reduce merges them ("The Verify
 *    Kernel Breakthrough", section "The Message in Context": KV-split
 *    flash-decode with partial+reduce; page "The Architecture Detective",
 *    section "The Split Verify Design": LSE merge). A partial state over a
 *    key range is (m, l, O) with m = max score, l = sum exp(s - m),
 *    O = sum exp(s - m) * v; the merge is
 *        m* = max m_s,  l* = sum l_s e^(m_s - m*),
 *        out = sum O_s e^(m_s - m*) / l*,  lse = m* + ln l*,
 *    and a state with l = 0 (no visible key) contributes nothing.
 *
 * Pins that check this file against things other than itself live in the
 * tests: chain tree == causal attention from a library routine, a single
 * visible token returns its latent row exactly, equal scores return the mean
 * row, permuting pool rows with kv_indices changes nothing, a numpy brute
 * force agrees on tiny inputs, and the merge of two partial states equals the
 * one-shot result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_D_LATENT 512
#define ORACLE_D_ROPE 64
#define ORACLE_D_QK (ORACLE_D_LATENT + ORACLE_D_ROPE)
#define ORACLE_MAX_TREE 64

/* bf16 bit pattern -> double, exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Ancestor-or-self masks of one tree. parents[0] must be -1 (node 0 is the
 * root); every other node i needs 0 <= parents[i] < i. Bit j of anc[i] is set
 * iff node j lies on the path from node i up to the root, i itself included.
 * Returns 0, or -1 for an invalid tree (anc is then left unspecified).
 */
int oracle_ancestor_masks(const int32_t *parents, int32_t T, uint64_t *anc) {
    if (T < 1 || T > ORACLE_MAX_TREE) return -1;
    if (parents[0] != -1) return -1;
    for (int32_t i = 1; i < T; ++i)
        if (parents[i] < 0 || parents[i] >= i) return -1;
    for (int32_t i = 0; i < T; ++i) {
        uint64_t bits = 0;
        int32_t j = i;
        while (j >= 0) {            /* walk up to the root */
            bits |= (uint64_t)1 << j;
            j = parents[j];
        }
        anc[i] = bits;
    }
    return 0;
}

/* Locate the request b and the tree node t of flattened token row r. */
static int find_request(int32_t B, const int32_t *qo_indptr, int64_t r, int32_t *b_out) {
    for (int32_t b = 0; b < B; ++b) {
        if (r >= qo_indptr[b] && r < qo_indptr[b + 1]) {
            *b_out = b;
            return 0;
        }
    }
    return -1;
}

/* Is KV position j of request (prefix L) visible to the node whose mask is anc? */
static int position_visible(int64_t j, int64_t L, uint64_t anc) {
    if (j < L) return 1;
    return (int)((anc >> (j - L)) & 1u);
}

/* s_j for one query row and one pool slot (scale included). */
static double score(const uint16_t *ql, const uint16_t *qr, const uint16_t *row, double scale) {
    double dot_latent = 0.0, dot_rope = 0.0;
    for (int d = 0; d < ORACLE_D_LATENT; ++d)
        dot_latent += bf16_to_double(ql[d]) * bf16_to_double(row[d]);
    for (int e = 0; e < ORACLE_D_ROPE; ++e)
        dot_rope += bf16_to_double(qr[e]) * bf16_to_double(row[ORACLE_D_LATENT + e]);
    return scale * (dot_latent + dot_rope);
}

typedef struct {
    int32_t batch, num_heads;
    const int32_t *qo_indptr, *kv_indptr, *kv_indices;
    const uint64_t *anc;                 /* [sumT] */
    const uint16_t *q_latent, *q_rope;   /* [sumT, H, 512], [sumT, H, 64] */
    const uint16_t *kv_pool;             /* [pool_slots, 576] */
    int64_t pool_slots;
    double scale;
} oracle_problem;

/* Resolve a query (flattened row q = token*H + head) to its request data. */
static int resolve(const oracle_problem *p, int64_t q, const uint16_t **ql, const uint16_t **qr,
                   int64_t *kv_begin, int64_t *n_kv, int64_t *L, uint64_t *anc) {
    int64_t r = q / p->num_heads, h = q % p->num_heads;
    int32_t b;
    if (find_request(p->batch, p->qo_indptr, r, &b)) return -1;
    int64_t T = p->qo_indptr[b + 1] - p->qo_indptr[b];
    *kv_begin = p->kv_indptr[b];
    *n_kv = p->kv_indptr[b + 1] - p->kv_indptr[b];
    *L = *n_kv - T;
    if (*L < 0) return -1;
    *anc = p->anc[r];
    *ql = p->q_latent + (r * p->num_heads + h) * ORACLE_D_LATENT;
    *qr = p->q_rope + (r * p->num_heads + h) * ORACLE_D_ROPE;
    return 0;
}

/*
 * The definition, one query row at a time: gather the visible positions,
 * compute their scores, p_j = exp(s_j - max) / sum_k exp(s_k - max),
 * out = sum_j p_j v_j, lse = max + ln sum exp(s - max). The visible count is
 * the size of the visible set. Returns -1 on a bad row or slot.
 */
static int attend_row(const oracle_problem *p, int64_t q, double *out, double *lse, int32_t *count) {
    const uint16_t *ql, *qr;
    int64_t kv_begin, n_kv, L;
    uint64_t anc;
    if (resolve(p, q, &ql, &qr, &kv_begin, &n_kv, &L, &anc)) return -1;

    int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_kv > 0 ? n_kv : 1));
    double *s = (double *)malloc(sizeof(double) * (size_t)(n_kv > 0 ? n_kv : 1));
    if (!pos || !s) { free(pos); free(s); return -1; }
    int64_t nv = 0;
    for (int64_t j = 0; j < n_kv; ++j)
        if (position_visible(j, L, anc)) pos[nv++] = j;

    for (int64_t k = 0; k < nv; ++k) {
        int64_t slot = p->kv_indices[kv_begin + pos[k]];
        if (slot < 0 || slot >= p->pool_slots) { free(pos); free(s); return -1; }
        s[k] = score(ql, qr, p->kv_pool + slot * ORACLE_D_QK, p->scale);
    }
    double mx = -INFINITY;
    for (int64_t k = 0; k < nv; ++k) if (s[k] > mx) mx = s[k];
    double denom = 0.0;
    for (int64_t k = 0; k < nv; ++k) denom += exp(s[k] - mx);

    for (int d = 0; d < ORACLE_D_LATENT; ++d) out[d] = 0.0;
    for (int64_t k = 0; k < nv; ++k) {
        double pk = exp(s[k] - mx) / denom;
        const uint16_t *row = p->kv_pool + p->kv_indices[kv_begin + pos[k]] * ORACLE_D_QK;
        for (int d = 0; d < ORACLE_D_LATENT; ++d) out[d] += pk * bf16_to_double(row[d]);
    }
    *lse = (nv > 0) ? mx + log(denom) : -INFINITY;
    *count = (int32_t)nv;
    free(pos);
    free(s);
    return 0;
}

/*
 * Partial state over the visible positions j with key_lo <= j < key_hi:
 * m = max s_j, l = sum exp(s_j - m), O = sum exp(s_j - m) v_j.
 * With no such position: m = -inf, l = 0, O = 0.
 */
static int partial_row(const oracle_problem *p, int64_t q, int64_t key_lo, int64_t key_hi,
                       double *m_out, double *l_out, double *o_out) {
    const uint16_t *ql, *qr;
    int64_t kv_begin, n_kv, L;
    uint64_t anc;
    if (resolve(p, q, &ql, &qr, &kv_begin, &n_kv, &L, &anc)) return -1;
    if (key_lo < 0) key_lo = 0;
    if (key_hi > n_kv) key_hi = n_kv;

    double mx = -INFINITY;
    for (int64_t j = key_lo; j < key_hi; ++j) {
        if (!position_visible(j, L, anc)) continue;
        int64_t slot = p->kv_indices[kv_begin + j];
        if (slot < 0 || slot >= p->pool_slots) return -1;
        double sj = score(ql, qr, p->kv_pool + slot * ORACLE_D_QK, p->scale);
        if (sj > mx) mx = sj;
    }
    double l = 0.0;
    for (int d = 0; d < ORACLE_D_LATENT; ++d) o_out[d] = 0.0;
    if (mx != -INFINITY) {
        for (int64_t j = key_lo; j < key_hi; ++j) {
            if (!position_visible(j, L, anc)) continue;
            const uint16_t *row = p->kv_pool + p->kv_indices[kv_begin + j] * ORACLE_D_QK;
            double e = exp(score(ql, qr, row, p->scale) - mx);
            l += e;
            for (int d = 0; d < ORACLE_D_LATENT; ++d) o_out[d] += e * bf16_to_double(row[d]);
        }
    }
    *m_out = mx;
    *l_out = l;
    return 0;
}

/*
 * Full verify output for a list of query rows (each q = token*H + head);
 * rows == NULL means every row 0..sumT*H-1 in order. out: [n_rows, 512],
 * lse: [n_rows], visible: [n_rows]. Any of the outputs may be NULL.
 * threads > 0 caps the OpenMP team (when built with OpenMP).
 */
int oracle_verify_rows(int32_t batch, int32_t num_heads,
                       const int32_t *qo_indptr, const int32_t *kv_indptr, const int32_t *kv_indices,
                       const uint64_t *anc, const uint16_t *q_latent, const uint16_t *q_rope,
                       const uint16_t *kv_pool, int64_t pool_slots, double scale,
                       const int64_t *rows, int64_t n_rows,
                       double *out, double *lse, int32_t *visible, int32_t threads) {
    oracle_problem p = {batch, num_heads, qo_indptr, kv_indptr, kv_indices, anc,
                        q_latent, q_rope, kv_pool, pool_slots, scale};
    int failed = 0;
    (void)threads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : omp_get_max_threads()) reduction(| : failed)
#endif
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t q = rows ? rows[i] : i;
        double o[ORACLE_D_LATENT], ls;
        int32_t cnt;
        if (attend_row(&p, q, o, &ls, &cnt)) { failed |= 1; continue; }
        if (out) memcpy(out + i * ORACLE_D_LATENT, o, sizeof o);
        if (lse) lse[i] = ls;
        if (visible) visible[i] = cnt;
    }
    return failed ? -1 : 0;
}

/* Partial states (m, l, O) of a list of query rows over KV positions [key_lo, key_hi). */
int oracle_partial_rows(int32_t batch, int32_t num_heads,
                        const int32_t *qo_indptr, const int32_t *kv_indptr, const int32_t *kv_indices,
                        const uint64_t *anc, const uint16_t *q_latent, const uint16_t *q_rope,
                        const uint16_t *kv_pool, int64_t pool_slots, double scale,
                        const int64_t *rows, int64_t n_rows, int64_t key_lo, int64_t key_hi,
                        double *m, double *l, double *o) {
    oracle_problem p = {batch, num_heads, qo_indptr, kv_indptr, kv_indices, anc,
                        q_latent, q_rope, kv_pool, pool_slots, scale};
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t q = rows ? rows[i] : i;
        if (partial_row(&p, q, key_lo, key_hi, m + i, l + i, o + i * ORACLE_D_LATENT)) return -1;
    }
    return 0;
}

/*
 * Merge n_states partial states per row (arrays [n_states, n_rows(, 512)])
 * into the normalised output and lse with the formula in the header comment.
 * A row whose states all have l = 0 gets out = 0 and lse = -inf.
 */
int oracle_merge_states(int32_t n_states, int64_t n_rows, const double *m, const double *l,
                        const double *o, double *out, double *lse) {
    for (int64_t r = 0; r < n_rows; ++r) {
        double mstar = -INFINITY;
        for (int32_t s = 0; s < n_states; ++s) {
            double ms = m[(int64_t)s * n_rows + r];
            if (l[(int64_t)s * n_rows + r] > 0.0 && ms > mstar) mstar = ms;
        }
        double lstar = 0.0;
        double acc[ORACLE_D_LATENT];
        for (int d = 0; d < ORACLE_D_LATENT; ++d) acc[d] = 0.0;
        if (mstar != -INFINITY) {
            for (int32_t s = 0; s < n_states; ++s) {
                int64_t i = (int64_t)s * n_rows + r;
                if (!(l[i] > 0.0)) continue;
                double w = exp(m[i] - mstar);
                lstar += l[i] * w;
                for (int d = 0; d < ORACLE_D_LATENT; ++d) acc[d] += o[i * ORACLE_D_LATENT + d] * w;
            }
        }
        for (int d = 0; d < ORACLE_D_LATENT; ++d)
            out[r * ORACLE_D_LATENT + d] = (lstar > 0.0) ? acc[d] / lstar : 0.0;
        lse[r] = (lstar > 0.0) ? mstar + log(lstar) : -INFINITY;
    }
    return 0;
}
