/*
 * A plain C99 consumer of include/verify_attn.h: it must compile with
 * -std=c99 -pedantic -Werror, link against the library, and run its
 * host-only calls (planning with an explicit SM count, argument checks,
 * the host tree-mask helper, error strings) without a GPU.
 * Exit status 0 when every check holds; the failing check is printed.
 */
#include <stdio.h>
#include <string.h>

#include "verify_attn.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(void) {
    verify_attn_params q;
    verify_attn_plan_t plan;
    size_t ws = 0;
    int32_t parents[4] = {-1, 0, 0, 1};
    uint64_t anc[4];
    verify_attn_defrag_args d;
    verify_attn_merge_args m;
    verify_attn_merge_stacked_args st;

    memset(&q, 0, sizeof q);
    q.max_batch = 1;
    q.num_heads = 64;
    q.max_tree = 64;
    q.d_latent = VERIFY_ATTN_D_LATENT;
    q.d_rope = VERIFY_ATTN_D_ROPE;
    q.num_sms = 148;
    q.max_kv_per_req = 65600;
    q.max_total_kv = 65600;
    q.pool_slots = 262144;
    q.sm_scale = 0.07216878f;
    CHECK(verify_attn_plan(&q, &plan, &ws) == VERIFY_ATTN_OK);
    CHECK(plan.version == VERIFY_ATTN_PLAN_VERSION);
    CHECK(plan.num_clusters == 74);
    CHECK((int64_t)ws == plan.ws_bytes && ws > 0);

    q.max_tree = 65;
    CHECK(verify_attn_plan(&q, &plan, &ws) == VERIFY_ATTN_UNSUPPORTED);
    CHECK(verify_attn_plan(NULL, &plan, &ws) == VERIFY_ATTN_EINVAL);

    CHECK(verify_attn_build_tree_mask(parents, 4, anc) == VERIFY_ATTN_OK);
    CHECK(anc[0] == 0x1u && anc[1] == 0x3u && anc[2] == 0x5u && anc[3] == 0xbu);
    parents[2] = 3;   /* a parent after its child */
    CHECK(verify_attn_build_tree_mask(parents, 4, anc) == VERIFY_ATTN_EINVAL);

    memset(&d, 0, sizeof d);
    CHECK(verify_attn_defrag(&d, NULL) == VERIFY_ATTN_EINVAL);
    memset(&m, 0, sizeof m);
    CHECK(verify_attn_merge_states(&m, NULL) == VERIFY_ATTN_EINVAL);
    memset(&st, 0, sizeof st);
    CHECK(verify_attn_merge_stacked(&st, NULL) == VERIFY_ATTN_EINVAL);

    CHECK(strlen(verify_attn_strerror(VERIFY_ATTN_DEVICE_TIMEOUT)) > 0);
    printf("c abi consumer ok: %lld workspace bytes, %d pairs\n", (long long)ws, plan.num_clusters);
    return 0;
}
