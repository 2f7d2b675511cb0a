/*
 * A plain C99 caller of the dllm_qgemm C ABI.  It includes only the public header and
 * links only the shared library, and it calls the entry points that need no device:
 * sizes, status strings, the GEMM work split, and argument rejection before any launch.
 * It prints one "name value" line per result for the test that builds and runs it.
 */
#include <stdio.h>
#include <string.h>

#include "dllm_qgemm.h"

int main(void)
{
    size_t wb = 0, qb = 0, sb = 0, ub = 0;
    int rc = dllm_repacked_bytes(DLLM_Q4_K, 4096, 4096, &wb);
    printf("repacked_q4k_rc %d\nrepacked_q4k_bytes %zu\n", rc, wb);
    rc = dllm_repacked_bytes(DLLM_Q6_K, 4096, 12288, &wb);
    printf("repacked_q6k_rc %d\nrepacked_q6k_bytes %zu\n", rc, wb);
    rc = dllm_act_bytes(160, 4096, &qb, &sb, &ub);
    printf("act_rc %d\nact_q %zu\nact_scale %zu\nact_sums %zu\n", rc, qb, sb, ub);
    printf("act_bad_k %d\n", dllm_act_bytes(160, 300, &qb, &sb, &ub));
    printf("repacked_bad_n %d\n", dllm_repacked_bytes(DLLM_Q4_K, 100, 4096, &wb));

    int64_t plan[8];
    rc = dllm_debug_plan(192, 4096, 128, 0, 148, plan);
    printf("plan_rc %d\nplan_kc %lld\nplan_full_tiles %lld\nplan_tail_k %lld\nplan_tail_big %lld\n", rc,
           (long long)plan[0], (long long)plan[1], (long long)plan[2], (long long)plan[3]);
    printf("plan_bad %d\n", dllm_debug_plan(0, 4096, 128, 0, 148, plan));

    /* rejected on the host, before any device call: a null activation pointer */
    printf("quantize_null %d\n", dllm_quantize_act(NULL, 4, 256, 256, NULL, NULL, NULL, NULL));
    printf("rmsnorm_eps0 %d\n",
           dllm_rmsnorm_quantize((const float*)0x10000, 4, 256, 256, (const float*)0x10000, 0.0f, NULL, 0,
                                 (int8_t*)0x10000, (float*)0x10000, (uint8_t*)0x10000, NULL));

    /* attention: argument errors and the empty query set, all decided on the host */
    {
        const void* d = (const void*)0x10000;
        float* o = (float*)0x10000;
        printf("attn_dh64 %d\n", dllm_attention(d, d, d, 4, 4, 2, 2, 64, o, NULL));
        printf("attn_group %d\n", dllm_attention(d, d, d, 4, 4, 3, 2, 128, o, NULL));
        printf("attn_no_keys %d\n", dllm_attention(d, d, d, 4, 0, 2, 2, 128, o, NULL));
        printf("attn_null %d\n", dllm_attention(NULL, d, d, 4, 4, 2, 2, 128, o, NULL));
        printf("attn_align %d\n", dllm_attention((const char*)d + 2, d, d, 4, 4, 2, 2, 128, o, NULL));
        printf("attn_empty %d\n", dllm_attention(NULL, NULL, NULL, 0, 0, 2, 2, 128, NULL, NULL));
    }

    const char* s = dllm_status_string(DLLM_ERR_ROW_RANGE);
    printf("status_row_range_nonempty %d\n", s != NULL && strlen(s) > 0);
    return 0;
}
