/*
 * A plain C (C99) consumer of include/q4k.h linked against libq4k_b200.so.
 * It makes only calls the library answers on the host (sizes, status strings,
 * launch plans, argument refusals), so it runs without a GPU. Exit status 0
 * means every check passed; otherwise it prints the failing check.
 */
#include <stdio.h>
#include <string.h>

#include "q4k.h"

static int failures = 0;

#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                                 \
        }                                                               \
    } while (0)

int main(void)
{
    /* the Q4_K size rule: n * (k/256) * 144 */
    CHECK(q4k_weight_bytes(128256, 4096) == (size_t)295501824);
    CHECK(q4k_weight_bytes(4, 255) == 0);
    CHECK(q4k_weight_bytes(0, 256) == 0);

    CHECK(strcmp(q4k_status_string(Q4K_OK), "ok") == 0);
    CHECK(strcmp(q4k_status_string(12345), "unknown status") == 0);

    /* host-only launch plans */
    q4k_gemv_plan plan;
    memset(&plan, 0, sizeof(plan));
    CHECK(q4k_gemv_plan_for(1, 4096, 4096, 148, &plan) == Q4K_OK);
    CHECK(plan.kernel == Q4K_KERNEL_STREAM && plan.grid >= 148 && plan.launches == 1);
    CHECK(q4k_gemv_plan_for(1, 128256, 4096, 148, &plan) == Q4K_OK && plan.kernel == Q4K_KERNEL_I8 &&
          plan.grid == 148 && plan.units == 1002 * 16 && plan.units_per_cta_max == 7 * 16 &&
          plan.launches == 1);
    CHECK(q4k_gemv_plan_for(1, 128256, 20480, 148, &plan) == Q4K_OK && plan.kernel == Q4K_KERNEL_STREAM &&
          plan.slices == 2);
    CHECK(q4k_gemv_plan_for(Q4K_MAX_M + 1, 4096, 4096, 148, &plan) == Q4K_ERR_UNSUPPORTED_M);
    CHECK(q4k_gemv_plan_for(1, 4096, 4000, 148, &plan) == Q4K_ERR_SHAPE);
    CHECK(q4k_gemv_swiglu_plan_for(1, 14336, 4096, 148, &plan) == Q4K_OK && plan.cluster == 1);
    CHECK(q4k_gemv_plan_for(1, 4096, 4096, 148, NULL) == Q4K_ERR_NULL);

    /* refusals before any CUDA call */
    CHECK(q4k_gemv(NULL, NULL, NULL, 1, 4, 256, NULL) == Q4K_ERR_NULL);
    CHECK(q4k_gemv_swiglu(NULL, NULL, NULL, NULL, 1, 4, 256, NULL) == Q4K_ERR_NULL);
    CHECK(q4k_dequant_f32(NULL, NULL, 4, 256, NULL) == Q4K_ERR_NULL);
    CHECK(q4k_embed_lookup_f32(NULL, 144 * 4, 4, 256, 256, 4, 1.0f, NULL, NULL) == Q4K_ERR_RANGE);
    CHECK(q4k_embed_lookup_f32(NULL, 144 * 4, 4, 512, 256, 0, 1.0f, NULL, NULL) == Q4K_ERR_SHAPE);
    CHECK(q4k_embed_gather_f32(NULL, 0, 1, 256, NULL, 1, 1.0f, NULL, NULL) == Q4K_ERR_NULL);
    CHECK(q4k_device_fault_flags(NULL) == Q4K_ERR_NULL);
    CHECK(q4k_last_cuda_error() == 0);

    if (failures == 0)
        printf("c abi check ok\n");
    return failures == 0 ? 0 : 1;
}
