/*
 * step_from_c.c -- drives libliteattn.so through include/liteattn.h alone,
 * from plain C (no Python, no PyTorch): the boundary's own contract.
 *
 *   step_from_c checks               argument checks that need no GPU
 *   step_from_c run IN OUT MASK      one step of a plan (B=1, H=2, N=1000,
 *                                    d=Br=Bc=64, tau=ln 1e-2) on q, k, v read
 *                                    from IN (3 x B*H*N*d bf16, [B][H][N][d]);
 *                                    writes o to OUT and the mask bits to MASK
 *
 * Exit status 0 on success; messages on stderr otherwise.  Device memory comes
 * from the CUDA runtime (cudaMalloc), which the program links as well.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "liteattn.h"

#define CHECK(cond, msg)                                         \
    do {                                                         \
        if (!(cond)) {                                           \
            fprintf(stderr, "step_from_c: %s (line %d)\n", msg, __LINE__); \
            return 1;                                            \
        }                                                        \
    } while (0)

static int checks(void) {
    float taus[2] = {-1.0f, -INFINITY};
    lite_attn_plan_t plan = NULL;
    CHECK(lite_attn_plan_create(NULL, 1, 1, 64, 64, 64, 64, taus, 1) == LITE_ERR_INVALID_ARG, "null out");
    CHECK(lite_attn_plan_create(&plan, 0, 1, 64, 64, 64, 64, taus, 1) == LITE_ERR_INVALID_ARG, "B = 0");
    CHECK(plan == NULL, "plan set on failure");
    float pos = 0.5f;
    CHECK(lite_attn_plan_create(&plan, 1, 1, 64, 64, 64, 64, &pos, 1) == LITE_ERR_INVALID_ARG, "tau > 0");
    CHECK(lite_attn_plan_create(&plan, 1, 1, 64, 96, 96, 96, taus, 1) == LITE_ERR_UNSUPPORTED, "d = 96");
    CHECK(lite_attn_plan_create_ex(&plan, 1, 1, 64, 64, 64, 64, taus, 1, 5, 0) == LITE_ERR_INVALID_ARG, "layout");
    CHECK(lite_attn_plan_create_ex(&plan, 1, 3, 64, 64, 64, 64, taus, 1, LITE_LAYOUT_BNHD, 2) == LITE_ERR_INVALID_ARG,
          "heads_total < H");
    CHECK(lite_attn_plan_destroy(NULL) == LITE_OK, "destroy NULL");
    CHECK(lite_attn_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == LITE_ERR_INVALID_ARG, "step NULL");
    CHECK(strcmp(lite_attn_error_string(LITE_ERR_PLAN_MISMATCH), "mask does not belong to this plan") == 0,
          "error string");
    CHECK(lite_attn_error_string(-1234) != NULL, "unknown code string");
    CHECK(lite_attn_launch_count() >= 0, "launch count");
    return 0;
}

static int run(const char *in, const char *out, const char *mask_path) {
    const int B = 1, H = 2, N = 1000, d = 64;
    const size_t n = (size_t)B * H * N * d, bytes = n * 2;
    uint16_t *host = malloc(3 * bytes);
    CHECK(host, "host alloc");
    FILE *f = fopen(in, "rb");
    CHECK(f && fread(host, 1, 3 * bytes, f) == 3 * bytes, "read inputs");
    fclose(f);
    float tau = logf(1e-2f);
    lite_attn_plan_t plan;
    lite_attn_mask_t mask;
    CHECK(lite_attn_plan_create(&plan, B, H, N, d, d, d, &tau, 1) == LITE_OK, "plan create");
    CHECK(lite_attn_mask_create(plan, &mask) == LITE_OK, "mask create");
    int Tq, Tk, W, G;
    CHECK(lite_attn_plan_info(plan, &Tq, &Tk, &W, &G) == LITE_OK, "plan info");
    void *dq, *dk, *dv, *dout;
    CHECK(cudaMalloc(&dq, bytes) == 0 && cudaMalloc(&dk, bytes) == 0 && cudaMalloc(&dv, bytes) == 0 &&
              cudaMalloc(&dout, bytes) == 0, "cudaMalloc");
    CHECK(cudaMemcpy(dq, host, bytes, cudaMemcpyHostToDevice) == 0 &&
              cudaMemcpy(dk, host + n, bytes, cudaMemcpyHostToDevice) == 0 &&
              cudaMemcpy(dv, host + 2 * n, bytes, cudaMemcpyHostToDevice) == 0, "copy in");
    /* o must not alias q: rejected before anything runs */
    CHECK(lite_attn_step(plan, dq, dk, dv, dq, mask, mask, 0, NULL) == LITE_ERR_INVALID_ARG, "aliasing o");
    CHECK(lite_attn_step(plan, dq, dk, dv, dout, mask, mask, 1, NULL) == LITE_ERR_INVALID_ARG, "step out of range");
    CHECK(lite_attn_step(plan, dq, dk, dv, dout, mask, mask, 0, NULL) == LITE_OK, "step");
    lite_attn_stats_t st;
    CHECK(lite_attn_stats(plan, mask, &st) == LITE_OK && st.device_status == LITE_OK, "stats");
    CHECK(st.tiles_total == (int64_t)B * H * Tq * Tk && st.live_in == st.tiles_total, "stats counts");
    CHECK(cudaMemcpy(host, dout, bytes, cudaMemcpyDeviceToHost) == 0, "copy out");
    uint32_t *bits = malloc((size_t)B * H * Tq * W * 4);
    CHECK(bits && lite_attn_mask_export(mask, bits, NULL) == LITE_OK, "mask export");
    f = fopen(out, "wb");
    CHECK(f && fwrite(host, 1, bytes, f) == bytes, "write output");
    fclose(f);
    f = fopen(mask_path, "wb");
    CHECK(f && fwrite(bits, 4, (size_t)B * H * Tq * W, f) == (size_t)B * H * Tq * W, "write mask");
    fclose(f);
    printf("live_out %lld of %lld\n", (long long)st.live_out, (long long)st.tiles_total);
    CHECK(lite_attn_mask_destroy(mask) == LITE_OK && lite_attn_plan_destroy(plan) == LITE_OK, "destroy");
    cudaFree(dq), cudaFree(dk), cudaFree(dv), cudaFree(dout);
    free(bits);
    free(host);
    return 0;
}

int main(int argc, char **argv) {
    if (argc == 2 && strcmp(argv[1], "checks") == 0) return checks();
    if (argc == 5 && strcmp(argv[1], "run") == 0) return run(argv[2], argv[3], argv[4]);
    fprintf(stderr, "usage: step_from_c checks | run IN OUT MASK\n");
    return 2;
}
