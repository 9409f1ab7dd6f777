/* The device path of the C-ABI from plain C99, with no Python and no torch:
 * plan the tiny bucket, let the library allocate it, fill it through the
 * exported bucket pointers, run the step resident and from host buffers,
 * and check the first step's closed form (p1 = p0 (1 - lr wd) - lr g/(|g| + eps'),
 * so about p0 - lr for |g| much larger than eps).  Built and run by
 * tests/test_c_abi.py on a GPU. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "dbuf.h"

static float bf16_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int main(void) {
    dbuf_tensor_desc t[3] = {{512, 256, 16, 0}, {512, 1, 512, 0}, {256, 1, 256, 0}};
    dbuf_plan_t* plan = NULL;
    dbuf_t* db = NULL;
    if (dbuf_plan(t, 3, 4, 16, 0, &plan) != DBUF_OK) return 1;
    if (dbuf_create(plan, NULL, 0, NULL, &db) != DBUF_OK) {
        printf("create: %s\n", dbuf_last_error());
        return 2;
    }
    void *master = NULL, *grad = NULL, *param = NULL;
    int64_t S = 0;
    if (dbuf_bucket(db, DBUF_MASTER_F32, &master, &S) != DBUF_OK) return 3;
    if (dbuf_bucket(db, DBUF_GRAD_BF16, &grad, NULL) != DBUF_OK) return 3;
    if (dbuf_bucket(db, DBUF_PARAM_BF16, &param, NULL) != DBUF_OK) return 3;
    float* p0 = (float*)malloc((size_t)S * 4);
    uint16_t* g = (uint16_t*)malloc((size_t)S * 2);
    uint16_t* pb = (uint16_t*)malloc((size_t)S * 2);
    float* p1 = (float*)malloc((size_t)S * 4);
    if (!p0 || !g || !pb || !p1) return 4;
    for (int64_t i = 0; i < S; ++i) {
        p0[i] = 0.01f;
        g[i] = (i & 1) ? 0x3A83u : 0xBA83u; /* +-0.001 in bf16 */
    }
    if (cudaMemcpy(master, p0, (size_t)S * 4, cudaMemcpyHostToDevice) != cudaSuccess) return 5;
    if (cudaMemcpy(grad, g, (size_t)S * 2, cudaMemcpyHostToDevice) != cudaSuccess) return 5;
    const dbuf_adam_hparams hp = {1e-3f, 0.9f, 0.999f, 1e-8f, 0.01f, 1};
    if (dbuf_adam8_step(db, &hp, 1.0f, NULL) != DBUF_OK) return 6;
    if (cudaDeviceSynchronize() != cudaSuccess) return 7;
    if (cudaMemcpy(p1, master, (size_t)S * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return 8;
    int64_t off[3];
    dbuf_plan_info(plan, NULL, NULL, NULL, NULL, off);
    double worst = 0.0;
    for (int k = 0; k < 3; ++k) {
        const int64_t n = t[k].rows * t[k].cols;
        for (int64_t i = 0; i < n; ++i) {
            const int64_t e = off[k] + i;
            const double sign = (e & 1) ? 1.0 : -1.0;
            const double want = 0.01 * (1.0 - 1e-5) - 1e-3 * sign;
            const double err = fabs((double)p1[e] - want);
            if (err > worst) worst = err;
        }
    }
    /* host-buffer path: same gradients again, params come back to the host */
    const dbuf_adam_hparams hp2 = {1e-3f, 0.9f, 0.999f, 1e-8f, 0.01f, 2};
    if (dbuf_adam8_step_host(db, &hp2, 1.0f, g, pb, NULL) != DBUF_OK) return 9;
    if (cudaDeviceSynchronize() != cudaSuccess) return 10;
    int32_t code = -1;
    if (dbuf_get_device_status(db, &code, NULL) != DBUF_OK) return 11;
    const float seen = bf16_to_float(pb[off[0] + 1]);
    printf("first_step_worst_abs_err=%.3e second_step_param=%.6f status=%d\n", worst, seen, (int)code);
    dbuf_destroy(db);
    dbuf_plan_free(plan);
    free(p0);
    free(g);
    free(pb);
    free(p1);
    return (worst < 1e-6 && code == 0) ? 0 : 12;
}
