/* Plain-C client of the library's C ABI (no Python, no PyTorch): allocates device
 * buffers with the CUDA runtime, fills q/k/v with a fixed pattern, runs
 * attn_prefix_fwd and attn_prefix_fwd_split + attn_lse_combine, and checks the result
 * against a small double-precision softmax written here.  Exit status 0 = pass.
 * Shapes: B=2, H=1, Tq=5, Tk=200, D=64, kv_len = {200, 37}; key slots at or beyond
 * kv_len hold NaN. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>

#include "attn_prefix.h"

enum { B = 2, H = 1, TQ = 5, TK = 200, D = 64 };

static uint16_t to_bf16(float f) {   /* round to nearest even */
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

#define CHECK(x)                                                              \
    do {                                                                      \
        if (!(x)) {                                                           \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #x);   \
            return 1;                                                         \
        }                                                                     \
    } while (0)

int main(void) {
    const int32_t kv_len[B] = {200, 37};
    const size_t nq = (size_t)B * H * TQ * D, nk = (size_t)B * H * TK * D;
    uint16_t *q = malloc(nq * 2), *k = malloc(nk * 2), *v = malloc(nk * 2), *o = malloc(nq * 2);
    float* lse = malloc(sizeof(float) * B * H * TQ);
    CHECK(q && k && v && o && lse);
    for (size_t i = 0; i < nq; ++i) q[i] = to_bf16((float)sin(0.37 * (double)i));
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < TK; ++j)
            for (int d = 0; d < D; ++d) {
                size_t i = ((size_t)b * TK + j) * D + d;
                float kv = (float)cos(0.11 * (double)i), vv = (float)sin(0.23 * (double)i + 1.0);
                k[i] = j < kv_len[b] ? to_bf16(kv) : 0x7fc0; /* NaN padding */
                v[i] = j < kv_len[b] ? to_bf16(vv) : 0x7fc0;
            }
    void *dq, *dk, *dv, *dout, *dkv;
    float *dlse, *dpo, *dpl;
    const int C = 3;
    CHECK(cudaMalloc(&dq, nq * 2) == cudaSuccess && cudaMalloc(&dk, nk * 2) == cudaSuccess &&
          cudaMalloc(&dv, nk * 2) == cudaSuccess && cudaMalloc(&dout, nq * 2) == cudaSuccess &&
          cudaMalloc(&dkv, sizeof kv_len) == cudaSuccess && cudaMalloc((void**)&dlse, sizeof(float) * B * H * TQ) == cudaSuccess);
    CHECK(cudaMalloc((void**)&dpo, sizeof(float) * C * nq) == cudaSuccess &&
          cudaMalloc((void**)&dpl, sizeof(float) * C * B * H * TQ) == cudaSuccess);
    CHECK(cudaMemcpy(dq, q, nq * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dk, k, nk * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dv, v, nk * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dkv, kv_len, sizeof kv_len, cudaMemcpyHostToDevice) == cudaSuccess);
    const float scale = 0.125f;

    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 0) {
            CHECK(attn_prefix_fwd(dq, dk, dv, (const int32_t*)dkv, dout, dlse, B, H, TQ, TK, D, scale, 0) == ATTN_OK);
        } else {
            CHECK(attn_prefix_fwd_split(dq, dk, dv, (const int32_t*)dkv, C, dpo, dpl, B, H, TQ, TK, D, scale, 0) ==
                  ATTN_OK);
            CHECK(attn_lse_combine(dpo, dpl, C, dout, dlse, B, H, TQ, D, 0) == ATTN_OK);
        }
        CHECK(attn_get_device_status(0) == ATTN_OK);
        CHECK(cudaMemcpy(o, dout, nq * 2, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(lse, dlse, sizeof(float) * B * H * TQ, cudaMemcpyDeviceToHost) == cudaSuccess);
        double worst = 0.0;
        for (int b = 0; b < B; ++b)
            for (int i = 0; i < TQ; ++i) {
                const uint16_t* qr = q + ((size_t)b * TQ + i) * D;
                double s[TK], m = -INFINITY, l = 0.0, ref[D];
                for (int j = 0; j < kv_len[b]; ++j) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += from_bf16(qr[d]) * from_bf16(k[((size_t)b * TK + j) * D + d]);
                    s[j] = scale * dot;
                    if (s[j] > m) m = s[j];
                }
                for (int d = 0; d < D; ++d) ref[d] = 0.0;
                for (int j = 0; j < kv_len[b]; ++j) {
                    const double w = exp(s[j] - m);
                    l += w;
                    for (int d = 0; d < D; ++d) ref[d] += w * from_bf16(v[((size_t)b * TK + j) * D + d]);
                }
                for (int d = 0; d < D; ++d) {
                    const double got = from_bf16(o[((size_t)b * TQ + i) * D + d]), want = ref[d] / l;
                    const double err = fabs(got - want);
                    CHECK(err <= 1e-2 + 1e-2 * fabs(want));
                    if (err > worst) worst = err;
                }
                CHECK(fabs((double)lse[b * TQ + i] - (m + log(l))) <= 1e-3);
            }
        printf("%s: max |out - ref| %.3g\n", pass == 0 ? "single pass" : "split + combine", worst);
    }
    printf("%s\n", attn_status_string(ATTN_ERR_TIMEOUT));
    cudaFree(dq); cudaFree(dk); cudaFree(dv); cudaFree(dout); cudaFree(dkv); cudaFree(dlse); cudaFree(dpo); cudaFree(dpl);
    free(q); free(k); free(v); free(o); free(lse);
    return 0;
}
