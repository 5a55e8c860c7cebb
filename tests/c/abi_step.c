/* The five calls of include/lmhead.h from plain C (no Python, no torch), on
 * one small integer-valued problem: M = 40 tokens, K = 256, V = 1000.
 * Device memory comes from the CUDA runtime; every input is made on the
 * host.  Checks, each with a definition written out here:
 *   - logits equal the integer dot products word for word (BF16 integers in
 *     [-8, 8], K * 64 < 2^24, so the FP32 sums are exact);
 *   - per valid row, loss >= 0 and m is the row maximum; ignored rows are 0;
 *   - every valid row of the FP32 gradient sums to ~0 and an ignored row is 0;
 *   - dX and dW of integer "dlogits" equal their integer sums word for word.
 * Prints "abi step ok" and exits 0, or names the first failed check and
 * exits 1. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "lmhead.h"

/* The few CUDA runtime entry points used, declared here so that the program
 * needs no CUDA header. */
typedef int cudaError_t;
extern cudaError_t cudaMalloc(void **p, size_t n);
extern cudaError_t cudaFree(void *p);
extern cudaError_t cudaMemcpy(void *dst, const void *src, size_t n, int kind);
extern cudaError_t cudaMemset(void *p, int v, size_t n);
extern cudaError_t cudaDeviceSynchronize(void);
enum { H2D = 1, D2H = 2 };

enum { M = 40, K = 256, V = 1000 };

static uint16_t bf16_of_int(int v) /* small integers are exact in BF16 */
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static uint32_t rng = 12345u;
static int rand_int(int lo, int hi) /* inclusive */
{
    rng = rng * 1664525u + 1013904223u;
    return lo + (int)((rng >> 8) % (uint32_t)(hi - lo + 1));
}

#define CHECK(c, msg)                                   \
    do {                                                \
        if (!(c)) {                                     \
            fprintf(stderr, "check failed: %s\n", msg); \
            return 1;                                   \
        }                                               \
    } while (0)
#define OK(call) CHECK((call) == 0, #call)

int main(void)
{
    static int xi[M][K], wi[V][K], dli[M][V];
    static uint16_t xh[M][K], wh[V][K], dlh[M][V];
    static float logits[M][V], stats[M][4], grad[M][V], dx[M][K], dw[V][K];
    static int64_t target[M];
    for (int i = 0; i < M; ++i)
        for (int k = 0; k < K; ++k) xh[i][k] = bf16_of_int(xi[i][k] = rand_int(-8, 8));
    for (int v = 0; v < V; ++v)
        for (int k = 0; k < K; ++k) wh[v][k] = bf16_of_int(wi[v][k] = rand_int(-8, 8));
    for (int i = 0; i < M; ++i)
        for (int v = 0; v < V; ++v) dlh[i][v] = bf16_of_int(dli[i][v] = rand_int(-8, 8));
    for (int i = 0; i < M; ++i) target[i] = (i % 7 == 3) ? -100 : rand_int(0, V - 1);

    void *dX, *dW, *dL, *dS, *dT, *dG, *dDL, *dGrad, *dDx, *dDw, *dStatus;
    OK(cudaMalloc(&dX, sizeof xh));
    OK(cudaMalloc(&dW, sizeof wh));
    OK(cudaMalloc(&dL, sizeof logits));
    OK(cudaMalloc(&dS, sizeof stats));
    OK(cudaMalloc(&dT, sizeof target));
    OK(cudaMalloc(&dG, sizeof(float)));
    OK(cudaMalloc(&dDL, sizeof dlh));
    OK(cudaMalloc(&dGrad, sizeof grad));
    OK(cudaMalloc(&dDx, sizeof dx));
    OK(cudaMalloc(&dDw, sizeof dw));
    OK(cudaMalloc(&dStatus, sizeof(int32_t)));
    const float g = 1.0f;
    OK(cudaMemcpy(dX, xh, sizeof xh, H2D));
    OK(cudaMemcpy(dW, wh, sizeof wh, H2D));
    OK(cudaMemcpy(dT, target, sizeof target, H2D));
    OK(cudaMemcpy(dG, &g, sizeof g, H2D));
    OK(cudaMemcpy(dDL, dlh, sizeof dlh, H2D));
    OK(cudaMemset(dStatus, 0, sizeof(int32_t)));

    int32_t *st = (int32_t *)dStatus;
    CHECK(lmhead_fwd(dX, dW, dL, LMH_F32, M, K, V, st, NULL) == LMH_OK, "lmhead_fwd");
    CHECK(ce_fwd((const float *)dL, (const int64_t *)dT, (float *)dS, M, V, -100, st, NULL) == LMH_OK,
          "ce_fwd");
    CHECK(ce_bwd((const float *)dL, (const int64_t *)dT, (const float *)dS, (const float *)dG, 0, dGrad,
                 LMH_F32, M, V, -100, st, NULL) == LMH_OK,
          "ce_bwd");
    CHECK(lmhead_bwd_dx(dDL, dW, dDx, LMH_F32, M, K, V, st, NULL) == LMH_OK, "lmhead_bwd_dx");
    CHECK(lmhead_bwd_dw(dDL, dX, dDw, LMH_F32, M, K, V, st, NULL) == LMH_OK, "lmhead_bwd_dw");
    CHECK(lmhead_fwd(dX, dW, dL, LMH_F16, M, K, V, st, NULL) == LMH_ERR_UNSUPPORTED, "fp16 rejected");
    OK(cudaDeviceSynchronize());
    int32_t status = -1;
    OK(cudaMemcpy(&status, dStatus, sizeof status, D2H));
    CHECK(status == 0, "device status word");
    OK(cudaMemcpy(logits, dL, sizeof logits, D2H));
    OK(cudaMemcpy(stats, dS, sizeof stats, D2H));
    OK(cudaMemcpy(grad, dGrad, sizeof grad, D2H));
    OK(cudaMemcpy(dx, dDx, sizeof dx, D2H));
    OK(cudaMemcpy(dw, dDw, sizeof dw, D2H));

    for (int i = 0; i < M; ++i)
        for (int v = 0; v < V; ++v) {
            long s = 0;
            for (int k = 0; k < K; ++k) s += (long)xi[i][k] * wi[v][k];
            CHECK(logits[i][v] == (float)s, "logits are the exact integer sums");
        }
    for (int i = 0; i < M; ++i) {
        double rowsum = 0.0;
        for (int v = 0; v < V; ++v) rowsum += grad[i][v];
        if (target[i] == -100) {
            CHECK(stats[i][0] == 0.f && stats[i][1] == 0.f && stats[i][3] == 0.f, "ignored stats");
            for (int v = 0; v < V; ++v) CHECK(grad[i][v] == 0.f, "ignored gradient row");
            continue;
        }
        float mx = logits[i][0];
        for (int v = 1; v < V; ++v) mx = logits[i][v] > mx ? logits[i][v] : mx;
        CHECK(stats[i][0] == mx, "m is the row maximum");
        CHECK(stats[i][2] == logits[i][target[i]], "x_y is the target logit");
        CHECK(stats[i][3] >= 0.f && stats[i][1] >= 1.f, "loss >= 0, d >= 1");
        CHECK(fabs(rowsum) < V * 1e-6, "gradient row sums to zero");
    }
    for (int i = 0; i < M; ++i)
        for (int k = 0; k < K; ++k) {
            long s = 0;
            for (int v = 0; v < V; ++v) s += (long)dli[i][v] * wi[v][k];
            CHECK(dx[i][k] == (float)s, "dX is the exact integer sum");
        }
    for (int v = 0; v < V; ++v)
        for (int k = 0; k < K; ++k) {
            long s = 0;
            for (int i = 0; i < M; ++i) s += (long)dli[i][v] * xi[i][k];
            CHECK(dw[v][k] == (float)s, "dW is the exact integer sum");
        }
    cudaFree(dX); cudaFree(dW); cudaFree(dL); cudaFree(dS); cudaFree(dT); cudaFree(dG);
    cudaFree(dDL); cudaFree(dGrad); cudaFree(dDx); cudaFree(dDw); cudaFree(dStatus);
    printf("abi step ok\n");
    return 0;
}
