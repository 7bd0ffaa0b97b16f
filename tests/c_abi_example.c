/*
 * c_abi_example.c -- the library driven from plain C through include/hsa.h,
 * the way a non-Python host program uses it: the caller allocates every
 * device buffer (inputs, outputs, a zero-filled workspace), calls
 * hsa_prefill and hsa_decode on one stream and reads device-side errors
 * through hsa_check.  Inputs are a small deterministic pattern; the program
 * prints a checksum of each output and exits non-zero on any failed status.
 *
 *   cc -std=c99 -I include -I <cuda>/include tests/c_abi_example.c \
 *      -L <package dir> -lhsa -L <cuda>/lib64 -lcudart -o c_abi_example
 */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "hsa.h"

#define CK_CUDA(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 1; } } while (0)
#define CK_HSA(x) do { hsa_status_t s_ = (x); if (s_ != HSA_OK) { \
    fprintf(stderr, "%s: %s\n", #x, hsa_status_string(s_)); return 1; } } while (0)

/* fp32 -> bf16, round to nearest even (inputs are finite) */
static uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
static float from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* a bf16 device buffer of n elements filled with a fixed pattern */
static void *dev_pattern(size_t n, unsigned seed) {
    uint16_t *h = (uint16_t *)malloc(n * 2);
    void *d = NULL;
    for (size_t i = 0; i < n; ++i) h[i] = to_bf16(sinf(0.37f * (float)(i % 9973) + (float)seed));
    if (h && cudaMalloc(&d, n * 2) == cudaSuccess && cudaMemcpy(d, h, n * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(d);
        d = NULL;
    }
    free(h);
    return d;
}

static double checksum(const void *dev, size_t n) {
    uint16_t *h = (uint16_t *)malloc(n * 2);
    double s = 0.0;
    if (h && cudaMemcpy(h, dev, n * 2, cudaMemcpyDeviceToHost) == cudaSuccess)
        for (size_t i = 0; i < n; ++i) s += fabs((double)from_bf16(h[i]));
    free(h);
    return s;
}

int main(void) {
    const int B = 1, H = 16, Hkv = 2, d = 128, S = 64, topk = 8;
    const int64_t L = 64 * 20 + 7, Lc = 64 * 40;
    cudaStream_t st;
    CK_CUDA(cudaStreamCreate(&st));

    /* prefill: Q [B, L, H, d], K and V [B, Hkv, L, d], DHSA landmarks (lm = NULL) */
    void *Q = dev_pattern((size_t)B * L * H * d, 1), *K = dev_pattern((size_t)B * Hkv * L * d, 2);
    void *V = dev_pattern((size_t)B * Hkv * L * d, 3), *O = NULL, *ws = NULL;
    if (!Q || !K || !V) return 1;
    CK_CUDA(cudaMalloc(&O, (size_t)B * L * H * d * 2));
    const size_t ws_bytes = hsa_prefill_workspace_size(B, H, Hkv, L, d, S, topk);
    if (ws_bytes == 0) return 1;
    CK_CUDA(cudaMalloc(&ws, ws_bytes));
    CK_CUDA(cudaMemset(ws, 0, ws_bytes));
    CK_HSA(hsa_prefill(Q, K, V, HSA_BF16, NULL, HSA_F32, B, H, Hkv, L, d, S, topk, 1, 0.0f,
                       O, NULL, NULL, ws, ws_bytes, st));
    CK_HSA(hsa_check(ws, st));
    printf("prefill O checksum %.6e\n", checksum(O, (size_t)B * L * H * d));

    /* decode: q [B, H, d] at position Lc of a [B, Hkv, Lc, d] cache, bf16 landmarks */
    void *q = dev_pattern((size_t)B * H * d, 4), *Kc = dev_pattern((size_t)B * Hkv * Lc * d, 5);
    void *Vc = dev_pattern((size_t)B * Hkv * Lc * d, 6), *lm = dev_pattern((size_t)B * Hkv * (Lc / S) * d, 7);
    void *Od = NULL, *wsd = NULL;
    if (!q || !Kc || !Vc || !lm) return 1;
    CK_CUDA(cudaMalloc(&Od, (size_t)B * H * d * 2));
    const size_t wsd_bytes = hsa_decode_workspace_size(B, H, Hkv, Lc, d, S, topk);
    if (wsd_bytes == 0) return 1;
    CK_CUDA(cudaMalloc(&wsd, wsd_bytes));
    CK_CUDA(cudaMemset(wsd, 0, wsd_bytes));
    CK_HSA(hsa_decode(q, Kc, Vc, HSA_BF16, lm, HSA_BF16, B, H, Hkv, Lc, d, S, topk, 0.0f,
                      Od, NULL, wsd, wsd_bytes, st));
    CK_HSA(hsa_check(wsd, st));
    printf("decode O checksum %.6e\n", checksum(Od, (size_t)B * H * d));

    cudaFree(Q); cudaFree(K); cudaFree(V); cudaFree(O); cudaFree(ws);
    cudaFree(q); cudaFree(Kc); cudaFree(Vc); cudaFree(lm); cudaFree(Od); cudaFree(wsd);
    cudaStreamDestroy(st);
    printf("hsa %d ok\n", hsa_version());
    return 0;
}
