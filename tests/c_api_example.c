/*
 * Calling libssd.so from plain C (no Python, no torch): one fp32 scan over two
 * short sequences, then one decode step that continues from the scan's final
 * state.  Built by tests/test_c_api.py against include/ssd.h and the in-tree
 * library.  Run with a file name, it writes every input and output there
 * (float32, in the order of dump() below) so that a test can check them
 * against an independent implementation.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

#include "ssd.h"

#define CHECK_CUDA(e)                                                            \
    do {                                                                         \
        cudaError_t err_ = (e);                                                  \
        if (err_ != cudaSuccess) {                                               \
            fprintf(stderr, "CUDA: %s\n", cudaGetErrorString(err_));             \
            return 1;                                                            \
        }                                                                        \
    } while (0)

static float* dev_fill(size_t n, float scale) {
    float* h = (float*)malloc(n * sizeof(float));
    for (size_t i = 0; i < n; ++i) h[i] = scale * (float)((i * 2654435761u) % 1000u) / 1000.f - 0.5f * scale;
    float* d = NULL;
    if (cudaMalloc((void**)&d, n * sizeof(float)) != cudaSuccess) d = NULL;
    if (d) cudaMemcpy(d, h, n * sizeof(float), cudaMemcpyHostToDevice);
    free(h);
    return d;
}

static int dump(FILE* f, const float* d, size_t n) {
    float* h = (float*)malloc(n * sizeof(float));
    if (!h || cudaMemcpy(h, d, n * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
    const int bad = fwrite(h, sizeof(float), n, f) != n;
    free(h);
    return bad;
}

int main(int argc, char** argv) {
    const int64_t b = 2, L = 100, H = 4, P = 16, N = 16, G = 2;
    ssd_dims dims = {b, L, H, P, N, G, 0, SSD_F32};
    float *x = dev_fill(b * L * H * P, 1.f), *dt = dev_fill(b * L * H, 1.f);
    float *Bm = dev_fill(b * L * G * N, 1.f), *Cm = dev_fill(b * L * G * N, 1.f);
    float *D = dev_fill(H, 1.f), *bias = dev_fill(H, 0.1f);
    const float A_host[4] = {-1.f, -2.f, -0.5f, -4.f};   /* A_h < 0: a decaying state */
    float* A = NULL;
    CHECK_CUDA(cudaMalloc((void**)&A, sizeof(A_host)));
    CHECK_CUDA(cudaMemcpy(A, A_host, sizeof(A_host), cudaMemcpyHostToDevice));
    float *y = NULL, *state = NULL;
    if (!x || !dt || !Bm || !Cm || !A || !D || !bias) return 1;
    CHECK_CUDA(cudaMalloc((void**)&y, b * L * H * P * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&state, b * H * N * P * sizeof(float)));

    int rc = ssd_chunk_scan_fwd(&dims, x, dt, bias, A, Bm, Cm, D, NULL, NULL, 64, y, state, NULL);
    if (rc != SSD_OK) {
        fprintf(stderr, "ssd_chunk_scan_fwd: %s (%s)\n", ssd_status_string(rc), ssd_last_error());
        return 2;
    }
    /* one more token per sequence, continuing from the final state in place */
    float *x1 = dev_fill(b * H * P, 1.f), *dt1 = dev_fill(b * H, 1.f);
    float *B1 = dev_fill(b * G * N, 1.f), *C1 = dev_fill(b * G * N, 1.f), *y1 = dev_fill(b * H * P, 0.f);
    rc = ssd_state_update(&dims, state, x1, dt1, A, B1, C1, D, y1, NULL, bias);
    if (rc != SSD_OK) {
        fprintf(stderr, "ssd_state_update: %s (%s)\n", ssd_status_string(rc), ssd_last_error());
        return 3;
    }
    CHECK_CUDA(cudaDeviceSynchronize());
    if (argc > 1) {
        FILE* f = fopen(argv[1], "wb");
        if (!f) return 4;
        int bad = 0;
        bad |= dump(f, x, b * L * H * P) | dump(f, dt, b * L * H) | dump(f, Bm, b * L * G * N);
        bad |= dump(f, Cm, b * L * G * N) | dump(f, A, H) | dump(f, D, H) | dump(f, bias, H);
        bad |= dump(f, y, b * L * H * P) | dump(f, x1, b * H * P) | dump(f, dt1, b * H);
        bad |= dump(f, B1, b * G * N) | dump(f, C1, b * G * N) | dump(f, y1, b * H * P);
        bad |= dump(f, state, b * H * N * P);
        fclose(f);
        if (bad) return 5;
    }
    printf("ok\n");
    return 0;
}
