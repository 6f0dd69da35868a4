/*
 * The forward called from plain C through include/flce.h: no Python, no
 * torch.  Reads bf16 H (N x D), bf16 W (V x D) and int64 y (N) as raw files,
 * allocates device memory with the CUDA runtime, runs flce_forward on the
 * default stream, reads the device status with flce_check, and writes loss,
 * lse and target logit (N float32 each) and the mean (1 float32) to a file.
 *
 *   flce_from_c N V D H.bin W.bin y.bin out.bin
 *
 * Exit status 0 on success; otherwise the failing call is printed with the
 * library's status string.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "flce.h"

static void* read_file(const char* path, size_t bytes) {
    FILE* f = fopen(path, "rb");
    if (!f) return NULL;
    void* p = malloc(bytes ? bytes : 1);
    size_t got = p ? fread(p, 1, bytes, f) : 0;
    fclose(f);
    if (got != bytes) {
        free(p);
        return NULL;
    }
    return p;
}

#define CUDA_OK(call)                                                        \
    do {                                                                     \
        cudaError_t e_ = (call);                                             \
        if (e_ != cudaSuccess) {                                             \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));      \
            return 2;                                                        \
        }                                                                    \
    } while (0)

int main(int argc, char** argv) {
    if (argc != 8) {
        fprintf(stderr, "usage: %s N V D H.bin W.bin y.bin out.bin\n", argv[0]);
        return 1;
    }
    const int64_t N = atoll(argv[1]), V = atoll(argv[2]), D = atoll(argv[3]);
    const size_t hb = (size_t)N * D * 2, wb = (size_t)V * D * 2, yb = (size_t)N * 8;
    void* H = read_file(argv[4], hb);
    void* W = read_file(argv[5], wb);
    void* y = read_file(argv[6], yb);
    if (!H || !W || !y) {
        fprintf(stderr, "could not read the inputs\n");
        return 1;
    }

    const size_t ws_bytes = flce_workspace_size(N, V, D, FLCE_BF16);
    if (ws_bytes == 0) {
        fprintf(stderr, "flce_workspace_size: invalid sizes\n");
        return 1;
    }
    void *dH, *dW, *dy, *ws;
    float* dout;   /* loss | lse | target | mean */
    CUDA_OK(cudaMalloc(&dH, hb));
    CUDA_OK(cudaMalloc(&dW, wb));
    CUDA_OK(cudaMalloc(&dy, yb));
    CUDA_OK(cudaMalloc((void**)&dout, (3 * (size_t)N + 1) * sizeof(float)));
    CUDA_OK(cudaMalloc(&ws, ws_bytes));
    CUDA_OK(cudaMemcpy(dH, H, hb, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(dW, W, wb, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(dy, y, yb, cudaMemcpyHostToDevice));

    flce_status s = flce_forward(dH, dW, (const int64_t*)dy, N, V, D, FLCE_BF16, dout, dout + N,
                                 dout + 2 * N, dout + 3 * N, ws, ws_bytes, NULL);
    if (s != FLCE_OK) {
        fprintf(stderr, "flce_forward: %s\n", flce_status_string(s));
        return 3;
    }
    s = flce_check(ws, NULL);
    if (s != FLCE_OK) {
        fprintf(stderr, "flce_check: %s\n", flce_status_string(s));
        return 4;
    }

    const size_t ob = (3 * (size_t)N + 1) * sizeof(float);
    float* out = (float*)malloc(ob);
    CUDA_OK(cudaMemcpy(out, dout, ob, cudaMemcpyDeviceToHost));
    FILE* f = fopen(argv[7], "wb");
    if (!f || fwrite(out, 1, ob, f) != ob) {
        fprintf(stderr, "could not write %s\n", argv[7]);
        return 1;
    }
    fclose(f);
    printf("mean loss %.6f over %lld tokens\n", out[3 * N], (long long)N);
    cudaFree(dH);
    cudaFree(dW);
    cudaFree(dy);
    cudaFree(dout);
    cudaFree(ws);
    free(out);
    free(H);
    free(W);
    free(y);
    return 0;
}
