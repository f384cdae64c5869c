/*
 * A plain C99 user of libw4a16: quantize a seeded 4096 x 1024 layer on the GPU, fold 1/s
 * into 4 tokens of activations, run the W4A16 linear and check the device status.  Given a
 * directory argument, it also writes its inputs and output there as raw little-endian files
 * (W.f32 [N][K], act.f32 [K], x.bf16 [M][K], y.bf16 [M][N]) for a checker to compare.
 *
 * The tests compile and link it on any machine (the header must be valid C and every
 * entry point it uses must resolve); run it on an sm_100 GPU to see the library work:
 *   gcc -std=c99 -I include -I /usr/local/cuda/include tests/c_abi/quantize_and_linear.c \
 *       -L w4a16_gemm_awq_b200 -lw4a16 -L /usr/local/cuda/lib64 -lcudart -o example
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "w4a16.h"

#define N_OUT 4096
#define K_IN 1024
#define M_TOK 4

static int cuda_ok(cudaError_t e, const char* what) {
    if (e != cudaSuccess) fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    return e == cudaSuccess;
}

static int lib_ok(w4a16_status s, const char* what) {
    if (s != W4A16_OK) fprintf(stderr, "%s: %s\n", what, w4a16_status_string(s));
    return s == W4A16_OK;
}

/* uniform in [lo, hi) from a 64-bit linear congruential generator */
static float uniform(uint64_t* state, float lo, float hi) {
    *state = *state * 6364136223846793005ull + 1442695040888963407ull;
    return lo + (hi - lo) * (float)((*state >> 40) * (1.0 / 16777216.0));
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs) */
static uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static int dump(const char* dir, const char* name, const void* data, size_t bytes) {
    char path[4096];
    FILE* f;
    size_t w;
    if (snprintf(path, sizeof path, "%s/%s", dir, name) >= (int)sizeof path) return 0;
    f = fopen(path, "wb");
    if (!f) {
        fprintf(stderr, "cannot write %s\n", path);
        return 0;
    }
    w = fwrite(data, 1, bytes, f);
    fclose(f);
    return w == bytes;
}

int main(int argc, char** argv) {
    const size_t nw = (size_t)N_OUT * K_IN, nx = (size_t)M_TOK * K_IN, ny = (size_t)M_TOK * N_OUT;
    const size_t groups = K_IN / 128;
    float* hW = malloc(nw * sizeof(float));
    float* ha = malloc(K_IN * sizeof(float));
    uint16_t* hx = malloc(nx * sizeof(uint16_t));
    uint16_t* hy = malloc(ny * sizeof(uint16_t));
    uint64_t st = 2024;
    size_t i;
    int ok = hW && ha && hx && hy;
    float *dW = NULL, *da = NULL, *ds = NULL;
    uint32_t *dq = NULL, *dz = NULL;
    uint16_t *dsc = NULL, *dx = NULL, *dxf = NULL, *dy = NULL;
    void* dws = NULL;
    const size_t ws_bytes = w4a16_workspace_bytes(M_TOK, N_OUT, K_IN);

    for (i = 0; ok && i < nw; ++i) hW[i] = uniform(&st, -0.05f, 0.05f);
    for (i = 0; ok && i < K_IN; ++i) ha[i] = uniform(&st, 0.25f, 4.0f);
    for (i = 0; ok && i < nx; ++i) hx[i] = to_bf16(uniform(&st, -1.0f, 1.0f));

    ok = ok && cuda_ok(cudaMalloc((void**)&dW, nw * sizeof(float)), "cudaMalloc W");
    ok = ok && cuda_ok(cudaMalloc((void**)&da, K_IN * sizeof(float)), "cudaMalloc act");
    ok = ok && cuda_ok(cudaMalloc((void**)&ds, K_IN * sizeof(float)), "cudaMalloc s");
    ok = ok && cuda_ok(cudaMalloc((void**)&dq, nw / 8 * sizeof(uint32_t)), "cudaMalloc qweight");
    ok = ok && cuda_ok(cudaMalloc((void**)&dsc, groups * N_OUT * sizeof(uint16_t)), "cudaMalloc scales");
    ok = ok && cuda_ok(cudaMalloc((void**)&dz, groups * (N_OUT / 8) * sizeof(uint32_t)), "cudaMalloc zeros");
    ok = ok && cuda_ok(cudaMalloc((void**)&dx, nx * sizeof(uint16_t)), "cudaMalloc x");
    ok = ok && cuda_ok(cudaMalloc((void**)&dxf, nx * sizeof(uint16_t)), "cudaMalloc x'");
    ok = ok && cuda_ok(cudaMalloc((void**)&dy, ny * sizeof(uint16_t)), "cudaMalloc y");
    ok = ok && ws_bytes > 0 && cuda_ok(cudaMalloc(&dws, ws_bytes), "cudaMalloc workspace");
    ok = ok && cuda_ok(cudaMemset(dws, 0, ws_bytes), "cudaMemset workspace");  /* zeroed once */
    ok = ok && cuda_ok(cudaMemcpy(dW, hW, nw * sizeof(float), cudaMemcpyHostToDevice), "copy W");
    ok = ok && cuda_ok(cudaMemcpy(da, ha, K_IN * sizeof(float), cudaMemcpyHostToDevice), "copy act");
    ok = ok && cuda_ok(cudaMemcpy(dx, hx, nx * sizeof(uint16_t), cudaMemcpyHostToDevice), "copy x");

    ok = ok && lib_ok(awq_quantize_g128(dW, da, 0.5f, N_OUT, K_IN, dq, dsc, dz, ds, NULL), "awq_quantize_g128");
    ok = ok && lib_ok(awq_fold_activations(dx, ds, dxf, M_TOK, K_IN, NULL), "awq_fold_activations");
    ok = ok && lib_ok(w4a16_linear(dxf, dq, dsc, dz, NULL, dy, M_TOK, N_OUT, K_IN, dws, ws_bytes, NULL),
                      "w4a16_linear");
    ok = ok && lib_ok(w4a16_check_device_status(NULL), "device status");
    ok = ok && cuda_ok(cudaMemcpy(hy, dy, ny * sizeof(uint16_t), cudaMemcpyDeviceToHost), "copy y");
    if (ok && argc > 1)
        ok = dump(argv[1], "W.f32", hW, nw * sizeof(float)) && dump(argv[1], "act.f32", ha, K_IN * sizeof(float)) &&
             dump(argv[1], "x.bf16", hx, nx * sizeof(uint16_t)) && dump(argv[1], "y.bf16", hy, ny * sizeof(uint16_t));
    if (ok)
        printf("y[0][0..3] = %g %g %g %g\nok\n", from_bf16(hy[0]), from_bf16(hy[1]), from_bf16(hy[2]),
               from_bf16(hy[3]));

    cudaFree(dW);
    cudaFree(da);
    cudaFree(ds);
    cudaFree(dq);
    cudaFree(dsc);
    cudaFree(dz);
    cudaFree(dx);
    cudaFree(dxf);
    cudaFree(dy);
    cudaFree(dws);
    free(hW);
    free(ha);
    free(hx);
    free(hy);
    return ok ? 0 : 1;
}
