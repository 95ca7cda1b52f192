/*
 * A plain C caller of the library: no Python, no torch. Reads a model and latents from the
 * binary files the test writes, runs create / encode / encode_step / decode / get_error on
 * the default stream through include/mimi_rvq.h, and writes the codes and decoded latents
 * back for the test to check against the float64 oracle.
 *
 * usage: c_abi_roundtrip <dir> <N>
 *   <dir>/codebooks.f32 [8][2048][256], W_in.f32 [256][512], W_out.f32 [512][256],
 *   latents.f32 [N][512]  ->  codes.i16 [N][8], step.i16 [N][8], decoded.f32 [N][512]
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "mimi_rvq.h"

static void *read_file(const char *dir, const char *name, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) return NULL;
    void *p = malloc(bytes);
    size_t got = p ? fread(p, 1, bytes, f) : 0;
    fclose(f);
    if (got != bytes) {
        free(p);
        return NULL;
    }
    return p;
}

static int write_file(const char *dir, const char *name, const void *p, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (!f) return 0;
    size_t put = fwrite(p, 1, bytes, f);
    fclose(f);
    return put == bytes;
}

static void *to_device(const void *host, size_t bytes) {
    void *d = NULL;
    if (cudaMalloc(&d, bytes) != cudaSuccess) return NULL;
    if (host && cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

#define CHECK(call)                                                                  \
    do {                                                                             \
        int st_ = (call);                                                            \
        if (st_ != MIMI_RVQ_OK) {                                                    \
            fprintf(stderr, "%s: %s\n", #call, mimi_rvq_strerror(st_));              \
            return 1;                                                                \
        }                                                                            \
    } while (0)

int main(int argc, char **argv) {
    if (argc != 3) return 2;
    const char *dir = argv[1];
    const long n = atol(argv[2]);
    const size_t nc = (size_t)MIMI_RVQ_NUM_CODEBOOKS * MIMI_RVQ_CODEBOOK_SIZE * MIMI_RVQ_DIM;
    const size_t nw = (size_t)MIMI_RVQ_DIM * MIMI_RVQ_LATENT_DIM;
    const size_t nz = (size_t)n * MIMI_RVQ_LATENT_DIM;
    const size_t ncodes = (size_t)n * MIMI_RVQ_NUM_CODEBOOKS;
    float *C = read_file(dir, "codebooks.f32", nc * 4);
    float *W_in = read_file(dir, "W_in.f32", nw * 4);
    float *W_out = read_file(dir, "W_out.f32", nw * 4);
    float *z = read_file(dir, "latents.f32", nz * 4);
    if (!C || !W_in || !W_out || !z) return 3;

    float *dC = to_device(C, nc * 4), *dWi = to_device(W_in, nw * 4), *dWo = to_device(W_out, nw * 4);
    float *dz = to_device(z, nz * 4), *dx = to_device(NULL, nz * 4);
    int16_t *dcodes = to_device(NULL, ncodes * 2), *dstep = to_device(NULL, ncodes * 2);
    if (!dC || !dWi || !dWo || !dz || !dx || !dcodes || !dstep) return 4;

    mimi_rvq_t h = NULL;
    CHECK(mimi_rvq_create(dC, dWi, dWo, &h));
    CHECK(mimi_rvq_encode(h, dz, MIMI_RVQ_F32, n, dcodes, NULL));
    CHECK(mimi_rvq_encode_step(h, dz, MIMI_RVQ_F32, (int)n, dstep, NULL));
    CHECK(mimi_rvq_decode(h, dcodes, n, dx, NULL));
    CHECK(mimi_rvq_get_error(h, NULL));
    /* argument errors come back at once */
    if (mimi_rvq_encode(h, dz, 7, n, dcodes, NULL) != MIMI_RVQ_EINVAL) return 5;

    int16_t *codes = malloc(ncodes * 2), *step = malloc(ncodes * 2);
    float *x = malloc(nz * 4);
    if (!codes || !step || !x) return 6;
    if (cudaMemcpy(codes, dcodes, ncodes * 2, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(step, dstep, ncodes * 2, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(x, dx, nz * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return 7;
    mimi_rvq_destroy(h);
    if (!write_file(dir, "codes.i16", codes, ncodes * 2) ||
        !write_file(dir, "step.i16", step, ncodes * 2) || !write_file(dir, "decoded.f32", x, nz * 4))
        return 8;
    printf("ok %ld frames\n", n);
    return 0;
}
