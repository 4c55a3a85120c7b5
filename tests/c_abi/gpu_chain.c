/*
 * A plain C program driving the GPU path through the C-ABI: device buffers
 * from the CUDA runtime, a reorder of arbitrary bytes and its inverse, and a
 * bit-exact comparison of the reorder with the oracle's byte-copy
 * permutation (test infrastructure, linked here only). Exit status 0 and
 * "ok" on success.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "atlas.h"

int atlas_oracle_cube_reorder(const unsigned char *src, unsigned char *dst, int64_t T,
                              int64_t H, int64_t W, int64_t ct, int64_t ch, int64_t cw,
                              int64_t row_bytes);

static int fail(const char *what) {
    fprintf(stderr, "FAIL: %s\n", what);
    return 1;
}

int main(void) {
    const atlas_grid3 grid = {5, 7, 9};
    const atlas_cube3 cube = {2, 3, 4};
    const int32_t heads = 2, hd = 64;
    const int64_t n = 5 * 7 * 9, row = (int64_t)heads * hd * 4;
    const size_t bytes = (size_t)(n * row);
    unsigned char *h_x = (unsigned char *)malloc(bytes), *h_y = (unsigned char *)malloc(bytes);
    unsigned char *h_ref = (unsigned char *)malloc(bytes), *h_z = (unsigned char *)malloc(bytes);
    uint64_t s = 0x9e3779b97f4a7c15ull;   /* input bytes: a fixed LCG stream */
    for (size_t i = 0; i < bytes; ++i) {
        s = s * 6364136223846793005ull + 1442695040888963407ull;
        h_x[i] = (unsigned char)(s >> 56);
    }
    void *d_x, *d_y, *d_z;
    if (cudaMalloc(&d_x, bytes) != cudaSuccess || cudaMalloc(&d_y, bytes) != cudaSuccess ||
        cudaMalloc(&d_z, bytes) != cudaSuccess)
        return fail("cudaMalloc");
    cudaMemcpy(d_x, h_x, bytes, cudaMemcpyHostToDevice);
    if (atlas_cube_reorder(d_x, d_y, grid, cube, heads, hd, ATLAS_FP32, NULL, NULL) != ATLAS_OK)
        return fail("reorder");
    if (atlas_cube_unorder(d_y, d_z, grid, cube, heads, hd, ATLAS_FP32, NULL) != ATLAS_OK)
        return fail("unorder");
    uint32_t code = 1;
    if (atlas_last_device_error(NULL, &code) != ATLAS_OK || code != 0) return fail("device error");
    cudaDeviceSynchronize();
    cudaMemcpy(h_y, d_y, bytes, cudaMemcpyDeviceToHost);
    cudaMemcpy(h_z, d_z, bytes, cudaMemcpyDeviceToHost);
    if (atlas_oracle_cube_reorder(h_x, h_ref, 5, 7, 9, 2, 3, 4, row) != 0) return fail("oracle");
    if (memcmp(h_y, h_ref, bytes) != 0) return fail("reorder differs from the oracle");
    if (memcmp(h_z, h_x, bytes) != 0) return fail("unorder is not the inverse");

    cudaFree(d_x);
    cudaFree(d_y);
    cudaFree(d_z);
    free(h_x);
    free(h_y);
    free(h_ref);
    free(h_z);
    printf("ok\n");
    return 0;
}
