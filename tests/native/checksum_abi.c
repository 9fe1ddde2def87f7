/* checksum_abi.c -- calls libdws's dws_checksum from plain C through the C ABI
 * (no Python in between) and prints what the library returned.
 *
 *   checksum_abi <input file>
 *
 * The input file holds: int64 pos_bytes, int64 nnz, then pos_bytes position
 * bytes and nnz bf16 values (uint16, little-endian).  The program copies them
 * to the device, calls dws_checksum, copies hashes[2] and checksum[2] back and
 * prints the four words in hex, one line: "<h0> <h1> <c0> <c1>".  Exit code 0
 * on success; any failing call prints its name and exits 1. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "dws.h"

static int fail(const char *what) {
    fprintf(stderr, "checksum_abi: %s failed\n", what);
    return 1;
}

int main(int argc, char **argv) {
    if (argc != 2) return fail("usage");
    FILE *f = fopen(argv[1], "rb");
    if (f == NULL) return fail("fopen");
    int64_t nb = 0, nv = 0;
    if (fread(&nb, 8, 1, f) != 1 || fread(&nv, 8, 1, f) != 1 || nb < 0 || nv < 0) return fail("header");
    uint8_t *hp = (uint8_t *)malloc((size_t)nb + 1);
    uint16_t *hv = (uint16_t *)malloc(2 * (size_t)nv + 2);
    if (hp == NULL || hv == NULL) return fail("malloc");
    if (fread(hp, 1, (size_t)nb, f) != (size_t)nb || fread(hv, 2, (size_t)nv, f) != (size_t)nv)
        return fail("read");
    fclose(f);

    uint8_t *dp = NULL;
    uint16_t *dv = NULL;
    uint64_t *dh = NULL;
    if (cudaMalloc((void **)&dp, (size_t)nb + 16) != cudaSuccess) return fail("cudaMalloc");
    if (cudaMalloc((void **)&dv, 2 * (size_t)nv + 16) != cudaSuccess) return fail("cudaMalloc");
    if (cudaMalloc((void **)&dh, 4 * sizeof(uint64_t)) != cudaSuccess) return fail("cudaMalloc");
    if (nb && cudaMemcpy(dp, hp, (size_t)nb, cudaMemcpyHostToDevice) != cudaSuccess) return fail("copy");
    if (nv && cudaMemcpy(dv, hv, 2 * (size_t)nv, cudaMemcpyHostToDevice) != cudaSuccess) return fail("copy");

    if (dws_checksum(dp, nb, dv, nv, dh, dh + 2, NULL) != DWS_OK) return fail("dws_checksum");
    uint64_t out[4];
    if (cudaMemcpy(out, dh, sizeof out, cudaMemcpyDeviceToHost) != cudaSuccess) return fail("copy back");
    printf("%016llx %016llx %016llx %016llx\n", (unsigned long long)out[0], (unsigned long long)out[1],
           (unsigned long long)out[2], (unsigned long long)out[3]);
    cudaFree(dp);
    cudaFree(dv);
    cudaFree(dh);
    free(hp);
    free(hv);
    return 0;
}
