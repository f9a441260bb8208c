/*
 * Calls across a device reset, from plain C (no Python, no torch, whose own context a
 * reset would break).  cudaDeviceReset ends this process's context on the device and
 * unloads the library's module; the next call runs in a new context, where a kernel's
 * shared-memory opt-in and the device address of the library's __device__ scratch array
 * must be set up again.  Each of two rounds -- before and after the reset -- allocates
 * its buffers, runs coact_count (E = 256: the shared-memory histogram, which needs the
 * opt-in) and plan_dispatch_noalloc (the library's own scratch), and writes the results.
 *
 * Input file (little endian): int32 N, k, E, R, n_nodes; int32 ids[N*k];
 * int32 expert_rank[E]; int32 rank_node[R].
 * Output file, per round: int32 err_flag; int64 pair[E*E]; int64 loads[E];
 * int32 rank_offsets[R+1]; int32 send_row[N*k]; int32 comb_row[N*k]; int64 stats[8].
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "coact.h"

#define CHECK_CUDA(x)                                                                    \
    do {                                                                                 \
        cudaError_t e_ = (x);                                                            \
        if (e_ != cudaSuccess) {                                                         \
            fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, cudaGetErrorString(e_));   \
            return 2;                                                                    \
        }                                                                                \
    } while (0)
#define CHECK_COACT(x)                                                                   \
    do {                                                                                 \
        int s_ = (x);                                                                    \
        if (s_ != COACT_OK) {                                                            \
            fprintf(stderr, "%s:%d %s (cuda %d)\n", __FILE__, __LINE__,                  \
                    coact_strerror(s_), coact_last_cuda_error());                        \
            return 3;                                                                    \
        }                                                                                \
    } while (0)

static int put(FILE *f, const void *dev, size_t bytes) {
    void *h = malloc(bytes ? bytes : 1);
    if (!h) return 1;
    int bad = bytes && cudaMemcpy(h, dev, bytes, cudaMemcpyDeviceToHost) != cudaSuccess;
    if (!bad && bytes && fwrite(h, 1, bytes, f) != bytes) bad = 1;
    free(h);
    return bad;
}

static int round_trip(FILE *fo, int32_t N, int32_t k, int32_t E, int32_t R, int32_t n_nodes,
                      const int32_t *ids_h, const int32_t *er_h, const int32_t *rn_h) {
    const size_t nk = (size_t)N * (size_t)k;
    const int64_t cap = (int64_t)N * (k < R ? k : R);
    int32_t *ids, *er, *rn, *rank_counts, *rank_offsets, *asg_offsets, *row_token, *send_row,
        *comb_row, *err;
    int64_t *pair, *loads, *stats;
    uint8_t *row_kmask;
    cudaStream_t st;
    CHECK_CUDA(cudaStreamCreate(&st));
    CHECK_CUDA(cudaMalloc((void **)&ids, nk * 4));
    CHECK_CUDA(cudaMalloc((void **)&er, (size_t)E * 4));
    CHECK_CUDA(cudaMalloc((void **)&rn, (size_t)R * 4));
    CHECK_CUDA(cudaMalloc((void **)&rank_counts, (size_t)R * 4));
    CHECK_CUDA(cudaMalloc((void **)&rank_offsets, (size_t)(R + 1) * 4));
    CHECK_CUDA(cudaMalloc((void **)&asg_offsets, (size_t)(R + 1) * 4));
    CHECK_CUDA(cudaMalloc((void **)&row_token, (size_t)cap * 4));
    CHECK_CUDA(cudaMalloc((void **)&row_kmask, (size_t)cap));
    CHECK_CUDA(cudaMalloc((void **)&send_row, nk * 4));
    CHECK_CUDA(cudaMalloc((void **)&comb_row, nk * 4));
    CHECK_CUDA(cudaMalloc((void **)&err, 4));
    CHECK_CUDA(cudaMalloc((void **)&pair, (size_t)E * E * 8));
    CHECK_CUDA(cudaMalloc((void **)&loads, (size_t)E * 8));
    CHECK_CUDA(cudaMalloc((void **)&stats, 8 * 8));
    CHECK_CUDA(cudaMemcpy(ids, ids_h, nk * 4, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(er, er_h, (size_t)E * 4, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(rn, rn_h, (size_t)R * 4, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemset(err, 0, 4));
    CHECK_CUDA(cudaMemset(pair, 0, (size_t)E * E * 8));
    CHECK_CUDA(cudaMemset(loads, 0, (size_t)E * 8));
    CHECK_COACT(coact_count(ids, N, k, E, NULL, 0, 0, pair, loads, err, (coact_stream_t)st));
    CHECK_COACT(plan_dispatch_noalloc(ids, N, k, E, er, R, rn, n_nodes, NULL, rank_counts,
                                      rank_offsets, asg_offsets, NULL, row_token, row_kmask, cap,
                                      send_row, comb_row, stats, NULL, err, (coact_stream_t)st));
    CHECK_CUDA(cudaStreamSynchronize(st));
    if (put(fo, err, 4) || put(fo, pair, (size_t)E * E * 8) || put(fo, loads, (size_t)E * 8) ||
        put(fo, rank_offsets, (size_t)(R + 1) * 4) || put(fo, send_row, nk * 4) ||
        put(fo, comb_row, nk * 4) || put(fo, stats, 8 * 8))
        return 5;
    void *bufs[] = {ids, er, rn, rank_counts, rank_offsets, asg_offsets, row_token, row_kmask,
                    send_row, comb_row, err, pair, loads, stats};
    for (size_t i = 0; i < sizeof bufs / sizeof bufs[0]; ++i) CHECK_CUDA(cudaFree(bufs[i]));
    CHECK_CUDA(cudaStreamDestroy(st));
    return 0;
}

int main(int argc, char **argv) {
    if (argc != 3) {
        fprintf(stderr, "usage: %s <inputs> <outputs>\n", argv[0]);
        return 1;
    }
    FILE *fi = fopen(argv[1], "rb");
    if (!fi) return 1;
    int32_t hdr[5];
    if (fread(hdr, 4, 5, fi) != 5) return 1;
    const int32_t N = hdr[0], k = hdr[1], E = hdr[2], R = hdr[3], n_nodes = hdr[4];
    const size_t nk = (size_t)N * (size_t)k;
    int32_t *ids = malloc(nk * 4), *er = malloc((size_t)E * 4), *rn = malloc((size_t)R * 4);
    if (!ids || !er || !rn) return 1;
    if (fread(ids, 4, nk, fi) != nk || fread(er, 4, (size_t)E, fi) != (size_t)E ||
        fread(rn, 4, (size_t)R, fi) != (size_t)R)
        return 1;
    fclose(fi);
    FILE *fo = fopen(argv[2], "wb");
    if (!fo) return 1;
    int rc = round_trip(fo, N, k, E, R, n_nodes, ids, er, rn);
    if (rc) return rc;
    CHECK_CUDA(cudaDeviceReset());
    rc = round_trip(fo, N, k, E, R, n_nodes, ids, er, rn);
    if (rc) return rc;
    fclose(fo);
    free(ids);
    free(er);
    free(rn);
    return 0;
}
