/*
 * The dispatch/combine path through the C ABI from plain C (no Python, no torch): reads
 * ids, gates, expert_rank, x and y from an input file, runs coact_count, plan_dispatch,
 * dispatch_gather and combine_scatter on its own CUDA stream with cudaMalloc'd buffers,
 * and writes pair, loads, the plan's send_row / comb_row / rank_offsets, the gathered
 * rows and the combined rows (fp32) to an output file.
 *
 * Input file (little endian): int32 N, k, E, R, H; int32 ids[N*k]; float gates[N*k];
 * int32 expert_rank[E]; uint16 x[N*H]; uint16 y[N*k*H].
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
            fprintf(stderr, "%s:%d %s\n", __FILE__, __LINE__, coact_strerror(s_));       \
            return 3;                                                                    \
        }                                                                                \
    } while (0)

static void *read_n(FILE *f, size_t bytes) {
    void *p = malloc(bytes ? bytes : 1);
    if (p && bytes && fread(p, 1, bytes, f) != bytes) {
        free(p);
        return NULL;
    }
    return p;
}

static void *to_dev(const void *h, size_t bytes) {
    void *d = NULL;
    if (cudaMalloc(&d, bytes ? bytes : 16) != cudaSuccess) return NULL;
    if (bytes && cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

int main(int argc, char **argv) {
    if (argc != 3) {
        fprintf(stderr, "usage: %s <inputs> <outputs>\n", argv[0]);
        return 1;
    }
    if (coact_abi_version() != COACT_ABI_VERSION) return 4;
    FILE *fi = fopen(argv[1], "rb");
    if (!fi) return 1;
    int32_t hdr[5];
    if (fread(hdr, sizeof(int32_t), 5, fi) != 5) return 1;
    const int64_t N = hdr[0], H = hdr[4];
    const int k = hdr[1], E = hdr[2], R = hdr[3];
    int32_t *ids = read_n(fi, sizeof(int32_t) * N * k);
    float *gates = read_n(fi, sizeof(float) * N * k);
    int32_t *er = read_n(fi, sizeof(int32_t) * E);
    uint16_t *x = read_n(fi, sizeof(uint16_t) * N * H);
    uint16_t *y = read_n(fi, sizeof(uint16_t) * N * k * H);
    fclose(fi);
    if (!ids || !gates || !er || !x || !y) return 1;

    cudaStream_t st;
    CHECK_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
    int32_t *d_ids = to_dev(ids, sizeof(int32_t) * N * k);
    float *d_gates = to_dev(gates, sizeof(float) * N * k);
    int32_t *d_er = to_dev(er, sizeof(int32_t) * E);
    uint16_t *d_x = to_dev(x, sizeof(uint16_t) * N * H);
    uint16_t *d_y = to_dev(y, sizeof(uint16_t) * N * k * H);
    const int64_t cap = N * (k < R ? k : R);
    int64_t *d_pair = NULL, *d_loads = NULL, *d_stats = NULL;
    int32_t *d_counts = NULL, *d_offs = NULL, *d_asg = NULL, *d_row_token = NULL;
    int32_t *d_send_row = NULL, *d_comb_row = NULL, *d_err = NULL;
    uint8_t *d_kmask = NULL;
    uint16_t *d_send = NULL;
    float *d_out = NULL;
    void *d_ws = NULL;
    const size_t ws = plan_dispatch_workspace_bytes(N, k, E, R);
    CHECK_CUDA(cudaMalloc((void **)&d_pair, sizeof(int64_t) * E * E));
    CHECK_CUDA(cudaMalloc((void **)&d_loads, sizeof(int64_t) * E));
    CHECK_CUDA(cudaMalloc((void **)&d_stats, sizeof(int64_t) * COACT_NUM_STATS));
    CHECK_CUDA(cudaMalloc((void **)&d_counts, sizeof(int32_t) * R));
    CHECK_CUDA(cudaMalloc((void **)&d_offs, sizeof(int32_t) * (R + 1)));
    CHECK_CUDA(cudaMalloc((void **)&d_asg, sizeof(int32_t) * (R + 1)));
    CHECK_CUDA(cudaMalloc((void **)&d_row_token, sizeof(int32_t) * cap));
    CHECK_CUDA(cudaMalloc((void **)&d_kmask, cap));
    CHECK_CUDA(cudaMalloc((void **)&d_send_row, sizeof(int32_t) * N * k));
    CHECK_CUDA(cudaMalloc((void **)&d_comb_row, sizeof(int32_t) * N * k));
    CHECK_CUDA(cudaMalloc((void **)&d_err, sizeof(int32_t)));
    CHECK_CUDA(cudaMalloc((void **)&d_send, sizeof(uint16_t) * cap * H));
    CHECK_CUDA(cudaMalloc((void **)&d_out, sizeof(float) * N * H));
    CHECK_CUDA(cudaMalloc(&d_ws, ws));
    if (!d_ids || !d_gates || !d_er || !d_x || !d_y) return 2;
    CHECK_CUDA(cudaMemsetAsync(d_pair, 0, sizeof(int64_t) * E * E, st));
    CHECK_CUDA(cudaMemsetAsync(d_loads, 0, sizeof(int64_t) * E, st));
    CHECK_CUDA(cudaMemsetAsync(d_err, 0, sizeof(int32_t), st));
    coact_stream_t cs = (coact_stream_t)st;

    CHECK_COACT(coact_count(d_ids, N, k, E, NULL, 0, 0, d_pair, d_loads, d_err, cs));
    CHECK_COACT(plan_dispatch(d_ids, N, k, E, d_er, R, NULL, 1, NULL, d_counts, d_offs, d_asg, NULL,
                              d_row_token, d_kmask, cap, d_send_row, d_comb_row, d_stats, NULL,
                              d_ws, ws, d_err, cs));
    CHECK_COACT(dispatch_gather(d_x, N, H, d_send_row, k, d_send, cap, d_err, cs));
    CHECK_COACT(combine_scatter(d_y, N * k, d_gates, d_comb_row, N, k, H, d_out, 1, d_err, cs));
    CHECK_CUDA(cudaStreamSynchronize(st));

    int32_t err = 0, offs_last = 0;
    CHECK_CUDA(cudaMemcpy(&err, d_err, sizeof(int32_t), cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(&offs_last, d_offs + R, sizeof(int32_t), cudaMemcpyDeviceToHost));
    const int64_t D = offs_last;
    int64_t *pair = malloc(sizeof(int64_t) * E * E), *loads = malloc(sizeof(int64_t) * E);
    int32_t *send_row = malloc(sizeof(int32_t) * N * k), *comb_row = malloc(sizeof(int32_t) * N * k);
    int32_t *offs = malloc(sizeof(int32_t) * (R + 1));
    uint16_t *send = malloc(sizeof(uint16_t) * (D > 0 ? D : 1) * H);
    float *out = malloc(sizeof(float) * N * H);
    CHECK_CUDA(cudaMemcpy(pair, d_pair, sizeof(int64_t) * E * E, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(loads, d_loads, sizeof(int64_t) * E, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(send_row, d_send_row, sizeof(int32_t) * N * k, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(comb_row, d_comb_row, sizeof(int32_t) * N * k, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(offs, d_offs, sizeof(int32_t) * (R + 1), cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(send, d_send, sizeof(uint16_t) * D * H, cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(out, d_out, sizeof(float) * N * H, cudaMemcpyDeviceToHost));

    FILE *fo = fopen(argv[2], "wb");
    if (!fo) return 1;
    fwrite(&err, sizeof(int32_t), 1, fo);
    fwrite(pair, sizeof(int64_t), E * E, fo);
    fwrite(loads, sizeof(int64_t), E, fo);
    fwrite(offs, sizeof(int32_t), R + 1, fo);
    fwrite(send_row, sizeof(int32_t), N * k, fo);
    fwrite(comb_row, sizeof(int32_t), N * k, fo);
    fwrite(send, sizeof(uint16_t), D * H, fo);
    fwrite(out, sizeof(float), N * H, fo);
    fclose(fo);
    CHECK_CUDA(cudaStreamDestroy(st));
    return 0;
}
