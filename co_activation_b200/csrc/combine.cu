// combine_scatter: weighted combine of expert outputs back to token order.
//
// Zyphra (arxivdaily 2610.09372), English abstract: all-to-all dispatches tokens to
// their experts "and then" combines the results; deduplicated dispatch leaves the
// routing decisions -- and so the combined result -- unchanged.
//
//   out[t] = sum_{j=0..k-1} gates[t,j] * y[comb_row[t,j]]
// per element: acc = +0.0f, acc = fmaf(g_j, y_j, acc) for j = 0..k-1 (one rounding per
// step, explicit __fmaf_rn so the compiler cannot reassociate), then fp32 out or bf16
// round-to-nearest-even.
//
// k_combine_v16: one warp per token.  Each lane covers 8 hidden elements per 16-byte
// column chunk and keeps U chunks x K rows of loads in flight before the FMAs.  The K
// source rows are scattered over y (expanded receive order), the output row is written
// once with streaming stores.  HBM traffic: N*k*H*2 (y) + N*H*(2|4) (out) + N*k*8.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace coact {
namespace {

template <int K, int U, bool F32>
__global__ void __launch_bounds__(256)
    k_combine_v16(const uint4 *__restrict__ y, int64_t n_rows, const float *__restrict__ gates,
                  const int32_t *__restrict__ comb_row, int64_t N, int64_t H16,
                  void *__restrict__ out, int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int flags = 0;
    for (int64_t t = gwarp; t < N; t += nwarps) {
        // lane j < K fetches row j and gate j; shuffles broadcast them
        int rl = -1;
        float gl = 0.f;
        if (lane < K) {
            rl = __ldg(comb_row + t * K + lane);
            gl = __ldg(gates + t * K + lane);
            if (rl < -1 || (int64_t)rl >= n_rows) flags |= COACT_EFLAG_ROW_RANGE;
            if (rl < 0 || (int64_t)rl >= n_rows) rl = -1;
        }
        int64_t row[K];
        float g[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            row[j] = __shfl_sync(0xffffffffu, rl, j);
            g[j] = __shfl_sync(0xffffffffu, gl, j);
        }
        for (int64_t c0 = 0; c0 < H16; c0 += 32 * U) {
            uint4 v[U][K];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
#pragma unroll
                for (int j = 0; j < K; ++j)
                    if (c < H16 && row[j] >= 0) v[u][j] = ld_stream(y + row[j] * H16 + c);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c >= H16) continue;
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    if (row[j] < 0) continue;
                    const uint32_t w[4] = {v[u][j].x, v[u][j].y, v[u][j].z, v[u][j].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] = __fmaf_rn(g[j], bf16lo(w[q]), acc[2 * q]);
                        acc[2 * q + 1] = __fmaf_rn(g[j], bf16hi(w[q]), acc[2 * q + 1]);
                    }
                }
                if (F32) {
                    float4 *o = reinterpret_cast<float4 *>(out) + (t * H16 + c) * 2;
                    __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
                    __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
                } else {
                    uint4 p;
                    uint32_t *pw = &p.x;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
                        pw[q] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    st_stream(reinterpret_cast<uint4 *>(out) + t * H16 + c, p);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

template <int K, bool F32>
int launch(const uint16_t *y, int64_t n_rows, const float *gates, const int32_t *comb_row,
           int64_t N, int64_t H, void *out, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
    // column chunks per lane: 8 loads in flight for k <= 2 (U = 4), U = 2 chunks for
    // k >= 3 (6-16 loads).  Measured on B200: U = 2 made k = 6 6% faster and k = 8
    // 0.4% faster than U = 1, while U = 8 made k = 2 1.6% slower than U = 4.
#if defined(COACT_COMBINE_LOADS)
    constexpr int U = K >= COACT_COMBINE_LOADS ? 1 : COACT_COMBINE_LOADS / K;  // experiments
#else
    constexpr int U = K <= 2 ? 4 : 2;
#endif
    const int64_t H16 = H / 8;
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(N, 8), (int64_t)di.sm_count * 8));
    return launch_pdl(k_combine_v16<K, U, F32>, blocks, 256, 0, st,
                      reinterpret_cast<const uint4 *>(y), n_rows, gates, comb_row, N, H16, out, err);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int combine_scatter(const uint16_t *y, int64_t n_rows, const float *gates,
                               const int32_t *comb_row, int64_t N, int k, int64_t H, void *out,
                               int out_dtype, int32_t *err_flag, coact_stream_t stream) {
    if (N < 0 || H < 0 || n_rows < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || (out_dtype != 0 && out_dtype != 1)) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return COACT_OK;
    if (!gates || !comb_row || !out || (n_rows > 0 && !y)) return COACT_ERR_INVALID;
    if ((y && !aligned16(y)) || !aligned16(out)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_COMBINE_CASE(KK)                                                                   \
    case KK:                                                                                     \
        return out_dtype ? launch<KK, true>(y, n_rows, gates, comb_row, N, H, out, err_flag, st, di) \
                         : launch<KK, false>(y, n_rows, gates, comb_row, N, H, out, err_flag, st, di);
    switch (k) {
        COACT_COMBINE_CASE(1)
        COACT_COMBINE_CASE(2)
        COACT_COMBINE_CASE(3)
        COACT_COMBINE_CASE(4)
        COACT_COMBINE_CASE(5)
        COACT_COMBINE_CASE(6)
        COACT_COMBINE_CASE(7)
        COACT_COMBINE_CASE(8)
    }
#undef COACT_COMBINE_CASE
    return COACT_ERR_UNSUPPORTED;
}
