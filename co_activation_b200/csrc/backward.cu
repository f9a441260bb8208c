// combine_scatter_backward: gradients of the combine with respect to the expert outputs
// and the gates.
//
// The combine out[t] = sum_j gates[t,j] * y[comb_row[t,j]] is linear in y and in the
// gates (Zyphra, arxivdaily 2610.09372, English abstract: dispatch "and then" combine),
// so for an upstream gradient grad_out:
//   grad_y[comb_row[t,j]] = gates[t,j] * grad_out[t]          fp32 product, bf16 RNE
//   grad_gates[t,j]       = <grad_out[t], y[comb_row[t,j]]>   fp32 dot product
// Units as in combine_rows: unit u is token row_token[u] restricted to the slots of
// row_kmask[u], with grad_out row u (the token's gradient row dispatched to that rank);
// without row_token, unit u is token u with all k slots.
//
// k_combine_bwd: one warp per unit.  The unit's live slots (with a row) are compacted in
// ascending slot order by a warp ballot.  Each lane owns 16 hidden elements per 32-byte
// column chunk (8 per 16-byte chunk where y, grad_out or grad_y is not 32-byte aligned);
// per group of U chunks it loads grad_out once, then streams the live rows of y G at a
// time, writing their scaled grad_y rows and accumulating one dot product per slot (fp32
// fma, a lane's elements in ascending order), reduced across the warp by a butterfly at
// the end.  Summation order of a dot product: each lane's chain of 16 * ceil(H/512)
// terms (8 * ceil(H/256) with 16-byte chunks), then 5 butterfly levels.
// HBM traffic: N*H*2 (grad_out) + N*k*H*2 (y) + N*k*H*2 (grad_y) + N*k*12.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace coact {
namespace {

template <int K, int U, int G, bool UNITS, typename V>
__global__ void __launch_bounds__(256)
    k_combine_bwd(const V *__restrict__ y, int64_t n_rows, const float *__restrict__ gates,
                  const int32_t *__restrict__ comb_row, int64_t N,
                  const int32_t *__restrict__ row_token, const uint8_t *__restrict__ row_kmask,
                  int64_t n_units, const int32_t *__restrict__ unit_count,
                  const V *__restrict__ g_out, int64_t Hv, V *__restrict__ g_y,
                  float *__restrict__ g_gates, int32_t *__restrict__ err) {
    constexpr int W = sizeof(V) / 4;   // 32-bit words (bf16 pairs) per chunk
    pdl_wait();
    pdl_trigger();
    if (UNITS && unit_count) n_units = min(n_units, (int64_t)max(__ldg(unit_count), 0));
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int flags = 0;
    for (int64_t u = gwarp; u < n_units; u += nwarps) {
        // lane j < K: slot j's row and gate (-1: slot not in this unit or no row)
        int rl = -1;
        float gl = 0.f;
        bool on = false;
        int64_t tok = u;
        if (lane < K) {
            on = true;
            if (UNITS) {
                tok = __ldg(row_token + u);
                on = (__ldg(row_kmask + u) >> lane) & 1;
                if (tok < 0 || tok >= N) {
                    if (on) flags |= COACT_EFLAG_ROW_RANGE;
                    on = false;
                }
            }
            if (on) {
                rl = __ldg(comb_row + tok * K + lane);
                gl = __ldg(gates + tok * K + lane);
                if (rl < -1 || (int64_t)rl >= n_rows) flags |= COACT_EFLAG_ROW_RANGE;
                if (rl < 0 || (int64_t)rl >= n_rows) rl = -1;
            }
        }
        // live slots compacted in ascending slot order; pos = this lane's place among them
        unsigned live = __ballot_sync(0xffffffffu, rl >= 0);
        const int m = __popc(live);
        const int pos = __popc(live & lanemask_lt());
        int64_t row[K];
        float g[K], dot[K];
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const int l = live ? __ffs(live) - 1 : 0;
            row[i] = __shfl_sync(0xffffffffu, rl, l);
            g[i] = __shfl_sync(0xffffffffu, gl, l);
            dot[i] = 0.0f;
            live &= live - 1;
        }
        const V *go_row = g_out + u * Hv;
        for (int64_t c0 = 0; c0 < Hv; c0 += 32 * U) {
            V vg[U];
#pragma unroll
            for (int q = 0; q < U; ++q) {
                const int64_t c = c0 + q * 32 + lane;
                if (c < Hv) vg[q] = ld_chunk<V>(go_row + c);
            }
#pragma unroll
            for (int i0 = 0; i0 < K; i0 += G) {
                if (i0 >= m) break;
                V vy[U][G];
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    const int64_t c = c0 + q * 32 + lane;
#pragma unroll
                    for (int gi = 0; gi < G; ++gi)
                        if (c < Hv && i0 + gi < K && i0 + gi < m)
                            vy[q][gi] = ld_chunk<V>(y + row[i0 + gi] * Hv + c);
                }
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    const int64_t c = c0 + q * 32 + lane;
                    if (c >= Hv) continue;
#pragma unroll
                    for (int gi = 0; gi < G; ++gi) {
                        const int i = i0 + gi;
                        if (i >= K || i >= m) continue;
                        V p;
#pragma unroll
                        for (int e = 0; e < W; ++e) {
                            const uint32_t wg = chunk_word(vg[q], e), w = chunk_word(vy[q][gi], e);
                            const float g0 = bf16lo(wg), g1 = bf16hi(wg);
                            dot[i] = __fmaf_rn(g0, bf16lo(w), dot[i]);
                            dot[i] = __fmaf_rn(g1, bf16hi(w), dot[i]);
                            const __nv_bfloat162 h2 =
                                __floats2bfloat162_rn(__fmul_rn(g[i], g0), __fmul_rn(g[i], g1));
                            set_chunk_word(p, e, *reinterpret_cast<const uint32_t *>(&h2));
                        }
                        st_chunk(g_y + row[i] * Hv + c, p);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < K; ++i) {
            if (i >= m) break;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot[i] += __shfl_xor_sync(0xffffffffu, dot[i], o);
        }
        // lane j writes slot j of this unit: its dot product, or 0 where it has no row
        float mine = 0.f;
#pragma unroll
        for (int i = 0; i < K; ++i)
            if (i == pos) mine = dot[i];
        if (on) g_gates[tok * K + lane] = rl >= 0 ? mine : 0.0f;
    }
    raise_flag_warp(err, flags);
}

template <int K, bool UNITS>
int launch(const uint16_t *y, int64_t n_rows, const float *gates, const int32_t *comb_row,
           int64_t N, const int32_t *row_token, const uint8_t *row_kmask, int64_t n_units,
           const int32_t *unit_count, const uint16_t *g_out, int64_t H, uint16_t *g_y,
           float *g_gates, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
    // loads in flight per lane: U chunks of grad_out + U x G rows of y (16-byte chunks);
    // one 32-byte chunk per row where y, grad_out and grad_y are 32-byte aligned
    constexpr int U = 2, G = 2;
#ifndef COACT_BWD_PER_SM
#define COACT_BWD_PER_SM 8
#endif
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(n_units, 8), (int64_t)di.sm_count * COACT_BWD_PER_SM));
    if (H % 16 == 0 && aligned32(y) && aligned32(g_out) && aligned32(g_y))
        return launch_pdl(k_combine_bwd<K, 1, G, UNITS, Row32>, blocks, 256, 0, st,
                          reinterpret_cast<const Row32 *>(y), n_rows, gates, comb_row, N,
                          row_token, row_kmask, n_units, unit_count,
                          reinterpret_cast<const Row32 *>(g_out), H / 16,
                          reinterpret_cast<Row32 *>(g_y), g_gates, err);
    return launch_pdl(k_combine_bwd<K, U, G, UNITS, uint4>, blocks, 256, 0, st,
                      reinterpret_cast<const uint4 *>(y), n_rows, gates, comb_row, N, row_token,
                      row_kmask, n_units, unit_count, reinterpret_cast<const uint4 *>(g_out), H / 8,
                      reinterpret_cast<uint4 *>(g_y), g_gates, err);
}

template <bool UNITS>
int dispatch_k(const uint16_t *y, int64_t n_rows, const float *gates, const int32_t *comb_row,
               int64_t N, int k, const int32_t *row_token, const uint8_t *row_kmask,
               int64_t n_units, const int32_t *unit_count, const uint16_t *g_out, int64_t H,
               uint16_t *g_y, float *g_gates, int32_t *err, cudaStream_t st,
               const DeviceInfo &di) {
#define COACT_BWD_CASE(KK)                                                                      \
    case KK:                                                                                    \
        return launch<KK, UNITS>(y, n_rows, gates, comb_row, N, row_token, row_kmask, n_units,  \
                                 unit_count, g_out, H, g_y, g_gates, err, st, di);
    switch (k) {
        COACT_BWD_CASE(1)
        COACT_BWD_CASE(2)
        COACT_BWD_CASE(3)
        COACT_BWD_CASE(4)
        COACT_BWD_CASE(5)
        COACT_BWD_CASE(6)
        COACT_BWD_CASE(7)
        COACT_BWD_CASE(8)
    }
#undef COACT_BWD_CASE
    return COACT_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int combine_scatter_backward(const uint16_t *y, int64_t n_rows, const float *gates,
                                        const int32_t *comb_row, int64_t N, int k,
                                        const int32_t *row_token, const uint8_t *row_kmask,
                                        int64_t n_units, const int32_t *unit_count,
                                        const uint16_t *grad_out, int64_t H,
                                        uint16_t *grad_y, float *grad_gates, int32_t *err_flag,
                                        coact_stream_t stream) {
    COACT_RANGE("combine_scatter_backward");
    if (N < 0 || H < 0 || n_rows < 0 || n_units < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (!row_token) n_units = N;
    if (n_units == 0 || H == 0) return COACT_OK;
    if (row_token && !row_kmask) return COACT_ERR_INVALID;
    if (!gates || !grad_out || !grad_gates || (N > 0 && !comb_row) ||
        (n_rows > 0 && (!y || !grad_y)))
        return COACT_ERR_INVALID;
    if ((y && !aligned16(y)) || !aligned16(grad_out) || (grad_y && !aligned16(grad_y)))
        return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (row_token)
        return dispatch_k<true>(y, n_rows, gates, comb_row, N, k, row_token, row_kmask, n_units,
                                unit_count, grad_out, H, grad_y, grad_gates, err_flag, st, di);
    return dispatch_k<false>(y, n_rows, gates, comb_row, N, k, nullptr, nullptr, N, nullptr,
                             grad_out, H, grad_y, grad_gates, err_flag, st, di);
}
