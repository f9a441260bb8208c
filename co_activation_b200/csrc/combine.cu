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
// The same kernel, over other index arrays, gives two more entry points:
//  * combine_rows -- units instead of tokens: unit u is token row_token[u] restricted to
//    the slots of row_kmask[u].  Over the plan's send rows this is the partial combine of
//    the pre-reduced reverse path (one row per (token, rank), summed where the experts ran).
//  * dispatch_gather_backward -- the transpose of the dispatch: comb_row := send_row
//    (-1 = no row) and unit weights, grad_x[t] = sum of grad_send over the token's send
//    rows.  fmaf(1, v, acc) rounds exactly like acc + v, so this is the fp32 add chain.
//
// k_combine_v16: one warp per token.  Each lane covers 16 hidden elements per 32-byte
// column chunk (one 256-bit access; 8 elements per 16-byte chunk where y or out is not
// 32-byte aligned) and keeps U chunks x K rows of loads in flight before the FMAs.  The K
// source rows are scattered over y (expanded receive order), the output row is written
// once with streaming stores.  HBM traffic: N*k*H*2 (y) + N*H*(2|4) (out) + N*k*8.
// Measured on B200 in the config-3 step (k = 8, 14 KB rows): 2,689 us with 16-byte
// chunks, 2,418 us with 32-byte chunks -- 7.0 TB/s, above the measured copy bandwidth
// because the combine's traffic is 89% reads.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace coact {
namespace {

// Unit u = token u with all K slots.  gates == nullptr: every weight is 1.  Chunks of
// type V: 16 bytes (uint4, 8 elements) or 32 bytes (Row32, 16 elements per lane, one
// 256-bit access) when y's rows and out are 32-byte aligned.
template <int K, int U, bool F32, typename V>
__global__ void __launch_bounds__(256)
    k_combine_v16(const V *__restrict__ y, int64_t n_rows, const float *__restrict__ gates,
                  const int32_t *__restrict__ comb_row, int64_t N, int64_t Hv,
                  void *__restrict__ out, int32_t *__restrict__ err) {
    constexpr int W = sizeof(V) / 4;   // 32-bit words (bf16 pairs) per chunk
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
            gl = gates ? __ldg(gates + t * K + lane) : 1.0f;
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
        for (int64_t c0 = 0; c0 < Hv; c0 += 32 * U) {
            V v[U][K];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
#pragma unroll
                for (int j = 0; j < K; ++j)
                    if (c < Hv && row[j] >= 0) v[u][j] = ld_chunk<V>(y + row[j] * Hv + c);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c >= Hv) continue;
                float acc[2 * W];
#pragma unroll
                for (int e = 0; e < 2 * W; ++e) acc[e] = 0.0f;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    if (row[j] < 0) continue;
#pragma unroll
                    for (int q = 0; q < W; ++q) {
                        const uint32_t w = chunk_word(v[u][j], q);
                        acc[2 * q] = __fmaf_rn(g[j], bf16lo(w), acc[2 * q]);
                        acc[2 * q + 1] = __fmaf_rn(g[j], bf16hi(w), acc[2 * q + 1]);
                    }
                }
                if (F32) {               // 2W floats: two chunks of V
                    V p0, p1;
#pragma unroll
                    for (int q = 0; q < W; ++q) {
                        set_chunk_word(p0, q, __float_as_uint(acc[q]));
                        set_chunk_word(p1, q, __float_as_uint(acc[W + q]));
                    }
                    V *o = reinterpret_cast<V *>(out) + (t * Hv + c) * 2;
                    st_chunk(o, p0);
                    st_chunk(o + 1, p1);
                } else {
                    V p;
#pragma unroll
                    for (int q = 0; q < W; ++q) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
                        set_chunk_word(p, q, *reinterpret_cast<const uint32_t *>(&h2));
                    }
                    st_chunk(reinterpret_cast<V *>(out) + t * Hv + c, p);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

// Sparse slots.  UNITS: unit u = (token row_token[u], the slots of row_kmask[u]) -- on the
// plan's send rows usually one or two of the K slots; otherwise unit u = token u, whose
// slots without a row (-1, e.g. send_row entries of a rank already seen) are absent.  The
// unit's live slots are compacted in ascending slot order with a warp ballot and streamed
// G rows at a time, U column chunks per lane (U*G loads in flight), accumulating in that
// order: the same fma chain as k_combine_v16, without registers and issue slots for
// absent slots.
// Three CTAs per SM (at most 85 registers): 79 for k = 6-8 without spills, against 128 (two
// CTAs per SM) unbounded.  Measured on B200, combine_rows + the transposed dispatch of the
// pre-reduced step: 65,536 tokens, k = 6: 1,011 + 542 -> 968 + 531 us; 131,072 tokens, k =
// 8: 3,531 + 1,516 -> 3,472 + 1,474 us; 16,384 tokens, k = 2: 50.9 -> 49.9 us.
template <int K, int U, int G, bool F32, bool UNITS, typename V>
__global__ void __launch_bounds__(256, 3)
    k_combine_units(const V *__restrict__ y, int64_t n_rows, const float *__restrict__ gates,
                    const int32_t *__restrict__ comb_row, int64_t N,
                    const int32_t *__restrict__ row_token, const uint8_t *__restrict__ row_kmask,
                    int64_t n_units, const int32_t *__restrict__ unit_count, int64_t Hv,
                    void *__restrict__ out, int32_t *__restrict__ err) {
    constexpr int W = sizeof(V) / 4;   // 32-bit words (bf16 pairs) per chunk
    pdl_wait();
    pdl_trigger();
    if (UNITS && unit_count) n_units = min(n_units, (int64_t)max(__ldg(unit_count), 0));
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int flags = 0;
    for (int64_t u = gwarp; u < n_units; u += nwarps) {
        int rl = -1;
        float gl = 0.f;
        if (lane < K) {
            int64_t tok = u;
            bool on = true;
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
                gl = gates ? __ldg(gates + tok * K + lane) : 1.0f;
                if (rl < -1 || (int64_t)rl >= n_rows) flags |= COACT_EFLAG_ROW_RANGE;
                if (rl < 0 || (int64_t)rl >= n_rows) rl = -1;
            }
        }
        unsigned live = __ballot_sync(0xffffffffu, rl >= 0);   // lanes >= K hold -1
        const int m = __popc(live);
        int64_t row[K];
        float g[K];
#pragma unroll
        for (int i = 0; i < K; ++i) {      // i-th live slot, ascending
            const int l = live ? __ffs(live) - 1 : 0;
            row[i] = __shfl_sync(0xffffffffu, rl, l);
            g[i] = __shfl_sync(0xffffffffu, gl, l);
            live &= live - 1;
        }
        for (int64_t c0 = 0; c0 < Hv; c0 += 32 * U) {
            float acc[U][2 * W];
#pragma unroll
            for (int q = 0; q < U; ++q)
#pragma unroll
                for (int e = 0; e < 2 * W; ++e) acc[q][e] = 0.0f;
#pragma unroll
            for (int i0 = 0; i0 < K; i0 += G) {
                if (i0 >= m) break;
                V v[U][G];
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    const int64_t c = c0 + q * 32 + lane;
#pragma unroll
                    for (int gi = 0; gi < G; ++gi)
                        if (c < Hv && i0 + gi < K && i0 + gi < m)
                            v[q][gi] = ld_chunk<V>(y + row[i0 + gi] * Hv + c);
                }
#pragma unroll
                for (int q = 0; q < U; ++q) {
#pragma unroll
                    for (int gi = 0; gi < G; ++gi) {
                        if (i0 + gi >= K || i0 + gi >= m) continue;
                        const float gg = g[i0 + gi];
#pragma unroll
                        for (int e = 0; e < W; ++e) {
                            const uint32_t w = chunk_word(v[q][gi], e);
                            acc[q][2 * e] = __fmaf_rn(gg, bf16lo(w), acc[q][2 * e]);
                            acc[q][2 * e + 1] = __fmaf_rn(gg, bf16hi(w), acc[q][2 * e + 1]);
                        }
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < U; ++q) {
                const int64_t c = c0 + q * 32 + lane;
                if (c >= Hv) continue;
                if (F32) {               // 2W floats: two chunks of V
                    V p0, p1;
#pragma unroll
                    for (int e = 0; e < W; ++e) {
                        set_chunk_word(p0, e, __float_as_uint(acc[q][e]));
                        set_chunk_word(p1, e, __float_as_uint(acc[q][W + e]));
                    }
                    V *o = reinterpret_cast<V *>(out) + (u * Hv + c) * 2;
                    st_chunk(o, p0);
                    st_chunk(o + 1, p1);
                } else {
                    V p;
#pragma unroll
                    for (int e = 0; e < W; ++e) {
                        const __nv_bfloat162 h2 =
                            __floats2bfloat162_rn(acc[q][2 * e], acc[q][2 * e + 1]);
                        set_chunk_word(p, e, *reinterpret_cast<const uint32_t *>(&h2));
                    }
                    st_chunk(reinterpret_cast<V *>(out) + u * Hv + c, p);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

template <int K, bool F32, bool UNITS, bool SPARSE>
int launch(const uint16_t *y, int64_t n_rows, const float *gates, const int32_t *comb_row,
           int64_t N, const int32_t *row_token, const uint8_t *row_kmask, int64_t n_units,
           const int32_t *unit_count, int64_t H, void *out, int32_t *err, cudaStream_t st,
           const DeviceInfo &di) {
    // column chunks per lane: 8 loads in flight for k <= 2 (U = 4), U = 2 chunks for
    // k >= 3 (6-16 loads).  Measured on B200: U = 2 made k = 6 6% faster and k = 8
    // 0.4% faster than U = 1, while U = 8 made k = 2 1.6% slower than U = 4.
#if defined(COACT_COMBINE_LOADS)
    constexpr int U = K >= COACT_COMBINE_LOADS ? 1 : COACT_COMBINE_LOADS / K;  // experiments
#else
    constexpr int U = K <= 2 ? 4 : 2;
#endif
    const int64_t H16 = H / 8;
#ifndef COACT_COMBINE_PER_SM
#define COACT_COMBINE_PER_SM 8  // CTAs per SM in the grid (0: one resident wave)
#endif
#ifndef COACT_COMBINE_PER_SM_K2
// k <= 2: one warp per token up to 128 CTAs per SM.  Measured on B200 in the step: config
// 4 (k = 2, 8 KB rows) both combines 495.7 -> 480.6 us, config 1 38.3 -> 37.4 us; over
// 14 KB rows the k = 1 combine 6.25 -> 6.75 TB/s.  For k >= 3 (one CTA of 184 registers
// resident per SM) finer grids were no faster.
#define COACT_COMBINE_PER_SM_K2 128
#endif
    constexpr int kPerSm = K <= 2 ? COACT_COMBINE_PER_SM_K2 : COACT_COMBINE_PER_SM;
#ifndef COACT_COMBINE_VEC
#define COACT_COMBINE_VEC 32  // 256-bit chunks where y and out are 32-byte aligned (16: never)
#endif
    const int blocks = grid_for(k_combine_v16<K, U, F32, uint4>, n_units, kPerSm, di);
    const bool wide = COACT_COMBINE_VEC == 32 && H % 16 == 0 && aligned32(y) && aligned32(out);
    if (UNITS || (SPARSE && K >= 3)) {   // sparse slots: units, or token rows with absent slots
#ifndef COACT_UNITS_PER_SM
#define COACT_UNITS_PER_SM COACT_COMBINE_PER_SM
#endif
        const int blocks = grid_for(k_combine_v16<K, U, F32, uint4>, n_units, COACT_UNITS_PER_SM, di);
        const int32_t *rt = UNITS ? row_token : nullptr;
        const uint8_t *km = UNITS ? row_kmask : nullptr;
        const int32_t *uc = UNITS ? unit_count : nullptr;
        // 32-byte chunks for k >= 3 (measured in the step: combine_rows 1,061 -> 1,009 us on
        // config 2, 3,633 -> 3,533 us on config 3); k <= 2 keeps 16-byte chunks (config 1's
        // combine_rows was not faster with 32-byte ones)
        if (wide && K >= 3)
            return launch_pdl(k_combine_units<K, 2, 2, F32, UNITS, Row32>, blocks, 256, 0, st,
                              reinterpret_cast<const Row32 *>(y), n_rows, gates, comb_row, N, rt,
                              km, n_units, uc, H / 16, out, err);
        return launch_pdl(k_combine_units<K, 4, 2, F32, UNITS, uint4>, blocks, 256, 0, st,
                          reinterpret_cast<const uint4 *>(y), n_rows, gates, comb_row, N, rt, km,
                          n_units, uc, H16, out, err);
    }
    if (wide) {
#if defined(COACT_COMBINE_LOADS)
        constexpr int UW = (U + 1) / 2;    // the same bytes in flight in 32-byte chunks
#else
        // 32-byte chunks per lane: two for k <= 2 and k >= 7, one for k = 3..6.  Measured on
        // B200 in the step: k = 8 (config 3) two chunks 2,418 us vs one 2,464 us; k = 2
        // (config 1) two chunks 38.0 us vs eight 51.0 us; k = 6 (config 2) one and three equal.
        constexpr int UW = (K <= 2 || K >= 7) ? 2 : 1;
#endif
        return launch_pdl(k_combine_v16<K, UW, F32, Row32>,
                          grid_for(k_combine_v16<K, UW, F32, Row32>, n_units, kPerSm, di),
                          256, 0, st, reinterpret_cast<const Row32 *>(y), n_rows, gates, comb_row,
                          N, H / 16, out, err);
    }
    return launch_pdl(k_combine_v16<K, U, F32, uint4>, blocks, 256, 0, st,
                      reinterpret_cast<const uint4 *>(y), n_rows, gates, comb_row, N, H16, out, err);
}

// k in 1..8 -> the K instantiation
template <bool UNITS, bool SPARSE>
int dispatch_k(const uint16_t *y, int64_t n_rows, const float *gates, const int32_t *comb_row,
               int64_t N, int k, const int32_t *row_token, const uint8_t *row_kmask,
               int64_t n_units, const int32_t *unit_count, int64_t H, void *out, int out_dtype,
               int32_t *err, cudaStream_t st, const DeviceInfo &di) {
#define COACT_COMBINE_CASE(KK)                                                                 \
    case KK:                                                                                   \
        return out_dtype ? launch<KK, true, UNITS, SPARSE>(y, n_rows, gates, comb_row, N, row_token,   \
                                                   row_kmask, n_units, unit_count, H, out, err, \
                                                   st, di)                                     \
                         : launch<KK, false, UNITS, SPARSE>(y, n_rows, gates, comb_row, N, row_token,  \
                                                    row_kmask, n_units, unit_count, H, out,    \
                                                    err, st, di);
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

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int combine_scatter(const uint16_t *y, int64_t n_rows, const float *gates,
                               const int32_t *comb_row, int64_t N, int k, int64_t H, void *out,
                               int out_dtype, int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("combine_scatter");
    if (N < 0 || H < 0 || n_rows < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || (out_dtype != 0 && out_dtype != 1)) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return COACT_OK;
    if (!gates || !comb_row || !out || (n_rows > 0 && !y)) return COACT_ERR_INVALID;
    if ((y && !aligned16(y)) || !aligned16(out)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    return dispatch_k<false, false>(y, n_rows, gates, comb_row, N, k, nullptr, nullptr, N, nullptr, H, out,
                             out_dtype, err_flag, reinterpret_cast<cudaStream_t>(stream), di);
}

extern "C" int combine_rows(const uint16_t *y, int64_t n_rows, const float *gates,
                            const int32_t *comb_row, int64_t N, int k, const int32_t *row_token,
                            const uint8_t *row_kmask, int64_t n_units, const int32_t *unit_count,
                            int64_t H, void *out, int out_dtype, int32_t *err_flag,
                            coact_stream_t stream) {
    COACT_RANGE("combine_rows");
    if (N < 0 || H < 0 || n_rows < 0 || n_units < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || (out_dtype != 0 && out_dtype != 1)) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (n_units == 0 || H == 0) return COACT_OK;
    if (!gates || !row_token || !row_kmask || !out || (N > 0 && !comb_row) || (n_rows > 0 && !y))
        return COACT_ERR_INVALID;
    if ((y && !aligned16(y)) || !aligned16(out)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    return dispatch_k<true, false>(y, n_rows, gates, comb_row, N, k, row_token, row_kmask, n_units,
                            unit_count, H, out, out_dtype, err_flag,
                            reinterpret_cast<cudaStream_t>(stream), di);
}

extern "C" int dispatch_gather_backward(const uint16_t *grad_send, int64_t n_rows,
                                        const int32_t *send_row, int64_t N, int k, int64_t H,
                                        void *grad_x, int out_dtype, int32_t *err_flag,
                                        coact_stream_t stream) {
    COACT_RANGE("dispatch_gather_backward");
    if (N < 0 || H < 0 || n_rows < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || (out_dtype != 0 && out_dtype != 1)) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return COACT_OK;
    if (!send_row || !grad_x || (n_rows > 0 && !grad_send)) return COACT_ERR_INVALID;
    if ((grad_send && !aligned16(grad_send)) || !aligned16(grad_x)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    return dispatch_k<false, true>(grad_send, n_rows, nullptr, send_row, N, k, nullptr, nullptr, N, nullptr,
                             H, grad_x, out_dtype, err_flag, reinterpret_cast<cudaStream_t>(stream),
                             di);
}
