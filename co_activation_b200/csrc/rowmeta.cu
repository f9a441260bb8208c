// plan_row_meta / gather_row_slots: the per-slot metadata that travels with the rows
// under expert parallelism, and the way back of one value per (send row, slot).
//
// Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English abstracts:
// under EP each token is sent to the ranks that hold its experts (with the deduplicated
// dispatcher each rank once), those ranks run the experts and the results go back to be
// combined.  A deduplicated row serves one or more of the token's k slots; the rank that
// receives it needs each served slot's expert id, its gate (for a combine or backward
// where the experts ran) and the position of its expert output in the rank's expanded
// receive order.  The plan fixes all three:
//   plan_row_meta, for d < min(row_capacity, rank_offsets[R]) and j < k, with
//   t = row_token[d] and r the rank whose segment holds d:
//     bit j of row_kmask[d] set:  experts[d,j] = ids[t,j], gates_out[d,j] = gates[t,j],
//                                 slots[d,j] = comb_row[t,j] + slot_base[r]
//     else                        -1, 0.0f, -1
//   gather_row_slots: out[t,j] = vals[d,j] for the send row d of token t that holds slot
//   j (d among the token's send_row entries), 0 where none does.
//
// k_row_meta: one thread per (row, slot), so every output array is written coalesced;
// the rank of a row is found by a binary search over rank_offsets staged in shared
// memory.  k_gather_row_slots: one thread per token (k <= 8 values), the token's send
// rows and their masks read once.  Both are latency-bound (a few bytes per slot).
#include <algorithm>

#include "common.cuh"

namespace coact {
namespace {

__global__ void __launch_bounds__(256)
    k_row_meta(const int32_t *__restrict__ row_token, const uint8_t *__restrict__ row_kmask,
               int64_t cap, const int32_t *__restrict__ rank_offsets, int R,
               const int32_t *__restrict__ ids, const float *__restrict__ gates,
               const int32_t *__restrict__ comb_row, int64_t N, int k,
               const int32_t *__restrict__ slot_base, int32_t *__restrict__ experts,
               float *__restrict__ gates_out, int32_t *__restrict__ slots,
               int32_t *__restrict__ err) {
    __shared__ int32_t s_off[COACT_MAX_R + 1];
    pdl_wait();
    pdl_trigger();
    for (int r = threadIdx.x; r <= R; r += blockDim.x) s_off[r] = __ldg(rank_offsets + r);
    __syncthreads();
    const int64_t n_rows = min(cap, (int64_t)max(s_off[R], 0));
    const int64_t total = n_rows * k;
    int flags = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t d = i / k;
        const int j = (int)(i - d * k);
        const int64_t t = __ldg(row_token + d);
        bool on = (__ldg(row_kmask + d) >> j) & 1;
        if (t < 0 || t >= N) {
            flags |= COACT_EFLAG_ROW_RANGE;
            on = false;
        }
        if (experts) experts[i] = on ? __ldg(ids + t * k + j) : -1;
        if (gates_out) gates_out[i] = on ? __ldg(gates + t * k + j) : 0.0f;
        if (slots) {
            int v = -1;
            if (on) {
                v = __ldg(comb_row + t * k + j);
                if (slot_base) {
                    // rank r: the last r with s_off[r] <= d (segments may be empty)
                    int lo = 0, hi = R - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if ((int64_t)s_off[mid] <= d) lo = mid;
                        else hi = mid - 1;
                    }
                    v += __ldg(slot_base + lo);
                }
            }
            slots[i] = v;
        }
    }
    raise_flag_warp(err, flags);
}

template <int K>
__global__ void __launch_bounds__(256)
    k_gather_row_slots(const float *__restrict__ vals, int64_t n_rows,
                       const int32_t *__restrict__ send_row, const uint8_t *__restrict__ row_kmask,
                       int64_t N, float *__restrict__ out, int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < N;
         t += (int64_t)gridDim.x * blockDim.x) {
        float v[K];
#pragma unroll
        for (int j = 0; j < K; ++j) v[j] = 0.0f;
#pragma unroll
        for (int j0 = 0; j0 < K; ++j0) {
            const int64_t d = __ldg(send_row + t * K + j0);
            if (d < 0) continue;
            if (d >= n_rows) {
                flags |= COACT_EFLAG_ROW_RANGE;
                continue;
            }
            const unsigned m = __ldg(row_kmask + d);
#pragma unroll
            for (int j = 0; j < K; ++j)
                if ((m >> j) & 1) v[j] = __ldg(vals + d * K + j);
        }
#pragma unroll
        for (int j = 0; j < K; ++j) out[t * K + j] = v[j];
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int plan_row_meta(const int32_t *row_token, const uint8_t *row_kmask,
                             int64_t row_capacity, const int32_t *rank_offsets, int R,
                             const int32_t *ids, const float *gates, const int32_t *comb_row,
                             int64_t N, int k, const int32_t *slot_base, int32_t *row_experts,
                             float *row_gates, int32_t *row_slots, int32_t *err_flag,
                             coact_stream_t stream) {
    COACT_RANGE("plan_row_meta");
    if (N < 0 || row_capacity < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || R < 1 || R > COACT_MAX_R) return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX / k || row_capacity > (int64_t)INT32_MAX / k)
        return COACT_ERR_UNSUPPORTED;
    if (!rank_offsets) return COACT_ERR_INVALID;
    if ((row_experts && !ids) || (row_gates && !gates) || (row_slots && !comb_row))
        return COACT_ERR_INVALID;
    if (row_capacity == 0 || (!row_experts && !row_gates && !row_slots)) return COACT_OK;
    if (!row_token || !row_kmask) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int blocks =
        (int)std::min<int64_t>(ceil_div(row_capacity * k, 256), (int64_t)di.sm_count * 8);
    return launch_pdl(k_row_meta, std::max(blocks, 1), 256, 0,
                      reinterpret_cast<cudaStream_t>(stream), row_token, row_kmask, row_capacity,
                      rank_offsets, R, ids, gates, comb_row, N, k, slot_base, row_experts,
                      row_gates, row_slots, err_flag);
}

extern "C" int gather_row_slots(const float *vals, int64_t n_rows, const int32_t *send_row,
                                const uint8_t *row_kmask, int64_t N, int k, float *out,
                                int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("gather_row_slots");
    if (N < 0 || n_rows < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K) return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX / k || n_rows > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    if (N == 0) return COACT_OK;
    if (!send_row || !out || (n_rows > 0 && (!vals || !row_kmask))) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int blocks = (int)std::min<int64_t>(ceil_div(N, 256), (int64_t)di.sm_count * 8);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_GRS_CASE(KK)                                                                      \
    case KK:                                                                                    \
        return launch_pdl(k_gather_row_slots<KK>, blocks, 256, 0, st, vals, n_rows, send_row, \
                          row_kmask, N, out, err_flag);
    switch (k) {
        COACT_GRS_CASE(1)
        COACT_GRS_CASE(2)
        COACT_GRS_CASE(3)
        COACT_GRS_CASE(4)
        COACT_GRS_CASE(5)
        COACT_GRS_CASE(6)
        COACT_GRS_CASE(7)
        COACT_GRS_CASE(8)
    }
#undef COACT_GRS_CASE
    return COACT_ERR_UNSUPPORTED;
}
