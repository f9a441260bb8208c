// Expert-parallel dispatch and combine across GPUs, through per-rank buffer tables.
//
// Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English abstracts:
// under expert parallelism every MoE layer exchanges tokens all-to-all to the GPUs that
// hold their experts and brings the results back to be combined; the deduplicated
// dispatcher sends each token to each GPU once.
//
// With one process per GPU (EP rank s holding its own tokens) the exchange is fused into
// the data movement: each source writes its rows directly into every destination rank's
// receive buffer (NVLink peer memory), and the combine reads the expert outputs directly
// from the destinations' output buffers.  Offsets come from the R x R count matrices the
// ranks exchange beforehand (C[s][r] rows, A[s][r] assignments): source s's rows start at
// sum_{s' < s} C[s'][r] in destination r's buffer, which makes every destination buffer
// exactly the rank-r segment the single-GPU plan would produce for all sources' tokens.
//  * k_gather_peer  -- dispatch_gather with the destination row mapped to
//                      (rank r, dst_off[r] + d - rank_offsets[r]) in bases[r]
//  * k_combine_peer -- combine_scatter with each assignment row mapped to
//                      (rank r, src_off[r] + a - asg_offsets[r]) in bases[r]; without
//                      gates (unit weights) over send_row / rank_offsets it is the
//                      transposed dispatch reading each row from its rank
// Plain loads and stores through generic pointers (no TMA multicast, no waits between
// ranks: ordering across GPUs is the caller's barrier).
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace coact {
namespace {

// Rank of a row in a segmented layout: the r with off[r] <= row < off[r+1] (R <= 64).
__device__ __forceinline__ int segment_of(const int *s_off, int R, int row) {
    int lo = 0, hi = R;  // off[lo] <= row < off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= row) lo = mid;
        else hi = mid;
    }
    return lo;
}

template <int UNROLL>
__global__ void __launch_bounds__(256)
    k_gather_peer(const uint4 *__restrict__ x, int64_t N, int64_t H16,
                  const int32_t *__restrict__ send_row, int k,
                  const int32_t *__restrict__ rank_offsets, int R,
                  const unsigned long long *__restrict__ bases,
                  const int32_t *__restrict__ dst_off, const int32_t *__restrict__ dst_cap,
                  int32_t *__restrict__ err) {
    __shared__ int s_off[COACT_MAX_R + 1];
    __shared__ int s_doff[COACT_MAX_R], s_dcap[COACT_MAX_R];
    __shared__ unsigned long long s_base[COACT_MAX_R];
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i <= R; i += blockDim.x) s_off[i] = __ldg(rank_offsets + i);
    for (int i = threadIdx.x; i < R; i += blockDim.x) {
        s_doff[i] = __ldg(dst_off + i);
        s_dcap[i] = __ldg(dst_cap + i);
        s_base[i] = __ldg(bases + i);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int D = s_off[R];
    int flags = 0;
    for (int64_t t = gwarp; t < N; t += nwarps) {
        // lane j < k resolves destination j: its rank buffer and row there
        unsigned long long dst = 0;
        bool has = false;
        if (lane < k) {
            const int d = __ldg(send_row + t * k + lane);
            if (d >= 0) {
                if (d >= D) {
                    flags |= COACT_EFLAG_ROW_RANGE;
                } else {
                    const int r = segment_of(s_off, R, d);
                    const int64_t row = (int64_t)s_doff[r] + (d - s_off[r]);
                    if (row >= s_dcap[r] || row < 0 || s_base[r] == 0) {
                        flags |= COACT_EFLAG_ROW_RANGE;
                    } else {
                        dst = s_base[r] + (unsigned long long)(row * H16) * sizeof(uint4);
                        has = true;
                    }
                }
            }
        }
        const unsigned dmask = __ballot_sync(0xffffffffu, has);
        const uint4 *src = x + t * H16;
        for (int64_t c0 = 0; c0 < H16; c0 += 32 * UNROLL) {
            uint4 v[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c < H16) v[u] = ld_stream(src + c);
            }
            unsigned m = dmask;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                uint4 *o = reinterpret_cast<uint4 *>(__shfl_sync(0xffffffffu, dst, j));
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int64_t c = c0 + u * 32 + lane;
                    if (c < H16) st_stream(o + c, v[u]);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

template <int K, int U, bool F32>
__global__ void __launch_bounds__(256)
    k_combine_peer(const unsigned long long *__restrict__ bases,
                   const int32_t *__restrict__ src_off, const int32_t *__restrict__ src_cap,
                   const int32_t *__restrict__ asg_offsets, int R,
                   const float *__restrict__ gates, const int32_t *__restrict__ comb_row,
                   int64_t N, int64_t H16, void *__restrict__ out, int32_t *__restrict__ err) {
    __shared__ int s_off[COACT_MAX_R + 1];
    __shared__ int s_soff[COACT_MAX_R], s_scap[COACT_MAX_R];
    __shared__ unsigned long long s_base[COACT_MAX_R];
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i <= R; i += blockDim.x) s_off[i] = __ldg(asg_offsets + i);
    for (int i = threadIdx.x; i < R; i += blockDim.x) {
        s_soff[i] = __ldg(src_off + i);
        s_scap[i] = __ldg(src_cap + i);
        s_base[i] = __ldg(bases + i);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int A = s_off[R];
    int flags = 0;
    for (int64_t t = gwarp; t < N; t += nwarps) {
        unsigned long long pl = 0;
        float gl = 0.f;
        if (lane < K) {
            const int a = __ldg(comb_row + t * K + lane);
            gl = gates ? __ldg(gates + t * K + lane) : 1.0f;
            if (a >= 0) {
                if (a >= A) {
                    flags |= COACT_EFLAG_ROW_RANGE;
                } else {
                    const int r = segment_of(s_off, R, a);
                    const int64_t row = (int64_t)s_soff[r] + (a - s_off[r]);
                    if (row >= s_scap[r] || row < 0 || s_base[r] == 0)
                        flags |= COACT_EFLAG_ROW_RANGE;
                    else
                        pl = s_base[r] + (unsigned long long)(row * H16) * sizeof(uint4);
                }
            } else if (a < -1) {
                flags |= COACT_EFLAG_ROW_RANGE;
            }
        }
        const uint4 *row[K];
        float g[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            row[j] = reinterpret_cast<const uint4 *>(__shfl_sync(0xffffffffu, pl, j));
            g[j] = __shfl_sync(0xffffffffu, gl, j);
        }
        for (int64_t c0 = 0; c0 < H16; c0 += 32 * U) {
            uint4 v[U][K];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
#pragma unroll
                for (int j = 0; j < K; ++j)
                    if (c < H16 && row[j]) v[u][j] = ld_stream(row[j] + c);
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
                    if (!row[j]) continue;
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

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int dispatch_gather_peer(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row,
                                    int k, const int32_t *rank_offsets, int R,
                                    const uint64_t *dst_bases, const int32_t *dst_row_offset,
                                    const int32_t *dst_capacity, int32_t *err_flag,
                                    coact_stream_t stream) {
    COACT_RANGE("dispatch_gather_peer");
    if (N < 0 || H < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || R < 1 || R > COACT_MAX_R) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return COACT_OK;
    if (!x || !send_row || !rank_offsets || !dst_bases || !dst_row_offset || !dst_capacity)
        return COACT_ERR_INVALID;
    if (!aligned16(x)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int64_t H16 = H / 8;
#ifndef COACT_PEER_PER_SM
// CTAs per SM in the peer gather's grid at most: one warp per token up to 128 per SM, as
// in dispatch_gather (tokens differ in fan-out).  Measured on B200 with every destination
// buffer in the GPU's own memory, one source holding a whole batch: 131,072 tokens, k = 8,
// 14 KB rows 2,693 -> 2,597 us; 65,536 tokens, k = 6, 8 KB rows 612 -> 587 us (8 per SM
// with a grid-stride loop before).
#define COACT_PEER_PER_SM 128
#endif
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(N, 8), (int64_t)di.sm_count * COACT_PEER_PER_SM));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    auto *b = reinterpret_cast<const unsigned long long *>(dst_bases);
    if (H16 <= 32)
        return launch_pdl(k_gather_peer<1>, blocks, 256, 0, st, xv, N, H16, send_row, k, rank_offsets,
                          R, b, dst_row_offset, dst_capacity, err_flag);
    if (H16 <= 128)
        return launch_pdl(k_gather_peer<4>, blocks, 256, 0, st, xv, N, H16, send_row, k, rank_offsets,
                          R, b, dst_row_offset, dst_capacity, err_flag);
    return launch_pdl(k_gather_peer<8>, blocks, 256, 0, st, xv, N, H16, send_row, k, rank_offsets, R,
                      b, dst_row_offset, dst_capacity, err_flag);
}

extern "C" int combine_scatter_peer(const uint64_t *y_bases, const int32_t *y_row_offset,
                                    const int32_t *y_capacity, const int32_t *asg_offsets, int R,
                                    const float *gates, const int32_t *comb_row, int64_t N, int k,
                                    int64_t H, void *out, int out_dtype, int32_t *err_flag,
                                    coact_stream_t stream) {
    COACT_RANGE("combine_scatter_peer");
    if (N < 0 || H < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || R < 1 || R > COACT_MAX_R || (out_dtype != 0 && out_dtype != 1))
        return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return COACT_OK;
    if (!y_bases || !y_row_offset || !y_capacity || !asg_offsets || !comb_row || !out)
        return COACT_ERR_INVALID;
    if (!aligned16(out)) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int64_t H16 = H / 8;
#ifndef COACT_PEER_COMBINE_PER_SM_K2
// CTAs per SM in the grid for k <= 2 (k >= 3: 8), as in combine_scatter.  Measured on B200
// with every rank's buffer in the GPU's own memory: 65,536 tokens, k = 2, 8 KB rows 253.3
// -> 247.4 us with 128 instead of 8; 16,384 tokens of 4 KB rows unchanged.
#define COACT_PEER_COMBINE_PER_SM_K2 128
#endif
    const int per_sm = k <= 2 ? COACT_PEER_COMBINE_PER_SM_K2 : 8;
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(N, 8), (int64_t)di.sm_count * per_sm));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto *b = reinterpret_cast<const unsigned long long *>(y_bases);
#define COACT_PEER_CASE(KK)                                                                        \
    case KK: {                                                                                     \
        constexpr int U = KK <= 2 ? 4 : 2;                                                         \
        return out_dtype ? launch_pdl(k_combine_peer<KK, U, true>, blocks, 256, 0, st, b,          \
                                      y_row_offset, y_capacity, asg_offsets, R, gates, comb_row,   \
                                      N, H16, out, err_flag)                                       \
                         : launch_pdl(k_combine_peer<KK, U, false>, blocks, 256, 0, st, b,         \
                                      y_row_offset, y_capacity, asg_offsets, R, gates, comb_row,   \
                                      N, H16, out, err_flag);                                      \
    }
    switch (k) {
        COACT_PEER_CASE(1)
        COACT_PEER_CASE(2)
        COACT_PEER_CASE(3)
        COACT_PEER_CASE(4)
        COACT_PEER_CASE(5)
        COACT_PEER_CASE(6)
        COACT_PEER_CASE(7)
        COACT_PEER_CASE(8)
    }
#undef COACT_PEER_CASE
    return COACT_ERR_UNSUPPORTED;
}
