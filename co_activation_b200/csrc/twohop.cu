// Two-hop dispatch: each token crosses to each destination NODE once, then is forwarded
// inside the node to each destination rank.
//
// Cobalt (arxivdaily 2609.36959), English abstract: communication-aware task assignment
// "routes tokens to fewer remote nodes".  Hop 1 is an ordinary plan_dispatch at node
// granularity (expert -> node map, home node); hop 2 reuses the rank-level plan.  This
// file adds the pieces that connect them:
//  * coact_compose_map  out[i] = b[a[i]] (e.g. expert -> rank -> node, token -> home
//                       rank -> home node)
//  * plan_forward       fwd_src[d] = the hop-1 (node-level) row that feeds rank-level
//                       row d, -1 past D
//  * forward_gather     dst[d] = src[fwd_src[d]]: the intra-node forward of hop 2
//  * forward_gather_tokens  the same rows, token-major: a token's rank rows are grouped
//                       by their hop-1 row, each hop-1 row is read once and written to
//                       every rank row it feeds (reads Dn rows instead of D)
#include <algorithm>

#include "common.cuh"

namespace coact {
namespace {

__global__ void __launch_bounds__(256)
    k_compose_map(const int32_t *__restrict__ a, int64_t n, const int32_t *__restrict__ b,
                  int64_t nb, int32_t *__restrict__ out, int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) {
        const int32_t v = __ldg(a + i);
        if (v < 0 || (int64_t)v >= nb) {
            flags |= COACT_EFLAG_ID_RANGE;
            out[i] = -1;
        } else {
            out[i] = __ldg(b + v);
        }
    }
    if (flags && err) atomicOr(err, flags);
}

// Blocks [0, token_blocks): one thread per token; for every rank-level send row of the
// token, the node-level row of (token, node of that rank) -- the node plan's send row at
// the token's first slot on that node.  Blocks after that: fwd_src = -1 on rows
// [D, row_capacity), D = rank_offsets[R].
template <int K>
__global__ void __launch_bounds__(256)
    k_plan_forward(const int32_t *__restrict__ ids, int64_t N, int E,
                   const int32_t *__restrict__ expert_rank, int R,
                   const int32_t *__restrict__ rank_node, int n_nodes,
                   const int32_t *__restrict__ send_row, const int32_t *__restrict__ rank_offsets,
                   const int32_t *__restrict__ node_send_row, int32_t *__restrict__ fwd_src,
                   int64_t cap, int token_blocks, int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    if ((int)blockIdx.x < token_blocks) {
        const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
        if (t < N) {
            int e[K];
            const int f = load_ids<K>(ids, t, E, e);
            if (!f) {
                int nd[K];
                bool ok = true;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int r = __ldg(expert_rank + e[j]);
                    if ((unsigned)r >= (unsigned)R) {
                        ok = false;
                        nd[j] = 0;
                        continue;
                    }
                    nd[j] = rank_node ? __ldg(rank_node + r) : 0;
                    if ((unsigned)nd[j] >= (unsigned)n_nodes) ok = false;
                }
                if (ok) {
#pragma unroll
                    for (int j = 0; j < K; ++j) {
                        const int d = __ldg(send_row + t * K + j);
                        if (d < 0) continue;
                        if ((int64_t)d >= cap) {
                            flags |= COACT_EFLAG_ROW_RANGE;
                            continue;
                        }
                        int first = j;
#pragma unroll
                        for (int jj = K - 1; jj >= 0; --jj)
                            if (jj < j && nd[jj] == nd[j]) first = jj;
                        fwd_src[d] = __ldg(node_send_row + t * K + first);
                    }
                } else {
                    flags |= COACT_EFLAG_ID_RANGE;
                }
            }
        }
    } else {
        const int64_t D = __ldg(rank_offsets + R);
        const int64_t stride = (int64_t)(gridDim.x - token_blocks) * blockDim.x;
        for (int64_t d = D + (int64_t)(blockIdx.x - token_blocks) * blockDim.x + threadIdx.x;
             d < cap; d += stride)
            fwd_src[d] = -1;
    }
    if (flags && err) atomicOr(err, flags);
}

// One warp per destination row, 16-byte vectors, UNROLL loads in flight per lane.
template <int UNROLL>
__global__ void __launch_bounds__(256)
    k_forward_gather(const uint4 *__restrict__ src, int64_t n_src, int64_t H16,
                     const int32_t *__restrict__ fwd_src, int64_t n_rows, uint4 *__restrict__ dst,
                     int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int flags = 0;
    for (int64_t d = gwarp; d < n_rows; d += nwarps) {
        const int s = __ldg(fwd_src + d);
        if (s < 0) continue;
        if ((int64_t)s >= n_src) {
            flags |= COACT_EFLAG_ROW_RANGE;
            continue;
        }
        const uint4 *in = src + (int64_t)s * H16;
        uint4 *o = dst + d * H16;
        for (int64_t c0 = 0; c0 < H16; c0 += 32 * UNROLL) {
            uint4 v[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c < H16) v[u] = ld_stream(in + c);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c < H16) st_stream(o + c, v[u]);
            }
        }
    }
    raise_flag_warp(err, flags);
}

// Token-major forward: one warp per token.  Lane j < K holds the token's rank row
// d_j = send_row[t, j] (first slot of each rank) and its hop-1 row s_j = fwd_src[d_j];
// lanes with the same s_j form a group (warp ballots), the group's source row is read
// once (UNROLL chunk loads per lane in flight) and stored to each of its rank rows.
// Rows of more than 2 KB take four 32-byte chunks per lane where src and dst are 32-byte
// aligned and H % 16 == 0 (measured on B200, hop 2 of config 3 with the two-stage
// layout: 2,547 us with eight 16-byte chunks, 2,518 us with four 32-byte ones, 2,686 us
// with two), else eight 16-byte chunks.
template <int K, int UNROLL, typename V>
__global__ void __launch_bounds__(256)
    k_forward_tokens(const V *__restrict__ src, int64_t n_src, int64_t Hv,
                     const int32_t *__restrict__ send_row, int64_t N,
                     const int32_t *__restrict__ fwd_src, int64_t n_rows, V *__restrict__ dst,
                     int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int flags = 0;
    for (int64_t t = gwarp; t < N; t += nwarps) {
        int d = -1, sr = -1;
        if (lane < K) {
            d = __ldg(send_row + t * K + lane);
            if (d >= 0) {
                if ((int64_t)d >= n_rows) {
                    flags |= COACT_EFLAG_ROW_RANGE;
                    d = -1;
                } else {
                    sr = __ldg(fwd_src + d);
                    if ((int64_t)sr >= n_src) {
                        flags |= COACT_EFLAG_ROW_RANGE;
                        sr = -1;
                    }
                    if (sr < 0) d = -1;
                }
            } else if (d < -1) {
                flags |= COACT_EFLAG_ROW_RANGE;
                d = -1;
            }
        }
        unsigned pending = __ballot_sync(0xffffffffu, d >= 0);
        while (pending) {
            const int s0 = __shfl_sync(0xffffffffu, sr, __ffs(pending) - 1);
            const unsigned grp = __ballot_sync(0xffffffffu, d >= 0 && sr == s0) & pending;
            pending &= ~grp;
            const int m = __popc(grp);
            int64_t drow[K];
            unsigned g = grp;
#pragma unroll
            for (int i = 0; i < K; ++i) {
                const int l = g ? __ffs(g) - 1 : 0;
                drow[i] = __shfl_sync(0xffffffffu, d, l);
                g &= g - 1;
            }
            const V *in = src + (int64_t)s0 * Hv;
            for (int64_t c0 = 0; c0 < Hv; c0 += 32 * UNROLL) {
                V v[UNROLL];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int64_t c = c0 + u * 32 + lane;
                    if (c < Hv) v[u] = ld_chunk<V>(in + c);
                }
#pragma unroll
                for (int i = 0; i < K; ++i) {
                    if (i >= m) break;
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u) {
                        const int64_t c = c0 + u * 32 + lane;
                        if (c < Hv) st_chunk(dst + drow[i] * Hv + c, v[u]);
                    }
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int coact_compose_map(const int32_t *a, int64_t n, const int32_t *b, int64_t nb,
                                 int32_t *out, int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("coact_compose_map");
    if (n < 0 || nb < 0) return COACT_ERR_INVALID;
    if (n == 0) return COACT_OK;
    if (!a || !b || !out) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int blocks = (int)std::min<int64_t>(ceil_div(n, 256), (int64_t)di.sm_count * 8);
    return launch_pdl(k_compose_map, blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream), a, n,
                      b, nb, out, err_flag);
}

extern "C" int plan_forward(const int32_t *ids, int64_t N, int k, int E, const int32_t *expert_rank,
                            int R, const int32_t *rank_node, int n_nodes, const int32_t *send_row,
                            const int32_t *rank_offsets, const int32_t *node_send_row,
                            int32_t *fwd_src, int64_t row_capacity, int32_t *err_flag,
                            coact_stream_t stream) {
    COACT_RANGE("plan_forward");
    if (N < 0 || row_capacity < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R)
        return COACT_ERR_UNSUPPORTED;
    if (rank_node && (n_nodes < 1 || n_nodes > 64)) return COACT_ERR_UNSUPPORTED;
    if (!rank_node) n_nodes = 1;
    if (N > (int64_t)INT32_MAX / k || row_capacity > (int64_t)INT32_MAX) return COACT_ERR_UNSUPPORTED;
    if (!expert_rank || !rank_offsets) return COACT_ERR_INVALID;
    if (N > 0 && (!ids || !send_row || !node_send_row)) return COACT_ERR_INVALID;
    if (row_capacity > 0 && !fwd_src) return COACT_ERR_INVALID;
    if (N == 0 && row_capacity == 0) return COACT_OK;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int token_blocks = (int)ceil_div(N, 256);
    const int fill_blocks =
        (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(row_capacity, 256), di.sm_count * 4));
    const int blocks = token_blocks + fill_blocks;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_FWD_CASE(KK)                                                                        \
    case KK:                                                                                      \
        return launch_pdl(k_plan_forward<KK>, blocks, 256, 0, st, ids, N, E, expert_rank, R,       \
                          rank_node, n_nodes, send_row, rank_offsets, node_send_row, fwd_src,     \
                          row_capacity, token_blocks, err_flag);
    switch (k) {
        COACT_FWD_CASE(1)
        COACT_FWD_CASE(2)
        COACT_FWD_CASE(3)
        COACT_FWD_CASE(4)
        COACT_FWD_CASE(5)
        COACT_FWD_CASE(6)
        COACT_FWD_CASE(7)
        COACT_FWD_CASE(8)
    }
#undef COACT_FWD_CASE
    return COACT_ERR_UNSUPPORTED;
}

extern "C" int forward_gather(const uint16_t *src, int64_t n_src_rows, int64_t H,
                              const int32_t *fwd_src, int64_t n_rows, uint16_t *dst,
                              int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("forward_gather");
    if (n_src_rows < 0 || H < 0 || n_rows < 0) return COACT_ERR_INVALID;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (n_rows == 0 || H == 0) return COACT_OK;
    if (!fwd_src || !dst || (n_src_rows > 0 && !src)) return COACT_ERR_INVALID;
    if ((src && !aligned16(src)) || !aligned16(dst)) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int64_t H16 = H / 8;
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(n_rows, 8), (int64_t)di.sm_count * 8));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *sv = reinterpret_cast<const uint4 *>(src);
    uint4 *dv = reinterpret_cast<uint4 *>(dst);
    if (H16 <= 32)
        return launch_pdl(k_forward_gather<1>, blocks, 256, 0, st, sv, n_src_rows, H16, fwd_src,
                          n_rows, dv, err_flag);
    if (H16 <= 128)
        return launch_pdl(k_forward_gather<4>, blocks, 256, 0, st, sv, n_src_rows, H16, fwd_src,
                          n_rows, dv, err_flag);
    return launch_pdl(k_forward_gather<8>, blocks, 256, 0, st, sv, n_src_rows, H16, fwd_src, n_rows,
                      dv, err_flag);
}

extern "C" int forward_gather_tokens(const uint16_t *src, int64_t n_src_rows, int64_t H,
                                     const int32_t *send_row, int64_t N, int k,
                                     const int32_t *fwd_src, int64_t n_rows, uint16_t *dst,
                                     int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("forward_gather_tokens");
    if (n_src_rows < 0 || H < 0 || n_rows < 0 || N < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || n_rows == 0 || H == 0) return COACT_OK;
    if (!send_row || !fwd_src || !dst || (n_src_rows > 0 && !src)) return COACT_ERR_INVALID;
    if ((src && !aligned16(src)) || !aligned16(dst)) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int64_t H16 = H / 8;
#ifndef COACT_FWD_PER_SM
// CTAs per SM in the grid at most: one warp per token up to 128 per SM.  Tokens forward
// to different numbers of rank rows, and one token per warp balances them to the end
// (measured on B200, hop 2 of 131,072 tokens with k = 8, 14 KB rows, two-stage layout:
// 2,488 us with 8 CTAs per SM and a grid-stride loop, 2,408 with 32, 2,377 with 128).
#define COACT_FWD_PER_SM 128
#endif
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(N, 8), (int64_t)di.sm_count * COACT_FWD_PER_SM));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint4 *sv = reinterpret_cast<const uint4 *>(src);
    uint4 *dv = reinterpret_cast<uint4 *>(dst);
#define COACT_FWT_CASE(KK)                                                                        \
    case KK:                                                                                      \
        if (H16 <= 32)                                                                            \
            return launch_pdl(k_forward_tokens<KK, 1, uint4>, blocks, 256, 0, st, sv, n_src_rows, H16,   \
                              send_row, N, fwd_src, n_rows, dv, err_flag);                        \
        if (H16 <= 128)                                                                           \
            return launch_pdl(k_forward_tokens<KK, 4, uint4>, blocks, 256, 0, st, sv, n_src_rows, H16,   \
                              send_row, N, fwd_src, n_rows, dv, err_flag);                        \
        if (H % 16 == 0 && aligned32(src) && aligned32(dst))                                     \
            return launch_pdl(k_forward_tokens<KK, 4, Row32>, blocks, 256, 0, st,                 \
                              reinterpret_cast<const Row32 *>(src), n_src_rows, H / 16, send_row, \
                              N, fwd_src, n_rows, reinterpret_cast<Row32 *>(dst), err_flag);      \
        return launch_pdl(k_forward_tokens<KK, 8, uint4>, blocks, 256, 0, st, sv, n_src_rows, H16, \
                          send_row, N, fwd_src, n_rows, dv, err_flag);
    switch (k) {
        COACT_FWT_CASE(1)
        COACT_FWT_CASE(2)
        COACT_FWT_CASE(3)
        COACT_FWT_CASE(4)
        COACT_FWT_CASE(5)
        COACT_FWT_CASE(6)
        COACT_FWT_CASE(7)
        COACT_FWT_CASE(8)
    }
#undef COACT_FWT_CASE
    return COACT_ERR_UNSUPPORTED;
}
