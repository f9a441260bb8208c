// assign_replicas: the replica each (token, slot) is served by.
//
// Cobalt (arxivdaily 2609.36959), English abstract: EP distributes expert replicas
// across GPUs, and a communication-aware task assignment routes tokens to fewer remote
// nodes under the current expert layout.  Per token t (home rank s, home node hn):
// slots whose expert has a single replica take it; the other slots, j ascending, take
// the first replica (ascending index) in the first non-empty class
//   (a) on s, (b) on a rank the token already uses, (c) on hn, (d) on a node the token
//   already uses,
// otherwise replica (t + j) mod n_rep[e], spreading the tokens that must open a new node.
// The result feeds plan_dispatch_slots.
//
// k_assign_replicas: one thread per token; the rank -> node table in shared memory, the
// token's used ranks and nodes as 64-bit masks.
#include <algorithm>

#include "common.cuh"

namespace coact {
namespace {

template <int K>
__global__ void __launch_bounds__(256)
    k_assign_replicas(const int32_t *__restrict__ ids, int64_t N, int E,
                      const int32_t *__restrict__ rep_rank, int max_rep,
                      const int32_t *__restrict__ n_rep, int R,
                      const int32_t *__restrict__ rank_node, int n_nodes,
                      const int32_t *__restrict__ src_rank, int32_t *__restrict__ slot_rank,
                      int32_t *__restrict__ err) {
    __shared__ int s_node[COACT_MAX_R];
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        int nd = rank_node ? __ldg(rank_node + r) : 0;
        if (nd < 0 || nd >= n_nodes) {
            if (blockIdx.x == 0) flags |= COACT_EFLAG_ID_RANGE;
            nd = 0;
        }
        s_node[r] = nd;
    }
    __syncthreads();
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t < N) {
        int e[K];
        int f = load_ids<K>(ids, t, E, e);
        const int s = src_rank ? __ldg(src_rank + t) : (int)((t * R) / N);
        if ((unsigned)s >= (unsigned)R) f |= COACT_EFLAG_SRC_RANK;
        int nrep[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            nrep[j] = 1;
            if (f & COACT_EFLAG_ID_RANGE) continue;
            nrep[j] = __ldg(n_rep + e[j]);
            if (nrep[j] < 1 || nrep[j] > max_rep) {
                f |= COACT_EFLAG_ID_RANGE;
                nrep[j] = 1;
                continue;
            }
            for (int i = 0; i < nrep[j]; ++i) {
                const int r = __ldg(rep_rank + (int64_t)e[j] * max_rep + i);
                if ((unsigned)r >= (unsigned)R) f |= COACT_EFLAG_ID_RANGE;
            }
        }
        int out[K];
#pragma unroll
        for (int j = 0; j < K; ++j) out[j] = -1;
        if (!f) {
            const int hn = s_node[s];
            unsigned long long used_rank = 0, used_node = 0;
#pragma unroll
            for (int j = 0; j < K; ++j)            // single replicas first
                if (nrep[j] == 1) {
                    const int r = __ldg(rep_rank + (int64_t)e[j] * max_rep);
                    out[j] = r;
                    used_rank |= 1ull << r;
                    used_node |= 1ull << s_node[r];
                }
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (out[j] >= 0) continue;
                const int32_t *rep = rep_rank + (int64_t)e[j] * max_rep;
                // best class over the replicas (0..3, 4 = none), first replica within it
                int best = 4, pick = -1;
                for (int i = 0; i < nrep[j]; ++i) {
                    const int r = __ldg(rep + i);
                    const int nd = s_node[r];
                    const int cls = r == s ? 0
                                    : ((used_rank >> r) & 1) ? 1
                                    : nd == hn ? 2
                                    : ((used_node >> nd) & 1) ? 3 : 4;
                    if (cls < best) {
                        best = cls;
                        pick = i;
                    }
                }
                if (best == 4) pick = (int)((t + j) % nrep[j]);
                const int r = __ldg(rep + pick);
                out[j] = r;
                used_rank |= 1ull << r;
                used_node |= 1ull << s_node[r];
            }
        }
        flags |= f;
#pragma unroll
        for (int j = 0; j < K; ++j) slot_rank[t * K + j] = out[j];
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int assign_replicas(const int32_t *ids, int64_t N, int k, int E, const int32_t *rep_rank,
                               int max_rep, const int32_t *n_rep, int R, const int32_t *rank_node,
                               int n_nodes, const int32_t *src_rank, int32_t *slot_rank,
                               int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("assign_replicas");
    if (N < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R ||
        max_rep < 1 || max_rep > COACT_MAX_REPLICAS)
        return COACT_ERR_UNSUPPORTED;
    if (rank_node && (n_nodes < 1 || n_nodes > 64)) return COACT_ERR_UNSUPPORTED;
    if (!rank_node) n_nodes = 1;
    if (N > (int64_t)INT32_MAX / k) return COACT_ERR_UNSUPPORTED;
    if (N == 0) return COACT_OK;
    if (!ids || !rep_rank || !n_rep || !slot_rank) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int blocks = (int)ceil_div(N, 256);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_REP_CASE(KK)                                                                        \
    case KK:                                                                                      \
        return launch_pdl(k_assign_replicas<KK>, blocks, 256, 0, st, ids, N, E, rep_rank, max_rep, \
                          n_rep, R, rank_node, n_nodes, src_rank, slot_rank, err_flag);
    switch (k) {
        COACT_REP_CASE(1)
        COACT_REP_CASE(2)
        COACT_REP_CASE(3)
        COACT_REP_CASE(4)
        COACT_REP_CASE(5)
        COACT_REP_CASE(6)
        COACT_REP_CASE(7)
        COACT_REP_CASE(8)
    }
#undef COACT_REP_CASE
    return COACT_ERR_UNSUPPORTED;
}
