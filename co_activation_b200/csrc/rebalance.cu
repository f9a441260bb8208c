// rebalance_ranks: Cobalt's per-step intra-node adjustment, on the device.
//
// Cobalt (arxivdaily 2609.36959), English abstract: the planner periodically co-locates
// frequently co-activated experts on the same node and "performs per-step intra-node
// adjustment to rebalance the workloads".  The pages give no algorithm; the reading is
// the plain longest-first greedy (the same as the host planner coact_rebalance_ranks):
// within each node, the node's experts by load descending (ties: lower id) each go to
// the node's rank with the least load so far that still has one of its E/R slots free
// (ties: lower rank).  No expert changes node.
//
// Per step the loads come from coact_count (device int64 [E]) and the result feeds
// plan_dispatch (device int32 [E]); doing the greedy here keeps the step on the GPU, with
// no device -> host copy of the loads and no host synchronisation.
//
// k_rebalance: one CTA.  The experts' order by (load desc, id asc) is computed in shared
// memory by counting, for each expert, the experts ahead of it (E^2 comparisons spread
// over the CTA).  Each warp then runs the greedy of one node: it walks the order in
// chunks of 32, compacts the node's experts with a ballot, and assigns them one by one,
// each to the (load, rank)-smallest rank with a free slot found by a warp reduction over
// the node's ranks (rank r held by lane r % 32).  Latency-bound: E <= 1024 experts.
#include <climits>

#include "common.cuh"

namespace coact {
namespace {

__global__ void __launch_bounds__(1024)
    k_rebalance(const int64_t *__restrict__ loads, const int32_t *__restrict__ expert_node, int E,
                const int32_t *__restrict__ rank_node, int R, int n_nodes,
                int32_t *__restrict__ expert_rank, int32_t *__restrict__ err) {
    __shared__ int64_t s_load[COACT_MAX_E];
    __shared__ int32_t s_enode[COACT_MAX_E];
    __shared__ int32_t s_order[COACT_MAX_E];
    __shared__ int32_t s_rnode[COACT_MAX_R];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    int flags = 0;
    for (int e = tid; e < E; e += blockDim.x) {
        s_load[e] = __ldg(loads + e);
        int n = __ldg(expert_node + e);
        if (n < 0 || n >= n_nodes) {        // no node of this layout: no rank either
            flags |= COACT_EFLAG_ID_RANGE;
            expert_rank[e] = -1;
            n = -1;
        }
        s_enode[e] = n;
    }
    for (int r = tid; r < R; r += blockDim.x) {
        int n = __ldg(rank_node + r);
        if (n < 0 || n >= n_nodes) {
            flags |= COACT_EFLAG_ID_RANGE;
            n = -1;
        }
        s_rnode[r] = n;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        const int64_t le = s_load[e];
        int pos = 0;
        for (int c = 0; c < E; ++c) {
            const int64_t lc = s_load[c];
            pos += (lc > le) || (lc == le && c < e);
        }
        s_order[pos] = e;
    }
    __syncthreads();
    const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int slots = E / R;
    for (int n = warp; n < n_nodes; n += nwarps) {
        const bool in0 = lane < R && s_rnode[lane] == n;
        const bool in1 = lane + 32 < R && s_rnode[lane + 32] == n;
        int64_t ld0 = 0, ld1 = 0;
        int fr0 = in0 ? slots : 0, fr1 = in1 ? slots : 0;
        for (int base = 0; base < E; base += 32) {
            const int i = base + lane;
            const int e = i < E ? s_order[i] : -1;
            unsigned m = __ballot_sync(0xffffffffu, e >= 0 && s_enode[e] == n);
            while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1;
                const int ee = __shfl_sync(0xffffffffu, e, src);
                int64_t bl = LLONG_MAX;
                int br = INT_MAX;
                if (fr0 > 0) {
                    bl = ld0;
                    br = lane;
                }
                if (fr1 > 0 && ld1 < bl) {
                    bl = ld1;
                    br = lane + 32;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const int64_t ol = __shfl_xor_sync(0xffffffffu, bl, o);
                    const int orr = __shfl_xor_sync(0xffffffffu, br, o);
                    if (ol < bl || (ol == bl && orr < br)) {
                        bl = ol;
                        br = orr;
                    }
                }
                if (br == INT_MAX) {                 // the node has no free slot left
                    flags |= COACT_EFLAG_ID_RANGE;
                    if (lane == 0) expert_rank[ee] = -1;
                    continue;
                }
                if (lane == 0) expert_rank[ee] = br;
                if (br == lane) {
                    ld0 += s_load[ee];
                    --fr0;
                } else if (br == lane + 32) {
                    ld1 += s_load[ee];
                    --fr1;
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int rebalance_ranks(const int64_t *loads, const int32_t *expert_node, int E,
                               const int32_t *rank_node, int R, int n_nodes, int32_t *expert_rank,
                               int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("rebalance_ranks");
    if (!loads || !expert_node || !rank_node || !expert_rank) return COACT_ERR_INVALID;
    if (E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R || E % R != 0 || n_nodes < 1 ||
        n_nodes > 64)
        return COACT_ERR_UNSUPPORTED;
    return launch_pdl(k_rebalance, 1, 1024, 0, reinterpret_cast<cudaStream_t>(stream), loads,
                      expert_node, E, rank_node, R, n_nodes, expert_rank, err_flag);
}
