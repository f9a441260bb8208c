// coact_place_correlated: correlated expert placement from co-activation counts.
//
// Zyphra (arxivdaily 2610.09372), English abstract: correlated expert placement puts
// experts that are often selected together on the same GPU; together with the
// once-per-GPU dispatcher it removes dispatched rows.  Cobalt (arxivdaily 2609.36959),
// English abstract: frequently co-activated experts are co-located to cut cross-node
// traffic.  The pages give no algorithm; this is the plain greedy reading:
//   1. weight(a, b) = pair[a][b] + pair[b][a] for every a < b with weight > 0;
//   2. visit pairs by weight descending, ties by (a, b) ascending;
//   3. both experts unplaced -> the lowest rank with two free slots;
//      one placed and its rank has a free slot -> the other joins it;
//   4. experts still unplaced, ascending id -> the lowest rank with a free slot.
// Every rank ends with exactly E / R experts.  Host code: reads a host copy of the
// counts, writes a host array.
#include <algorithm>
#include <vector>

#include "common.cuh"

extern "C" int coact_place_correlated(const int64_t *pair, int E, int R, int32_t *expert_rank) {
    COACT_RANGE("coact_place_correlated");
    if (!pair || !expert_rank) return COACT_ERR_INVALID;
    if (E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R || E % R != 0)
        return COACT_ERR_UNSUPPORTED;
    const int slots = E / R;
    struct Edge {
        int64_t w;
        int a, b;
    };
    std::vector<Edge> edges;
    edges.reserve((size_t)E * (E - 1) / 2);
    for (int a = 0; a < E; ++a)
        for (int b = a + 1; b < E; ++b) {
            const int64_t w = pair[(int64_t)a * E + b] + pair[(int64_t)b * E + a];
            if (w > 0) edges.push_back({w, a, b});
        }
    std::sort(edges.begin(), edges.end(), [](const Edge &x, const Edge &y) {
        if (x.w != y.w) return x.w > y.w;
        if (x.a != y.a) return x.a < y.a;
        return x.b < y.b;
    });
    std::vector<int> rank_of(E, -1), free_slots(R, slots);
    for (const Edge &ed : edges) {
        const int ra = rank_of[ed.a], rb = rank_of[ed.b];
        if (ra < 0 && rb < 0) {
            for (int r = 0; r < R; ++r)
                if (free_slots[r] >= 2) {
                    rank_of[ed.a] = rank_of[ed.b] = r;
                    free_slots[r] -= 2;
                    break;
                }
        } else if (ra >= 0 && rb < 0) {
            if (free_slots[ra] > 0) {
                rank_of[ed.b] = ra;
                free_slots[ra] -= 1;
            }
        } else if (rb >= 0 && ra < 0) {
            if (free_slots[rb] > 0) {
                rank_of[ed.a] = rb;
                free_slots[rb] -= 1;
            }
        }
    }
    for (int e = 0; e < E; ++e) {
        if (rank_of[e] >= 0) continue;
        for (int r = 0; r < R; ++r)
            if (free_slots[r] > 0) {
                rank_of[e] = r;
                free_slots[r] -= 1;
                break;
            }
    }
    for (int e = 0; e < E; ++e) expert_rank[e] = rank_of[e];
    return COACT_OK;
}

// coact_rebalance_ranks: Cobalt's second planner stage.
//
// Cobalt (arxivdaily 2609.36959), English abstract: the planner periodically co-locates
// frequently co-activated experts on the same node, then "performs per-step intra-node
// adjustment to rebalance the workloads".  The pages give no algorithm; this is the plain
// longest-first greedy: within each node, its experts by load descending (ties: lower id)
// each go to the node's rank with the least load so far that still has a free slot (ties:
// lower rank).  Every rank ends with E/R experts; no expert changes node.
extern "C" int coact_rebalance_ranks(const int64_t *loads, const int32_t *expert_node, int E,
                                     const int32_t *rank_node, int R, int32_t *expert_rank) {
    COACT_RANGE("coact_rebalance_ranks");
    if (!loads || !expert_node || !rank_node || !expert_rank) return COACT_ERR_INVALID;
    if (E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R || E % R != 0)
        return COACT_ERR_UNSUPPORTED;
    const int slots = E / R;
    int n_nodes = 0;
    for (int r = 0; r < R; ++r) {
        if (rank_node[r] < 0 || rank_node[r] >= 64) return COACT_ERR_INVALID;
        n_nodes = std::max(n_nodes, rank_node[r] + 1);
    }
    std::vector<int> node_cap(n_nodes, 0), node_size(n_nodes, 0);
    for (int r = 0; r < R; ++r) node_cap[rank_node[r]] += slots;
    for (int e = 0; e < E; ++e) {
        if (expert_node[e] < 0 || expert_node[e] >= n_nodes) return COACT_ERR_INVALID;
        node_size[expert_node[e]] += 1;
    }
    for (int n = 0; n < n_nodes; ++n)
        if (node_size[n] != node_cap[n]) return COACT_ERR_INVALID;   // the node layout must fit
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return loads[a] > loads[b]; });
    std::vector<int64_t> rank_load(R, 0);
    std::vector<int> free_slots(R, slots);
    for (int e : order) {
        int best = -1;
        for (int r = 0; r < R; ++r) {
            if (rank_node[r] != expert_node[e] || free_slots[r] == 0) continue;
            if (best < 0 || rank_load[r] < rank_load[best]) best = r;
        }
        expert_rank[e] = best;
        rank_load[best] += loads[e];
        free_slots[best] -= 1;
    }
    return COACT_OK;
}

// coact_place_replicas: a replica layout from co-activation and workload statistics.
//
// Cobalt (arxivdaily 2609.36959), English abstract: EP distributes expert replicas across
// GPUs, and the layout planner follows co-activation and workload statistics.  The pages
// give no algorithm; the reading taken: an expert's load is shared equally by its
// replicas (in units of 1/840, exact for up to 8 replicas); `budget` times, the heaviest
// rank that holds a replicable expert (fewer than max_rep replicas, some rank without
// one) gives its heaviest such share a new replica, placed on a node that holds none
// of that expert yet (if any rank on such a node is left), choosing the node whose
// experts (by replica 0) are most co-activated with it, then that node's least loaded
// rank; ties go to the lower expert / node / rank.  Host code.
extern "C" int coact_place_replicas(const int64_t *pair, const int64_t *loads,
                                    const int32_t *expert_rank, int E, const int32_t *rank_node,
                                    int R, int budget, int max_rep, int32_t *rep_rank,
                                    int32_t *n_rep) {
    COACT_RANGE("coact_place_replicas");
    if (!pair || !loads || !expert_rank || !rank_node || !rep_rank || !n_rep)
        return COACT_ERR_INVALID;
    if (E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R || max_rep < 1 ||
        max_rep > COACT_MAX_REPLICAS || budget < 0)
        return COACT_ERR_UNSUPPORTED;
    int n_nodes = 0;
    for (int r = 0; r < R; ++r) {
        if (rank_node[r] < 0 || rank_node[r] >= 64) return COACT_ERR_INVALID;
        n_nodes = std::max(n_nodes, rank_node[r] + 1);
    }
    for (int e = 0; e < E; ++e)
        if (expert_rank[e] < 0 || expert_rank[e] >= R || loads[e] < 0) return COACT_ERR_INVALID;

    constexpr int64_t kUnit = 840;   // lcm(1..8): every replica's share is an integer
    std::vector<std::vector<int>> reps(E);
    std::vector<int64_t> rank_load(R, 0);
    for (int e = 0; e < E; ++e) {
        reps[e].push_back(expert_rank[e]);
        rank_load[expert_rank[e]] += loads[e] * kUnit;
    }
    auto share = [&](int e) { return loads[e] * kUnit / (int64_t)reps[e].size(); };
    int added = 0;
    auto replicable = [&](int e) {
        return (int)reps[e].size() < max_rep && (int)reps[e].size() < R;
    };
    while (added < budget) {
        // ranks by load (descending, ties lower rank): the first one holding a replicable
        // expert gives up its largest such share
        std::vector<int> by_load(R);
        for (int r = 0; r < R; ++r) by_load[r] = r;
        std::stable_sort(by_load.begin(), by_load.end(),
                         [&](int a, int b) { return rank_load[a] > rank_load[b]; });
        int pick = -1;
        for (int hot : by_load) {
            for (int e = 0; e < E; ++e) {
                if (!replicable(e)) continue;
                if (std::find(reps[e].begin(), reps[e].end(), hot) == reps[e].end()) continue;
                if (pick < 0 || share(e) > share(pick)) pick = e;
            }
            if (pick >= 0) break;
        }
        if (pick < 0) break;
        std::vector<char> rank_has(R, 0), node_has(n_nodes, 0);
        for (int r : reps[pick]) {
            rank_has[r] = 1;
            node_has[rank_node[r]] = 1;
        }
        bool fresh = false;
        for (int r = 0; r < R; ++r) fresh = fresh || (!rank_has[r] && !node_has[rank_node[r]]);
        std::vector<int64_t> affinity(n_nodes, 0);
        for (int f = 0; f < E; ++f)
            if (f != pick)
                affinity[rank_node[expert_rank[f]]] +=
                    pair[(int64_t)pick * E + f] + pair[(int64_t)f * E + pick];
        int node = -1;
        for (int n = 0; n < n_nodes; ++n) {
            if (fresh && node_has[n]) continue;
            bool room = false;
            for (int r = 0; r < R; ++r) room = room || (rank_node[r] == n && !rank_has[r]);
            if (room && (node < 0 || affinity[n] > affinity[node])) node = n;
        }
        if (node < 0) break;
        int target = -1;
        for (int r = 0; r < R; ++r)
            if (rank_node[r] == node && !rank_has[r] && (target < 0 || rank_load[r] < rank_load[target]))
                target = r;
        for (int r : reps[pick]) rank_load[r] -= share(pick);
        reps[pick].push_back(target);
        for (int r : reps[pick]) rank_load[r] += share(pick);
        ++added;
    }
    for (int e = 0; e < E; ++e) {
        n_rep[e] = (int32_t)reps[e].size();
        for (int i = 0; i < max_rep; ++i)
            rep_rank[(int64_t)e * max_rep + i] = i < (int)reps[e].size() ? reps[e][i] : -1;
    }
    return added;
}
