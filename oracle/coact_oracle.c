/*
 * coact_oracle.c -- plain, slow, single-threaded CPU oracle for the co-activation
 * dispatch/combine path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Every function is the plain definition of what the method computes, written as
 * straight loops, with no blocking, fusion or reordering.  Sources (web pages):
 *   [Cobalt]  "Cobalt: efficient distributed MoE training using expert co-activation"
 *             (arxivdaily 2609.36959), English abstract: expert pairs co-activated by
 *             single tokens; per-expert workload statistics; routing tokens to fewer
 *             remote nodes; all-to-all token exchange under EP.
 *   [Zyphra]  correlated expert placement / token shuffling (arxivdaily 2610.09372),
 *             English abstract: "a dispatcher that sends each token to each GPU once",
 *             dispatch then combine, expert pairs selected together, next-layer
 *             prediction, locally served token--expert assignments, and routing
 *             decisions left unchanged by both methods.
 * Where the pages leave a step open, the reading taken is stated at the function.
 *
 * Floating point: the pages fix no precision.  The combine reference is computed in
 * float64 (oracle_combine_f64).  oracle_combine_f32chain additionally spells out the
 * fixed-order fp32 accumulation the library specifies (acc = fma(g_j, y_j, acc) for
 * j = 0..k-1 from +0), so that order can be checked bit for bit.
 *
 * Error flags returned (bit-or): 1 = expert id out of range, 2 = repeated id within a
 * token, 4 = row capacity exceeded, 8 = source rank out of range.  A token with an
 * invalid id or source rank is skipped entirely (it contributes nothing).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OF_ID_RANGE 1
#define OF_DUP_ID 2
#define OF_CAPACITY 4
#define OF_SRC_RANK 8

/* Flags for token t: ids in [0,E) and pairwise distinct. */
static int token_flags(const int32_t *ids, int64_t t, int k, int E) {
    int f = 0;
    for (int j = 0; j < k; ++j) {
        int32_t a = ids[t * k + j];
        if (a < 0 || a >= E) f |= OF_ID_RANGE;
        for (int jj = 0; jj < j; ++jj)
            if (ids[t * k + jj] == a) f |= OF_DUP_ID;
    }
    return f;
}

/*
 * Co-activation pair counts and per-expert loads.
 * [Cobalt] "many pairs of experts are frequently co-activated by individual tokens";
 * "per-expert workload statistics".  [Zyphra] "expert pairs ... selected together".
 *   pair[a*E+b] += #{t : a and b both among token t's k experts, a != b}
 *   loads[e]    += #{(t,j) : ids[t,j] == e}
 * Reading: unordered distinct pairs, so the E x E matrix is symmetric with a zero
 * diagonal and its strict upper triangle gains N*k*(k-1)/2; loads are kept apart.
 * Counts accumulate into the caller's arrays.  loads may be NULL.
 */
int oracle_count(const int32_t *ids, int64_t N, int k, int E, int64_t *pair, int64_t *loads) {
    int flags = 0;
    for (int64_t t = 0; t < N; ++t) {
        int f = token_flags(ids, t, k, E);
        flags |= f;
        if (f) continue;
        for (int j = 0; j < k; ++j) {
            int32_t a = ids[t * k + j];
            if (loads) loads[a] += 1;
            for (int jj = 0; jj < k; ++jj) {
                if (jj == j) continue;
                int32_t b = ids[t * k + jj];
                pair[(int64_t)a * E + b] += 1;
            }
        }
    }
    return flags;
}

/*
 * Cross-layer counts.  [Zyphra] "the experts a token selects at one layer predict the
 * experts it selects at the next layer".
 *   C12[a*E2+b] += #{(t,j,j') : ids1[t,j] == a, ids2[t,j'] == b}
 * Not symmetric; a == b is a legitimate entry.  loads1 (may be NULL) gains the
 * layer-1 loads.  A token is skipped if either layer's ids are invalid.
 */
int oracle_count_cross(const int32_t *ids1, int k1, int E1, const int32_t *ids2, int k2, int E2,
                       int64_t N, int64_t *C12, int64_t *loads1) {
    int flags = 0;
    for (int64_t t = 0; t < N; ++t) {
        int f = token_flags(ids1, t, k1, E1) | token_flags(ids2, t, k2, E2);
        flags |= f;
        if (f) continue;
        for (int j = 0; j < k1; ++j) {
            int32_t a = ids1[t * k1 + j];
            if (loads1) loads1[a] += 1;
            for (int jj = 0; jj < k2; ++jj) C12[(int64_t)a * E2 + ids2[t * k2 + jj]] += 1;
        }
    }
    return flags;
}

/*
 * Deduplicated dispatch plan.  [Zyphra] "a dispatcher that sends each token to each
 * GPU once" (rows), [Cobalt] "routes tokens to fewer remote nodes" (node statistics)
 * and all-to-all exchange of tokens under EP.
 *
 * Inputs: ids [N,k]; expert_rank [E] (expert -> logical rank); rank_node [R] (rank ->
 * node, NULL = one node); src_rank [N] (token's home rank, NULL = contiguous shards
 * floor(t*R/N)).
 * Definitions (rank(j) = expert_rank[ids[t,j]]):
 *   rank_mask[t]  = OR_j 1<<rank(j)
 *   kmask(t,r)    = OR_{j : rank(j) == r} 1<<j        (mask over the token's k slots)
 *   rank_counts[r]= #{t : r in rank_mask[t]}           (rows sent to r)
 *   asg(r)        = sum_t popcount(kmask(t,r))         (token-expert assignments on r)
 *   rank_offsets / asg_offsets = exclusive prefix sums over r, with totals at [R]
 * Row order inside rank r's segment: ascending token index (reading: "stable"; with
 * contiguous source shards this is the all-to-all receive order).  Walking r = 0..R-1
 * and t = 0..N-1:
 *   row_token[pos] = t, row_kmask[pos] = kmask(t,r)   (pos < row_capacity; else flag 4)
 *   send_row[t,j]  = pos for the smallest slot j with rank(j) == r, -1 for r's other slots
 *   comb_row[t,j]  = next assignment row of r, slots in ascending j
 * so the expert outputs sit in "expanded receive order": rank segments, send rows in
 * order, one row per set slot in ascending j.
 * Statistics (int64 [8]):
 *   0 naive rows N*k          1 dedup rows D = rank_offsets[R]
 *   2 remote rows     = sum_t popcount(rank_mask[t] without src[t])
 *   3 cross-node rows = sum_t #{r in rank_mask[t] : node(r) != node(src[t])}
 *   4 node-dedup cross-node rows = sum_t #{nodes n != node(src[t]) touched by t}
 *   5 local-served assignments = #{(t,j) : rank(j) == src[t]}
 *   6 remote assignments = N*k - stat5
 *   7 cross-node assignments = #{(t,j) : node(rank(j)) != node(src[t])}
 * src_dst [R*R] (may be NULL): src_dst[s*R+r] = #{t : src[t] == s, r in rank_mask[t]}.
 * rank_mask [N] (may be NULL) is written as uint64.
 * Invalid tokens (bad id, repeated id, bad expert_rank entry, bad src) contribute
 * nothing; their send_row / comb_row entries are -1.
 * oracle_plan_slots states all of this for a rank per slot, slot_rank[t*k + j] (with
 * expert replicas a token's slot may go to any replica of its expert); oracle_plan is
 * the case slot_rank[t*k + j] = expert_rank[ids[t*k + j]].
 */
int oracle_plan_slots(const int32_t *ids, int64_t N, int k, int E, const int32_t *slot_rank, int R,
                const int32_t *rank_node, int n_nodes, const int32_t *src_rank,
                int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                uint64_t *rank_mask_out, int32_t *row_token, uint8_t *row_kmask,
                int64_t row_capacity, int32_t *send_row, int32_t *comb_row, int64_t *stats,
                int32_t *src_dst) {
    int flags = 0;
    (void)n_nodes;
    for (int64_t i = 0; i < N * k; ++i) { send_row[i] = -1; comb_row[i] = -1; }
    for (int s = 0; s < 8; ++s) stats[s] = 0;
    if (src_dst) for (int64_t i = 0; i < (int64_t)R * R; ++i) src_dst[i] = 0;

    /* per-token source rank and validity (an invalid token contributes nothing) */
    int64_t *src = (int64_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(int64_t));
    char *valid = (char *)malloc((size_t)(N > 0 ? N : 1));
    for (int64_t t = 0; t < N; ++t) {
        int f = token_flags(ids, t, k, E);
        src[t] = src_rank ? src_rank[t] : (t * R) / N;
        if (!(f & OF_ID_RANGE))
            for (int j = 0; j < k; ++j) {
                int32_t r = slot_rank[t * k + j];
                if (r < 0 || r >= R) f |= OF_ID_RANGE;
            }
        if (src[t] < 0 || src[t] >= R) f |= OF_SRC_RANK;
        flags |= f;
        valid[t] = (char)(f == 0);
        uint64_t m = 0;
        if (valid[t])
            for (int j = 0; j < k; ++j) m |= 1ull << slot_rank[t * k + j];
        if (rank_mask_out) rank_mask_out[t] = m;
    }

    /* counts and exclusive offsets, by a loop over r */
    int64_t row_acc = 0, asg_acc = 0;
    for (int r = 0; r < R; ++r) {
        int64_t rows = 0, asg = 0;
        for (int64_t t = 0; t < N; ++t) {
            if (!valid[t]) continue;
            int in = 0;
            for (int j = 0; j < k; ++j)
                if (slot_rank[t * k + j] == r) { in = 1; asg += 1; }
            rows += in;
        }
        rank_counts[r] = (int32_t)rows;
        rank_offsets[r] = (int32_t)row_acc;
        asg_offsets[r] = (int32_t)asg_acc;
        row_acc += rows;
        asg_acc += asg;
    }
    rank_offsets[R] = (int32_t)row_acc;
    asg_offsets[R] = (int32_t)asg_acc;

    /* stable positions: walk ranks, then tokens in ascending order */
    for (int r = 0; r < R; ++r) {
        int64_t pos = rank_offsets[r];
        int64_t apos = asg_offsets[r];
        for (int64_t t = 0; t < N; ++t) {
            if (!valid[t]) continue;
            uint32_t km = 0;
            for (int j = 0; j < k; ++j)
                if (slot_rank[t * k + j] == r) km |= 1u << j;
            if (!km) continue;
            int first = 1;
            for (int j = 0; j < k; ++j) {
                if (!(km & (1u << j))) continue;
                if (first) {
                    send_row[t * k + j] = pos < row_capacity ? (int32_t)pos : -1;
                    first = 0;
                }
                comb_row[t * k + j] = (int32_t)apos;
                apos += 1;
            }
            if (pos < row_capacity) {
                row_token[pos] = (int32_t)t;
                row_kmask[pos] = (uint8_t)km;
            } else {
                flags |= OF_CAPACITY;
            }
            if (src_dst) src_dst[src[t] * R + r] += 1;
            pos += 1;
        }
    }

    /* statistics, from the sets of ranks and nodes each token touches */
    stats[0] = N * (int64_t)k;
    stats[1] = row_acc;
    for (int64_t t = 0; t < N; ++t) {
        if (!valid[t]) continue;
        char rank_set[64] = {0}, node_set[64] = {0};
        int node_src = rank_node ? rank_node[src[t]] : 0;
        for (int j = 0; j < k; ++j) {
            int32_t r = slot_rank[t * k + j];
            int nd = rank_node ? rank_node[r] : 0;
            rank_set[r] = 1;
            node_set[nd] = 1;
            if (r == src[t]) stats[5] += 1;
            if (nd != node_src) stats[7] += 1;
        }
        for (int r = 0; r < R; ++r) {
            if (!rank_set[r]) continue;
            if (r != src[t]) stats[2] += 1;
            if ((rank_node ? rank_node[r] : 0) != node_src) stats[3] += 1;
        }
        for (int nd = 0; nd < 64; ++nd)
            if (node_set[nd] && nd != node_src) stats[4] += 1;
    }
    stats[6] = asg_acc - stats[5];   /* every assignment of a valid token that is not local */
    free(src);
    free(valid);
    return flags;
}

/*
 * The plan with each expert on one rank: slot (t, j) goes to expert_rank[ids[t,j]]
 * (the definitions above, through oracle_plan_slots).
 */
int oracle_plan(const int32_t *ids, int64_t N, int k, int E, const int32_t *expert_rank, int R,
                const int32_t *rank_node, int n_nodes, const int32_t *src_rank,
                int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                uint64_t *rank_mask_out, int32_t *row_token, uint8_t *row_kmask,
                int64_t row_capacity, int32_t *send_row, int32_t *comb_row, int64_t *stats,
                int32_t *src_dst) {
    int32_t *slot = (int32_t *)malloc((size_t)(N * k > 0 ? N * k : 1) * sizeof(int32_t));
    for (int64_t i = 0; i < N * k; ++i)
        slot[i] = (ids[i] >= 0 && ids[i] < E) ? expert_rank[ids[i]] : -1;
    int f = oracle_plan_slots(ids, N, k, E, slot, R, rank_node, n_nodes, src_rank, rank_counts,
                              rank_offsets, asg_offsets, rank_mask_out, row_token, row_kmask,
                              row_capacity, send_row, comb_row, stats, src_dst);
    free(slot);
    return f;
}

/* Gathered send buffer: send[d] = x[row_token[d]] for d < D (bf16 rows copied as bits). */
void oracle_gather(const uint16_t *x, int64_t H, const int32_t *row_token, int64_t D,
                   uint16_t *send) {
    for (int64_t d = 0; d < D; ++d)
        memcpy(send + d * H, x + (int64_t)row_token[d] * H, (size_t)H * sizeof(uint16_t));
}

/* bf16 bits -> float: the bf16 pattern is the top half of the float32 pattern. */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/*
 * float32 -> bf16, IEEE round to nearest, ties to even, from the definition: keep
 * the top 16 bits; look at the 16 dropped bits; round up if they exceed half an ulp,
 * or equal half an ulp and the kept part is odd.  A carry out of the mantissa rolls
 * into the exponent (and up to infinity), which is the correct IEEE result.  NaN
 * stays NaN (quiet bit set).
 */
uint16_t oracle_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1;
    return (uint16_t)kept;
}

void oracle_bf16_rne_array(const float *in, uint16_t *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rne(in[i]);
}

/*
 * Weighted combine in float64.  [Zyphra] dispatch tokens to their experts "and then
 * combine the results":
 *   out[t][h] = sum_j gate[t,j] * y[comb_row[t,j]][h]
 * y is bf16 [n_rows, H] in expanded receive order.  Rows with comb_row < 0 or
 * >= n_rows are skipped (invalid tokens).
 */
void oracle_combine_f64(const uint16_t *y, int64_t n_rows, const float *gates,
                        const int32_t *comb_row, int64_t N, int k, int64_t H, double *out) {
    for (int64_t t = 0; t < N; ++t)
        for (int64_t h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int64_t row = comb_row[t * k + j];
                if (row < 0 || row >= n_rows) continue;
                acc += (double)gates[t * k + j] * (double)bf16_to_f32(y[row * H + h]);
            }
            out[t * H + h] = acc;
        }
}

/*
 * The library's specified fp32 accumulation, spelled out: acc starts at +0.0f and
 * takes one fused multiply-add per slot in ascending j (C99 fmaf: one rounding).
 */
void oracle_combine_f32chain(const uint16_t *y, int64_t n_rows, const float *gates,
                             const int32_t *comb_row, int64_t N, int k, int64_t H, float *out) {
    for (int64_t t = 0; t < N; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t row = comb_row[t * k + j];
                if (row < 0 || row >= n_rows) continue;
                acc = fmaf(gates[t * k + j], bf16_to_f32(y[row * H + h]), acc);
            }
            out[t * H + h] = acc;
        }
}

/*
 * Expert outputs of *identity* experts in expanded receive order: for each send row d
 * in order and each set slot of row_kmask[d] in ascending order, one copy of
 * x[row_token[d]].  Returns the number of rows written.
 */
int64_t oracle_expand_identity(const uint16_t *x, int64_t H, const int32_t *row_token,
                               const uint8_t *row_kmask, int64_t D, uint16_t *y) {
    int64_t a = 0;
    for (int64_t d = 0; d < D; ++d)
        for (int j = 0; j < 8; ++j)
            if (row_kmask[d] & (1u << j)) {
                memcpy(y + a * H, x + (int64_t)row_token[d] * H, (size_t)H * sizeof(uint16_t));
                a += 1;
            }
    return a;
}

/*
 * Naive (non-deduplicated) combine with identity experts: one row per (t,j), so
 * every slot's output is x[t]; same fp32 chain as above.  [Zyphra] "neither method
 * changes the models' underlying routing decisions": the deduplicated combine must
 * equal this bit for bit.
 */
void oracle_naive_combine_identity_f32(const uint16_t *x, const float *gates, int64_t N, int k,
                                       int64_t H, float *out) {
    for (int64_t t = 0; t < N; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) acc = fmaf(gates[t * k + j], bf16_to_f32(x[t * H + h]), acc);
            out[t * H + h] = acc;
        }
}

/*
 * Token shuffling's home prediction.  [Zyphra] each token moves "to the GPU predicted
 * to hold its next-layer experts".  Reading: score(t,r) = sum over the token's layer-1
 * experts a of the calibration counts C12[a][b] summed over the layer-2 experts b
 * placed on rank r; the predicted home is the rank with the largest score, ties to the
 * lowest rank.  Tokens with invalid ids get home -1 and flag 1/2.
 */
int oracle_predict_home(const int32_t *ids1, int64_t N, int k1, int E1, const int64_t *C12,
                        int E2, const int32_t *expert_rank2, int R, int32_t *home) {
    int flags = 0;
    for (int64_t t = 0; t < N; ++t) {
        int f = token_flags(ids1, t, k1, E1);
        flags |= f;
        if (f) { home[t] = -1; continue; }
        int best = 0;
        int64_t best_score = -1;
        for (int r = 0; r < R; ++r) {
            int64_t score = 0;
            for (int j = 0; j < k1; ++j) {
                int32_t a = ids1[t * k1 + j];
                for (int b = 0; b < E2; ++b)
                    if (expert_rank2[b] == r) score += C12[(int64_t)a * E2 + b];
            }
            if (score > best_score) { best_score = score; best = r; }
        }
        home[t] = best;
    }
    return flags;
}

/*
 * Correlated expert placement.  [Zyphra] experts that are often selected together are
 * put on the same GPU; [Cobalt] frequently co-activated experts are co-located.  The
 * pages give no algorithm; the reading is a greedy over pair weights
 * w(a,b) = pair[a][b] + pair[b][a] (a < b, w > 0), heaviest first (ties: smaller a, then
 * smaller b): two unplaced experts take the lowest rank with two free slots; an unplaced
 * expert joins its placed partner's rank if a slot is free; then every unplaced expert,
 * in ascending id, takes the lowest rank with a free slot.  E/R slots per rank.
 */
typedef struct { int64_t w; int a, b; } oracle_edge;

static int edge_order(const void *p, const void *q) {
    const oracle_edge *x = (const oracle_edge *)p, *y = (const oracle_edge *)q;
    if (x->w != y->w) return x->w > y->w ? -1 : 1;
    if (x->a != y->a) return x->a < y->a ? -1 : 1;
    if (x->b != y->b) return x->b < y->b ? -1 : 1;
    return 0;
}

int oracle_place_correlated(const int64_t *pair, int E, int R, int32_t *expert_rank) {
    if (E % R != 0) return -1;
    int per_rank = E / R;
    oracle_edge *edges = (oracle_edge *)malloc(sizeof(oracle_edge) * (size_t)E * (size_t)E);
    int *free_slots = (int *)malloc(sizeof(int) * (size_t)R);
    int64_t n = 0;
    for (int a = 0; a < E; ++a)
        for (int b = a + 1; b < E; ++b) {
            int64_t w = pair[(int64_t)a * E + b] + pair[(int64_t)b * E + a];
            if (w > 0) { edges[n].w = w; edges[n].a = a; edges[n].b = b; ++n; }
        }
    qsort(edges, (size_t)n, sizeof(oracle_edge), edge_order);
    for (int e = 0; e < E; ++e) expert_rank[e] = -1;
    for (int r = 0; r < R; ++r) free_slots[r] = per_rank;
    for (int64_t i = 0; i < n; ++i) {
        int a = edges[i].a, b = edges[i].b;
        if (expert_rank[a] < 0 && expert_rank[b] < 0) {
            for (int r = 0; r < R; ++r)
                if (free_slots[r] >= 2) {
                    expert_rank[a] = r;
                    expert_rank[b] = r;
                    free_slots[r] -= 2;
                    break;
                }
        } else if (expert_rank[a] < 0 || expert_rank[b] < 0) {
            int placed = expert_rank[a] >= 0 ? a : b;
            int other = placed == a ? b : a;
            int r = expert_rank[placed];
            if (free_slots[r] > 0) {
                expert_rank[other] = r;
                free_slots[r] -= 1;
            }
        }
    }
    for (int e = 0; e < E; ++e) {
        if (expert_rank[e] >= 0) continue;
        for (int r = 0; r < R; ++r)
            if (free_slots[r] > 0) {
                expert_rank[e] = r;
                free_slots[r] -= 1;
                break;
            }
    }
    free(edges);
    free(free_slots);
    return 0;
}

/*
 * Two-hop dispatch (node level, then rank level).  [Cobalt] routes tokens "to fewer
 * remote nodes": a token crosses to each destination node once (hop 1) and is then
 * forwarded inside the node to each destination rank (hop 2).  The hop-1 plan is the
 * ordinary plan with nodes in place of ranks (expert -> node map, home node).  For each
 * rank-level send row d of token t on rank r, the hop-1 row that feeds it is the node-level
 * row of (t, node(r)):
 *   fwd_src[d] = the e with node_row_token[e] == t inside node(r)'s segment,  d < D
 *   fwd_src[d] = -1                                                           D <= d < cap
 * Definition by lookup: every node-level row e of node n in [node_offsets[n],
 * node_offsets[n+1]) is indexed by (node_row_token[e], n).
 */
void oracle_forward_src(const int32_t *row_token, const int32_t *rank_offsets, int R,
                        const int32_t *rank_node, const int32_t *node_row_token,
                        const int32_t *node_offsets, int n_nodes, int64_t N, int64_t cap,
                        int32_t *fwd_src) {
    /* index[(t, n)] = node-level row, as a dense N x n_nodes table */
    int32_t *index = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1) * (size_t)n_nodes);
    for (int64_t i = 0; i < N * n_nodes; ++i) index[i] = -1;
    for (int n = 0; n < n_nodes; ++n)
        for (int64_t e = node_offsets[n]; e < node_offsets[n + 1]; ++e)
            index[(int64_t)node_row_token[e] * n_nodes + n] = (int32_t)e;
    for (int64_t d = 0; d < cap; ++d) fwd_src[d] = -1;
    for (int r = 0; r < R; ++r) {
        int n = rank_node ? rank_node[r] : 0;
        for (int64_t d = rank_offsets[r]; d < rank_offsets[r + 1] && d < cap; ++d)
            fwd_src[d] = index[(int64_t)row_token[d] * n_nodes + n];
    }
    free(index);
}

/* Row gather: dst[d] = src[fwd_src[d]] for every d with fwd_src[d] >= 0 (bf16 bits). */
void oracle_forward_gather(const uint16_t *src, int64_t H, const int32_t *fwd_src, int64_t cap,
                           uint16_t *dst) {
    for (int64_t d = 0; d < cap; ++d)
        if (fwd_src[d] >= 0)
            memcpy(dst + d * H, src + (int64_t)fwd_src[d] * H, (size_t)H * sizeof(uint16_t));
}

/*
 * Intra-node load rebalancing.  [Cobalt] "per-step intra-node adjustment to rebalance the
 * workloads".  The pages give no algorithm; the reading is the longest-first greedy: take
 * the experts in order of load, heaviest first (equal loads: smaller id first); put each
 * on the least-loaded rank of its own node that has a free slot (equal loads: smaller
 * rank).  E/R slots per rank.  Returns -1 if a node's expert count does not match its
 * slots.
 */
int oracle_rebalance_ranks(const int64_t *loads, const int32_t *expert_node, int E,
                           const int32_t *rank_node, int R, int32_t *expert_rank) {
    if (R < 1 || E < 1) return -1;   /* no rank or no expert: nothing to balance */
    int per_rank = E / R;
    int64_t *rank_load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    int *free_slots = (int *)malloc(sizeof(int) * (size_t)R);
    char *done = (char *)calloc((size_t)E, 1);
    for (int r = 0; r < R; ++r) free_slots[r] = per_rank;
    int status = 0;
    for (int step = 0; step < E; ++step) {
        /* the heaviest expert not yet placed (smallest id among equals) */
        int e = -1;
        for (int c = 0; c < E; ++c)
            if (!done[c] && (e < 0 || loads[c] > loads[e])) e = c;
        done[e] = 1;
        int best = -1;
        for (int r = 0; r < R; ++r)
            if (rank_node[r] == expert_node[e] && free_slots[r] > 0 &&
                (best < 0 || rank_load[r] < rank_load[best]))
                best = r;
        if (best < 0) { status = -1; expert_rank[e] = -1; continue; }
        expert_rank[e] = best;
        rank_load[best] += loads[e];
        free_slots[best] -= 1;
    }
    free(rank_load);
    free(free_slots);
    free(done);
    return status;
}

/* ------------------------------------------------------------------------------------
 * Backward pass and the pre-reduced reverse path.
 *
 * Both forward maps are linear in the rows they move.  The dispatch copies x[t] to every
 * send row of the token (send_row[t,j] >= 0, one per destination rank) and the combine
 * takes a gate-weighted sum of the token's expert outputs, so their gradients are the
 * transposed maps over the same plan.  [Zyphra] dispatch sends each token to each GPU
 * once "and then" combines the results; the reverse direction can therefore also carry one
 * row per (token, GPU): each GPU first sums, with the gates, the outputs of the slots it
 * served (one row per received row), and the token's rank adds those partial rows -- the
 * transposed dispatch again.  Reading taken: the partial rows travel as bf16 (the type of
 * the rows on the wire), accumulated in fp32 in ascending slot order.
 * ------------------------------------------------------------------------------------ */

/*
 * Transpose of the dispatch: grad_x[t] = sum over j ascending with send_row[t,j] >= 0 of
 * grad_send[send_row[t,j]], an fp32 add chain from +0 (caller rounds to bf16 if wanted).
 * Rows outside [0, n_rows) are skipped.
 */
void oracle_gather_backward_f32chain(const uint16_t *g_send, int64_t n_rows, const int32_t *send_row,
                                     int64_t N, int k, int64_t H, float *g_x) {
    for (int64_t t = 0; t < N; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t row = send_row[t * k + j];
                if (row < 0 || row >= n_rows) continue;
                acc = acc + bf16_to_f32(g_send[row * H + h]);
            }
            g_x[t * H + h] = acc;
        }
}

/*
 * Combine driven by units.  Unit u stands for token t = row_token[u] and the slots set in
 * row_kmask[u]; with row_token == NULL unit u is token u with all k slots.
 *   out[u] = sum over set slots j ascending of gates[t,j] * y[comb_row[t,j]]
 * as an fp32 fma chain from +0.  With the plan's rows as units (row_token, row_kmask) this
 * is the partial combine of the pre-reduced reverse path: one row per send row.
 */
void oracle_combine_units_f32chain(const uint16_t *y, int64_t n_rows, const float *gates,
                                   const int32_t *comb_row, int k, const int32_t *row_token,
                                   const uint8_t *row_kmask, int64_t n_units, int64_t H,
                                   float *out) {
    for (int64_t u = 0; u < n_units; ++u) {
        int64_t t = row_token ? row_token[u] : u;
        unsigned m = row_kmask ? row_kmask[u] : 0xffu;
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                if (!((m >> j) & 1u)) continue;
                int64_t row = comb_row[t * k + j];
                if (row < 0 || row >= n_rows) continue;
                acc = fmaf(gates[t * k + j], bf16_to_f32(y[row * H + h]), acc);
            }
            out[u * H + h] = acc;
        }
    }
}

/*
 * Backward of the combine out[t] = sum_j gates[t,j] * y[comb_row[t,j]], over units as in
 * oracle_combine_units_f32chain (g_out has one row per unit):
 *   g_y[comb_row[t,j]]  = bf16_rne(gates[t,j] * g_out[u])   (fp32 product, then RNE)
 *   g_gates[t*k+j]      = sum_h g_out[u,h] * y[comb_row[t,j],h]   in float64
 *   g_gates_abs[t*k+j]  = sum_h |g_out[u,h] * y[comb_row[t,j],h]| (error scale)
 * for every set slot of every unit; a slot whose comb_row is outside [0, n_rows) gets
 * g_gates = 0 and writes no g_y row.  g_y rows no slot names are not written.
 */
void oracle_combine_backward(const uint16_t *y, int64_t n_rows, const float *gates,
                             const int32_t *comb_row, int k, const int32_t *row_token,
                             const uint8_t *row_kmask, int64_t n_units, int64_t H,
                             const uint16_t *g_out, uint16_t *g_y, double *g_gates,
                             double *g_gates_abs) {
    for (int64_t u = 0; u < n_units; ++u) {
        int64_t t = row_token ? row_token[u] : u;
        unsigned m = row_kmask ? row_kmask[u] : 0xffu;
        for (int j = 0; j < k; ++j) {
            if (!((m >> j) & 1u)) continue;
            int64_t row = comb_row[t * k + j];
            double dot = 0.0, mag = 0.0;
            if (row >= 0 && row < n_rows) {
                float g = gates[t * k + j];
                for (int64_t h = 0; h < H; ++h) {
                    float go = bf16_to_f32(g_out[u * H + h]);
                    float p = g * go;
                    g_y[row * H + h] = oracle_bf16_rne(p);
                    double term = (double)go * (double)bf16_to_f32(y[row * H + h]);
                    dot += term;
                    mag += fabs(term);
                }
            }
            g_gates[t * k + j] = dot;
            g_gates_abs[t * k + j] = mag;
        }
    }
}

/* ------------------------------------------------------------------------------------
 * Token shuffling fused into the post-attention reduce-scatter.
 *
 * [Zyphra] under sequence parallelism each token is moved, during the reduce-scatter
 * that follows attention, to the GPU predicted to hold its next-layer experts.  Reading
 * taken: the reduce-scatter runs over the group whose P ranks each hold a partial
 * attention output for all N tokens; rank r receives the tokens whose predicted home is
 * r, in ascending token order (the stable grouping the dispatch plan gives with k = 1),
 * each row the sum of the P partial rows, added in rank order q = 0..P-1 in fp32 from +0.
 * ------------------------------------------------------------------------------------ */

/*
 * out[i] = sum over q = 0..P-1 of parts[q][row_token[i]] (fp32 add chain, caller rounds);
 * parts: P consecutive bf16 [N, H] blocks.  A row_token outside [0, N) gives a zero row.
 */
void oracle_shuffle_reduce_f32chain(const uint16_t *parts, int P, int64_t N, int64_t H,
                                    const int32_t *row_token, int64_t n_out, float *out) {
    for (int64_t i = 0; i < n_out; ++i) {
        int64_t t = row_token[i];
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            if (t >= 0 && t < N)
                for (int q = 0; q < P; ++q) acc = acc + bf16_to_f32(parts[((int64_t)q * N + t) * H + h]);
            out[i * H + h] = acc;
        }
    }
}


/* ------------------------------------------------------------------------------------
 * Replica choice.
 *
 * [Cobalt] EP distributes expert replicas across GPUs, and a communication-aware task
 * assignment routes tokens to fewer remote nodes under the current expert layout.  The
 * pages give no algorithm; the reading taken is a per-token greedy over the slots:
 * expert e has n_rep[e] replicas, on ranks rep_rank[e*max_rep + i], i < n_rep[e].  For a
 * valid token t with home rank s and home node hn:
 *   1. slots whose expert has one replica take it;
 *   2. the other slots, j ascending, take the first replica (ascending i) in the first
 *      non-empty class: (a) on s; (b) on a rank the token already uses; (c) on hn;
 *      (d) on a node the token already uses; otherwise replica (t + j) mod n_rep[e],
 *      which spreads the tokens that must open a new node over the replicas.
 * "Uses" = chosen before, step 1 included.  slot_rank[t*k + j] = the chosen rank; -1 for
 * every slot of an invalid token (bad id, repeated id, bad home rank, or a replica table
 * entry of one of its experts out of range: n_rep outside [1, max_rep] or a rank outside
 * [0, R)).  Returns the error flags.
 * ------------------------------------------------------------------------------------ */
int oracle_assign_replicas(const int32_t *ids, int64_t N, int k, int E, const int32_t *rep_rank,
                           int max_rep, const int32_t *n_rep, int R, const int32_t *rank_node,
                           int n_nodes, const int32_t *src_rank, int32_t *slot_rank) {
    int flags = 0;
    (void)n_nodes;
    for (int64_t t = 0; t < N; ++t) {
        int f = token_flags(ids, t, k, E);
        int64_t s = src_rank ? src_rank[t] : (t * R) / N;
        if (s < 0 || s >= R) f |= OF_SRC_RANK;
        if (!(f & OF_ID_RANGE))
            for (int j = 0; j < k; ++j) {
                int e = ids[t * k + j];
                if (n_rep[e] < 1 || n_rep[e] > max_rep) { f |= OF_ID_RANGE; continue; }
                for (int i = 0; i < n_rep[e]; ++i) {
                    int r = rep_rank[e * max_rep + i];
                    if (r < 0 || r >= R) f |= OF_ID_RANGE;
                }
            }
        flags |= f;
        for (int j = 0; j < k; ++j) slot_rank[t * k + j] = -1;
        if (f) continue;
        int hn = rank_node ? rank_node[s] : 0;
        char used_rank[64] = {0}, used_node[64] = {0};
        for (int j = 0; j < k; ++j) {                      /* step 1 */
            int e = ids[t * k + j];
            if (n_rep[e] == 1) {
                int r = rep_rank[e * max_rep];
                slot_rank[t * k + j] = r;
                used_rank[r] = 1;
                used_node[rank_node ? rank_node[r] : 0] = 1;
            }
        }
        for (int j = 0; j < k; ++j) {                      /* step 2 */
            if (slot_rank[t * k + j] >= 0) continue;
            int e = ids[t * k + j];
            const int32_t *rep = rep_rank + e * max_rep;
            int pick = -1;
            for (int cls = 0; cls < 4 && pick < 0; ++cls)
                for (int i = 0; i < n_rep[e] && pick < 0; ++i) {
                    int r = rep[i];
                    int nd = rank_node ? rank_node[r] : 0;
                    if ((cls == 0 && r == s) || (cls == 1 && used_rank[r]) ||
                        (cls == 2 && nd == hn) || (cls == 3 && used_node[nd]))
                        pick = i;
                }
            if (pick < 0) pick = (int)((t + j) % n_rep[e]);
            int r = rep[pick];
            slot_rank[t * k + j] = r;
            used_rank[r] = 1;
            used_node[rank_node ? rank_node[r] : 0] = 1;
        }
    }
    return flags;
}

/* ------------------------------------------------------------------------------------
 * Replica placement.
 *
 * [Cobalt] EP distributes expert replicas across GPUs; its planner acts on co-activation
 * and workload statistics.  The pages give no algorithm; reading taken (integer
 * arithmetic throughout: an expert's load is shared equally by its replicas, counted in
 * units of 1/840 so every share is exact for up to 8 replicas):
 *   every expert starts with its rank as replica 0; rank_load[r] = sum over the experts
 *   with a replica on r of loads[e]*840/n_rep[e].  An expert is replicable while it has
 *   fewer than max_rep replicas and some rank holds none of them.  Then, budget times:
 *   1. r* = the most loaded rank holding a replica of a replicable expert (ties: lower
 *      rank); none -> stop;
 *   2. e* = among those experts on r*, the one with the largest share
 *      loads[e]*840/n_rep[e] (ties: lower id);
 *   3. candidate ranks: those without a replica of e*, on a node without one if any such
 *      rank exists; among them the node with the largest affinity
 *      A(node) = sum over experts f != e* whose replica 0 is on the node of
 *      pair[e*][f] + pair[f][e*] (ties: lower node), then on it the rank with the
 *      smallest load (ties: lower rank); none -> stop;
 *   4. add that rank as e*'s next replica and recompute the shares of e*'s replicas.
 * Returns the number of replicas added.  rep_rank [E*max_rep] (-1 padded), n_rep [E].
 * ------------------------------------------------------------------------------------ */
int oracle_place_replicas(const int64_t *pair, const int64_t *loads, const int32_t *expert_rank,
                          int E, const int32_t *rank_node, int R, int budget, int max_rep,
                          int32_t *rep_rank, int32_t *n_rep) {
    const int64_t L = 840;
    int64_t *rank_load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    int n_nodes = 1;
    for (int r = 0; r < R; ++r)
        if (rank_node[r] + 1 > n_nodes) n_nodes = rank_node[r] + 1;
    int64_t *aff = (int64_t *)calloc((size_t)n_nodes, sizeof(int64_t));
    for (int e = 0; e < E; ++e) {
        for (int i = 0; i < max_rep; ++i) rep_rank[e * max_rep + i] = -1;
        rep_rank[e * max_rep] = expert_rank[e];
        n_rep[e] = 1;
        rank_load[expert_rank[e]] += loads[e] * L;
    }
    int added = 0;
    for (int b = 0; b < budget; ++b) {
        int rs = -1, es = -1;                                    /* steps 1 and 2 */
        int64_t best_share = -1;
        for (int r = 0; r < R; ++r) {
            if (rs >= 0 && rank_load[r] <= rank_load[rs]) continue;
            int pick = -1;
            int64_t pick_share = -1;
            for (int e = 0; e < E; ++e) {
                if (n_rep[e] >= max_rep || n_rep[e] >= R) continue;
                int on = 0;
                for (int i = 0; i < n_rep[e]; ++i) on |= rep_rank[e * max_rep + i] == r;
                if (!on) continue;
                int64_t share = loads[e] * L / n_rep[e];
                if (share > pick_share) { pick_share = share; pick = e; }
            }
            if (pick >= 0) { rs = r; es = pick; best_share = pick_share; }
        }
        (void)best_share;
        if (es < 0) break;
        /* step 3: ranks and nodes that already hold a replica of es */
        char *has_rank = (char *)calloc((size_t)R, 1);
        char *has_node = (char *)calloc((size_t)n_nodes, 1);
        for (int i = 0; i < n_rep[es]; ++i) {
            has_rank[rep_rank[es * max_rep + i]] = 1;
            has_node[rank_node[rep_rank[es * max_rep + i]]] = 1;
        }
        int fresh_node_exists = 0;
        for (int r = 0; r < R; ++r)
            if (!has_rank[r] && !has_node[rank_node[r]]) fresh_node_exists = 1;
        for (int n = 0; n < n_nodes; ++n) aff[n] = 0;
        for (int f = 0; f < E; ++f)
            if (f != es) aff[rank_node[expert_rank[f]]] += pair[(int64_t)es * E + f] + pair[(int64_t)f * E + es];
        int bn = -1;
        for (int n = 0; n < n_nodes; ++n) {
            int usable = 0;
            for (int r = 0; r < R; ++r)
                if (rank_node[r] == n && !has_rank[r] && (!fresh_node_exists || !has_node[n])) usable = 1;
            if (!usable) continue;
            if (bn < 0 || aff[n] > aff[bn]) bn = n;
        }
        int rt = -1;
        if (bn >= 0)
            for (int r = 0; r < R; ++r) {
                if (rank_node[r] != bn || has_rank[r]) continue;
                if (rt < 0 || rank_load[r] < rank_load[rt]) rt = r;
            }
        free(has_rank);
        free(has_node);
        if (rt < 0) break;
        /* step 4 */
        for (int i = 0; i < n_rep[es]; ++i) rank_load[rep_rank[es * max_rep + i]] -= loads[es] * L / n_rep[es];
        rep_rank[es * max_rep + n_rep[es]] = rt;
        n_rep[es] += 1;
        for (int i = 0; i < n_rep[es]; ++i) rank_load[rep_rank[es * max_rep + i]] += loads[es] * L / n_rep[es];
        added += 1;
    }
    free(rank_load);
    free(aff);
    return added;
}

/* ------------------------------------------------------------------ EP row metadata
 *
 * [Cobalt], [Zyphra]: under expert parallelism every token travels to the ranks that
 * hold its experts (each rank once), those ranks run the experts, and the results travel
 * back to be combined.  A rank receiving a deduplicated row needs, besides the row, the
 * expert id and the gate of each slot the row serves, and where each slot's expert
 * output goes among the rank's outputs.  Reading taken (the pages define no format): one
 * entry per (send row, slot), -1 / 0 / -1 for the slots the row does not serve.
 *
 * oracle_row_meta: for d < n_rows, t = row_token[d], r = the rank whose segment
 * [rank_offsets[r], rank_offsets[r+1]) holds d; for j < k:
 *   bit j of row_kmask[d] set:  experts[d,j] = ids[t,j], gates_out[d,j] = gates[t,j],
 *                               slots[d,j] = comb_row[t,j] + slot_base[r]
 *   else:                       -1, 0, -1
 * (slot_base NULL: 0).  With slot_base[r] = (rows of rank r's outputs that earlier
 * sources send it) - asg_offsets[r], slots[d,j] is where slot j's output sits in the
 * destination's expanded receive order.  Any output pointer may be NULL (skipped);
 * a row whose token is outside [0, N) gets -1 / 0 / -1 everywhere and returns flag 16.
 */
int oracle_row_meta(const int32_t *row_token, const uint8_t *row_kmask, int64_t n_rows,
                    const int32_t *rank_offsets, int R, const int32_t *ids, const float *gates,
                    const int32_t *comb_row, int64_t N, int k, const int32_t *slot_base,
                    int32_t *experts, float *gates_out, int32_t *slots) {
    int flags = 0;
    for (int64_t d = 0; d < n_rows; ++d) {
        int r = 0;
        while (r + 1 < R && d >= rank_offsets[r + 1]) ++r;
        int64_t t = row_token[d];
        int ok = t >= 0 && t < N;
        if (!ok) flags |= 16;
        for (int j = 0; j < k; ++j) {
            int on = ok && ((row_kmask[d] >> j) & 1);
            if (experts) experts[d * k + j] = on ? ids[t * k + j] : -1;
            if (gates_out) gates_out[d * k + j] = on ? gates[t * k + j] : 0.0f;
            if (slots) slots[d * k + j] = on ? comb_row[t * k + j] + (slot_base ? slot_base[r] : 0) : -1;
        }
    }
    return flags;
}

/* oracle_gather_row_slots: the way back of one value per (send row, slot) -- e.g. the
 * gate gradients computed where the experts ran -- to token order:
 *   out[t,j] = vals[d,j] for the send row d of token t whose mask holds bit j,
 *   0 for a slot that none of the token's send rows holds.
 * The token's send rows are the send_row[t, j0] >= 0.  A send row outside [0, n_rows)
 * is skipped and returns flag 16. */
int oracle_gather_row_slots(const float *vals, int64_t n_rows, const int32_t *send_row,
                            const uint8_t *row_kmask, int64_t N, int k, float *out) {
    int flags = 0;
    for (int64_t t = 0; t < N; ++t) {
        for (int j = 0; j < k; ++j) out[t * k + j] = 0.0f;
        for (int j0 = 0; j0 < k; ++j0) {
            int64_t d = send_row[t * k + j0];
            if (d < 0) continue;
            if (d >= n_rows) { flags |= 16; continue; }
            for (int j = 0; j < k; ++j)
                if ((row_kmask[d] >> j) & 1) out[t * k + j] = vals[d * k + j];
        }
    }
    return flags;
}
