/*
 * coact.h -- C ABI of the B200 (sm_100a) co-activation dispatch/combine library.
 *
 * The library implements the data-parallel hot path that two pages share:
 *   Cobalt, "efficient distributed MoE training using expert co-activation"
 *     (arxivdaily 2609.36959), English abstract;
 *   Zyphra correlated expert placement and token shuffling
 *     (arxivdaily 2610.09372), English abstract.
 * Under expert parallelism (EP) tokens travel to the ranks that hold their experts and
 * the expert outputs come back to be combined.  The library counts which experts are
 * co-activated, plans a dispatch that sends each token to each destination rank once,
 * gathers the hidden rows into per-rank send buffers and combines expert outputs back
 * in token order.  Logical ranks are partitions of one GPU's memory.
 *
 * Conventions for every entry point:
 *  - Array pointers are DEVICE pointers owned by the caller (e.g. torch tensors).  The
 *    library never allocates, frees or synchronises; all work is enqueued on `stream`
 *    (a cudaStream_t; NULL = the legacy default stream).  Calls are asynchronous.
 *  - Kernels are launched with programmatic stream serialisation (programmatic dependent
 *    launch): a library kernel may start while the previous kernel on the stream drains,
 *    and waits for it (griddepcontrol.wait) before touching its outputs.  Work that the
 *    caller enqueues normally after a call sees all of that call's results.  A kernel
 *    of the caller's own that is launched with programmatic stream serialisation right
 *    after a call must likewise wait before reading that call's outputs: a library
 *    kernel lets its successor start once its own wait has returned, before it finishes
 *    (the last kernel of plan_dispatch excepted: its successor starts when it completes).
 *  - Return value: COACT_OK (0) or a negative coact_status.  A negative status is
 *    decided on the host before anything is enqueued (except COACT_ERR_CUDA, which
 *    reports a failed launch).
 *  - Data errors that only the device can see (an expert id out of range, a repeated
 *    id within a token, a row index out of range, a full send buffer) set bits of
 *    coact_eflag in *err_flag with an atomic OR.  err_flag is an int32 DEVICE pointer
 *    and may be NULL; the caller zeroes it and reads it after the stream syncs.  When a
 *    bit is set, the outputs that depend on the offending tokens are unspecified, but
 *    no kernel ever reads or writes outside the buffers it was given, traps or hangs.
 *  - Row data are bf16, passed as uint16_t bit patterns, row-major, rows of H elements.
 *    Row buffers must be 16-byte aligned and H a multiple of 8 (16-byte rows).
 *  - Limits: 1 <= k <= 8 experts per token, 2 <= E <= 1024 experts, 1 <= R <= 64
 *    ranks, 1 <= n_nodes <= 64, N*k < 2^31, row_capacity < 2^31.
 */
#ifndef COACT_H
#define COACT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *coact_stream_t;

enum coact_status {
    COACT_OK = 0,
    COACT_ERR_INVALID = -1,      /* NULL required pointer, negative size, bad alignment */
    COACT_ERR_UNSUPPORTED = -2,  /* argument outside the documented limits */
    COACT_ERR_CUDA = -3,         /* a CUDA launch or attribute call failed */
    COACT_ERR_WORKSPACE = -4,    /* workspace NULL or smaller than the query says */
    COACT_ERR_TIMEOUT = -5       /* reserved: a bounded device wait gave up */
};

enum coact_eflag {
    COACT_EFLAG_ID_RANGE = 1,    /* expert id (or its rank) outside its range; token skipped */
    COACT_EFLAG_DUP_ID = 2,      /* the same expert twice in one token; token skipped */
    COACT_EFLAG_CAPACITY = 4,    /* a send row fell at or beyond row_capacity; not written */
    COACT_EFLAG_SRC_RANK = 8,    /* src_rank[t] outside [0, R); token skipped */
    COACT_EFLAG_ROW_RANGE = 16,  /* send_row / comb_row entry outside the row buffer; skipped */
    COACT_EFLAG_TIMEOUT = 32     /* a bounded wait on an mbarrier gave up; outputs unspecified */
};

#define COACT_MAX_K 8
#define COACT_MAX_E 1024
#define COACT_MAX_R 64
#define COACT_MAX_REPLICAS 8   /* replicas per expert (assign_replicas) */
#define COACT_NUM_STATS 8

/* Indices into the stats[8] array written by plan_dispatch. */
enum coact_stat {
    COACT_STAT_NAIVE_ROWS = 0,          /* N*k: one row per token-expert assignment */
    COACT_STAT_DEDUP_ROWS = 1,          /* D: one row per (token, destination rank) */
    COACT_STAT_REMOTE_ROWS = 2,         /* rows whose rank is not the token's home rank */
    COACT_STAT_CROSSNODE_ROWS = 3,      /* rows whose rank sits on another node */
    COACT_STAT_NODE_DEDUP_ROWS = 4,     /* (token, remote node) pairs: rows if sent once per node */
    COACT_STAT_LOCAL_ASG = 5,           /* assignments whose expert is on the home rank */
    COACT_STAT_REMOTE_ASG = 6,          /* assignments whose expert is elsewhere */
    COACT_STAT_CROSSNODE_ASG = 7        /* assignments whose expert is on another node */
};

/* Static text for a coact_status value. */
const char *coact_strerror(int status);

/* ABI version of this header (bumped on any signature change). */
int coact_abi_version(void);

/*
 * coact_last_cuda_error -- the cudaError_t behind the last COACT_ERR_CUDA returned on the
 * calling host thread (0 if none).  A failed CUDA call inside the library is recorded
 * here and consumed, so no later, unrelated cudaGetLastError check reports it again.
 */
int coact_last_cuda_error(void);

/* ABI versions (additions only; no earlier call changed meaning):
 *   1  count, plan, gather, combine, predict_home, placement, two-hop, peer calls, noalloc
 *   2  dispatch_gather_tma, backward (dispatch_gather_backward, combine_scatter_backward),
 *      combine_rows, shuffle_reduce_scatter, assign_replicas, plan_dispatch_slots,
 *      forward_gather_tokens, coact_last_cuda_error; combine_scatter_peer takes NULL gates
 *   3  plan_row_meta, gather_row_slots, rebalance_ranks */
#define COACT_ABI_VERSION 3

/*
 * coact_count -- expert co-activation pair counts and per-expert loads.
 * Cobalt, English abstract: many pairs of experts are co-activated by single tokens,
 * and per-expert workload statistics drive the layout planner; Zyphra, English
 * abstract: a small share of expert pairs is selected together by a large share of
 * tokens, and the experts a token picks at one layer predict those at the next.
 *
 * Co-activation mode (ids2 == NULL):
 *   pair[a*E+b] += #{t : a and b are both among ids[t, 0..k-1], a != b}
 *   The increment is symmetric with a zero diagonal; its strict upper triangle sums
 *   to N*k*(k-1)/2.
 * Cross-layer mode (ids2 != NULL, same N):
 *   pair[a*E2+b] += #{(t, j, j2) : ids[t,j] == a, ids2[t,j2] == b}   (E x E2, not symmetric)
 * loads[e] += #{(t, j) : ids[t,j] == e}   (loads may be NULL).
 *
 * ids: int32 [N, k] row-major; ids2: int32 [N, k2] or NULL (then k2, E2 are ignored).
 * pair: int64 [E*E] (or [E*E2]), loads: int64 [E]; both ACCUMULATE (+=), so zero them
 * for fresh counts.  A token with an id outside [0, E) (or [0, E2)) or a repeated id
 * is not counted and sets COACT_EFLAG_ID_RANGE / COACT_EFLAG_DUP_ID.
 */
int coact_count(const int32_t *ids, int64_t N, int k, int E,
                const int32_t *ids2, int k2, int E2,
                int64_t *pair, int64_t *loads,
                int32_t *err_flag, coact_stream_t stream);

/* Bytes of device workspace plan_dispatch needs for these sizes (0 if N == 0). */
size_t plan_dispatch_workspace_bytes(int64_t N, int k, int E, int R);

/*
 * plan_dispatch -- the deduplicated dispatch layout.
 * Zyphra, English abstract: a dispatcher that sends each token to each GPU once;
 * Cobalt, English abstract: routing tokens to fewer remote nodes under the current
 * expert layout (node-level statistics).
 *
 * Inputs (device): ids int32 [N,k]; expert_rank int32 [E] (expert -> rank in [0,R));
 * rank_node int32 [R] (rank -> node in [0,n_nodes)) or NULL (one node); src_rank int32
 * [N] (the token's home rank) or NULL (contiguous shards: floor(t*R/N)).
 * With rank(j) = expert_rank[ids[t,j]]:
 *   rank_mask[t]   = OR_j 1 << rank(j)                         (uint64 [N], may be NULL)
 *   kmask(t, r)    = OR_{j : rank(j) == r} 1 << j              (mask over the k slots)
 *   rank_counts[r] = #{t : r in rank_mask[t]}                  (int32 [R])
 *   rank_offsets   = exclusive prefix sum of rank_counts; rank_offsets[R] = D (int32 [R+1])
 *   asg_offsets    = exclusive prefix sum over r of sum_t popcount(kmask(t,r));
 *                    asg_offsets[R] = number of valid assignments (int32 [R+1])
 * Rows of rank r occupy [rank_offsets[r], rank_offsets[r+1]) in ascending token order:
 *   row_token[d] = t, row_kmask[d] = kmask(t, r)   (int32 / uint8 [row_capacity])
 *   send_row[t,j] = the row of (t, rank(j)) if j is the smallest slot on rank(j),
 *                   else -1                                     (int32 [N,k])
 *   comb_row[t,j] = the row of assignment (t, j) in "expanded receive order": rank
 *                   segments starting at asg_offsets[r], rows in order, one row per set
 *                   slot in ascending j                         (int32 [N,k])
 * Rows at or beyond row_capacity are not written (their send_row is -1) and set
 * COACT_EFLAG_CAPACITY; row_capacity >= N*min(k,R) can never overflow.  Rows of
 * [D, row_capacity) are left untouched.
 * stats int64 [8] (see coact_stat), src_dst int32 [R*R] or NULL:
 *   src_dst[s*R + r] = #{t : src[t] == s, r in rank_mask[t]} (the all-to-all split sizes).
 * workspace: device memory of at least plan_dispatch_workspace_bytes(N,k,E,R) bytes,
 * 16-byte aligned; its contents need no initialisation and are scratch afterwards.
 * Tokens with invalid ids, an expert_rank entry outside [0,R) or a src_rank outside
 * [0,R) contribute no rows, get send_row = comb_row = -1, and set their flag.
 * Deterministic: no result depends on scheduling.
 */
int plan_dispatch(const int32_t *ids, int64_t N, int k, int E,
                  const int32_t *expert_rank, int R,
                  const int32_t *rank_node, int n_nodes,
                  const int32_t *src_rank,
                  int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                  uint64_t *rank_mask,
                  int32_t *row_token, uint8_t *row_kmask, int64_t row_capacity,
                  int32_t *send_row, int32_t *comb_row,
                  int64_t *stats, int32_t *src_dst,
                  void *workspace, size_t workspace_bytes,
                  int32_t *err_flag, coact_stream_t stream);

/*
 * assign_replicas -- which replica serves each (token, slot).
 * Cobalt, English abstract: EP distributes expert replicas across GPUs, and a
 * communication-aware task assignment routes tokens to fewer remote nodes under the
 * current expert layout.  Expert e has n_rep[e] replicas (1 <= n_rep[e] <= max_rep <=
 * COACT_MAX_REPLICAS) on ranks rep_rank[e*max_rep + i], i < n_rep[e] (int32 DEVICE
 * arrays).  Per token t (home rank s = src_rank[t], or floor(t*R/N) when src_rank is
 * NULL; home node hn): slots whose expert has one replica take it; the other slots, j
 * ascending, take the first replica (ascending i) in the first non-empty class -- (a) on
 * s, (b) on a rank the token already uses, (c) on hn, (d) on a node the token already
 * uses -- otherwise replica (t + j) mod n_rep[e].  slot_rank: int32 [N, k] out, the
 * chosen rank per slot, -1 for every slot of an invalid token (bad or repeated id, bad
 * home rank: COACT_EFLAG_ID_RANGE / _DUP_ID / _SRC_RANK; a replica table entry out of
 * range: COACT_EFLAG_ID_RANGE).  The pages give no algorithm; this greedy is the reading
 * taken.  Feed the result to plan_dispatch_slots.
 */
int assign_replicas(const int32_t *ids, int64_t N, int k, int E,
                    const int32_t *rep_rank, int max_rep, const int32_t *n_rep, int R,
                    const int32_t *rank_node, int n_nodes, const int32_t *src_rank,
                    int32_t *slot_rank, int32_t *err_flag, coact_stream_t stream);

/*
 * plan_dispatch_slots -- plan_dispatch with a rank per slot instead of a rank per expert:
 * slot (t, j) goes to slot_rank[t*k + j] (int32 [N, k] DEVICE, e.g. from assign_replicas;
 * a value outside [0, R) makes the token invalid, COACT_EFLAG_ID_RANGE).  ids are still
 * validated (range, repeats) and every output, layout and flag is as in plan_dispatch
 * with expert_rank[ids[t,j]] replaced by slot_rank[t*k + j]; same workspace size.
 */
int plan_dispatch_slots(const int32_t *ids, int64_t N, int k, int E,
                        const int32_t *slot_rank, int R,
                        const int32_t *rank_node, int n_nodes,
                        const int32_t *src_rank,
                        int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                        uint64_t *rank_mask,
                        int32_t *row_token, uint8_t *row_kmask, int64_t row_capacity,
                        int32_t *send_row, int32_t *comb_row,
                        int64_t *stats, int32_t *src_dst,
                        void *workspace, size_t workspace_bytes,
                        int32_t *err_flag, coact_stream_t stream);

/*
 * dispatch_gather -- fill the per-rank send buffers.
 * Cobalt / Zyphra, English abstracts: tokens are exchanged through all-to-all so that
 * each reaches the ranks holding its experts, each rank once.
 *   send[send_row[t,j]] = x[t]   for every (t, j) with send_row[t,j] >= 0
 * i.e. send[d] = x[row_token[d]] for d < D.  Each x row is read once and written to
 * every distinct destination row.
 * x: bf16 [N, H]; send_row: int32 [N, k] (from plan_dispatch); send: bf16
 * [row_capacity, H].  Entries >= row_capacity set COACT_EFLAG_ROW_RANGE and are skipped;
 * rows not named by send_row are left untouched.  Copies are bit-exact.
 */
int dispatch_gather(const uint16_t *x, int64_t N, int64_t H,
                    const int32_t *send_row, int k,
                    uint16_t *send, int64_t row_capacity,
                    int32_t *err_flag, coact_stream_t stream);

/*
 * dispatch_gather_tma -- dispatch_gather through the Tensor Memory Accelerator: rows are
 * staged in shared memory with bulk asynchronous copies (cp.async.bulk, one issuing warp
 * per CTA, completion tracked by mbarriers whose waits are bounded by wall clock) and
 * written to every destination with bulk stores.  Same arguments, results and flags as
 * dispatch_gather (plus COACT_EFLAG_TIMEOUT if a bounded wait gives up); rows up to 32 KB
 * (H <= 16384), else COACT_ERR_UNSUPPORTED.  One warp per CTA and no row registers; on
 * B200 it is 2-3% slower than dispatch_gather, alone and next to a concurrent GEMM alike
 * (both are bound by HBM bandwidth, not by SM resources).
 */
int dispatch_gather_tma(const uint16_t *x, int64_t N, int64_t H,
                        const int32_t *send_row, int k,
                        uint16_t *send, int64_t row_capacity,
                        int32_t *err_flag, coact_stream_t stream);

/*
 * combine_scatter -- the weighted combine back to token order.
 * Zyphra, English abstract: tokens are dispatched to their experts "and then" the
 * results are combined; neither method changes the routing decisions.
 *   out[t] = sum_{j=0..k-1} gates[t,j] * y[comb_row[t,j]]
 * computed per element in fp32 as acc = +0.0f; acc = fmaf(gates[t,j], y, acc) for
 * j = 0, 1, ..., k-1 in that order (one rounding per step), then stored as fp32 or
 * rounded to bf16 nearest-even.
 * y: bf16 [n_rows, H] expert outputs in expanded receive order (n_rows = N*k for a full
 * plan); gates: fp32 [N, k]; comb_row: int32 [N, k]; out: [N, H] of bf16 (out_dtype 0)
 * or fp32 (out_dtype 1).  A comb_row entry outside [0, n_rows) is skipped: -1 silently
 * (a slot of an invalid token), any other value with COACT_EFLAG_ROW_RANGE.
 * Rate: bound by HBM reads, with the loads in flight staged in each SM's L1 data cache,
 * so it runs at full rate only where the L1 is not given over to shared memory.  Its
 * CTAs take whatever shared-memory carveout an SM already has when they start beside
 * another kernel's blocks (after a predecessor that triggers its dependents early, or on
 * another stream): on B200 the combine of 131,072 tokens with k = 8 and H = 7168 took
 * 3.0 ms instead of 2.4 under the largest carveout.
 */
int combine_scatter(const uint16_t *y, int64_t n_rows, const float *gates,
                    const int32_t *comb_row, int64_t N, int k, int64_t H,
                    void *out, int out_dtype,
                    int32_t *err_flag, coact_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Backward pass and the pre-reduced reverse path.
 *
 * The dispatch copies x[t] to the token's send rows and the combine is a gate-weighted
 * sum, both linear, so their gradients are the transposed maps over the same plan.  The
 * reverse direction can also carry one row per (token, rank) -- as Zyphra's dispatcher
 * sends each token to each GPU once: the rank that ran the experts first sums, with the
 * gates, the outputs of the slots it served (combine_rows over the plan's send rows), and
 * the token's rank adds those partial rows (dispatch_gather_backward, the transposed
 * dispatch), so D rows travel back instead of N*k.
 *
 * Units: combine_rows and combine_scatter_backward take an optional unit list.  Unit u
 * is token row_token[u] restricted to the slots set in row_kmask[u] (e.g. the plan's
 * row_token / row_kmask over its D send rows); with row_token NULL (backward only) unit u
 * is token u with all k slots.  A row_token entry outside [0, N) on a unit with slots set
 * raises COACT_EFLAG_ROW_RANGE and the unit contributes nothing.  unit_count (DEVICE
 * int32, may be NULL): when given, only units u < min(n_units, *unit_count) are processed
 * -- e.g. &rank_offsets[R] = D, so that n_units can be the plan's row_capacity and the
 * call needs no host synchronisation; output rows of the other units are not written.
 * ------------------------------------------------------------------------------------ */

/*
 * combine_rows -- the combine over units:
 *   out[u] = sum over the slots j set in row_kmask[u], ascending, of
 *            gates[t,j] * y[comb_row[t,j]],   t = row_token[u]
 * as the fp32 fma chain of combine_scatter (from +0.0f), stored fp32 (out_dtype 1) or
 * rounded to bf16 nearest-even (out_dtype 0).  out: [n_units, H].  Other arguments and
 * flags as combine_scatter.
 */
int combine_rows(const uint16_t *y, int64_t n_rows, const float *gates,
                 const int32_t *comb_row, int64_t N, int k,
                 const int32_t *row_token, const uint8_t *row_kmask, int64_t n_units,
                 const int32_t *unit_count, int64_t H, void *out, int out_dtype,
                 int32_t *err_flag, coact_stream_t stream);

/*
 * dispatch_gather_backward -- the transpose of dispatch_gather:
 *   grad_x[t] = sum over j ascending with send_row[t,j] >= 0 of grad_send[send_row[t,j]]
 * per element an fp32 add chain from +0.0f, stored fp32 (out_dtype 1) or rounded to bf16
 * nearest-even (out_dtype 0).  grad_send: bf16 [n_rows, H] (n_rows = the plan's
 * row_capacity, rows >= D unread); send_row: the plan's int32 [N, k]; grad_x: [N, H].
 * It is also the second stage of the pre-reduced combine (grad_send := the partial rows).
 * A send_row entry below -1 or >= n_rows sets COACT_EFLAG_ROW_RANGE and is skipped.
 */
int dispatch_gather_backward(const uint16_t *grad_send, int64_t n_rows,
                             const int32_t *send_row, int64_t N, int k, int64_t H,
                             void *grad_x, int out_dtype,
                             int32_t *err_flag, coact_stream_t stream);

/*
 * combine_scatter_backward -- gradients of the combine, per unit u (token t) and set slot j:
 *   grad_y[comb_row[t,j]]  = bf16_rne(gates[t,j] * grad_out[u])   (fp32 product, per element)
 *   grad_gates[t*k + j]    = sum_h grad_out[u,h] * y[comb_row[t,j],h]   (fp32)
 * grad_out: bf16 [n_units, H] (token mode: [N, H]); grad_y: bf16 [n_rows, H], rows no
 * slot names are not written; grad_gates: fp32 [N, k], slots no unit covers are not
 * written, a covered slot without a row (comb_row -1) gets 0.  The dot product sums, per
 * lane of a warp, m products in ascending order with fma -- m = 16*ceil(H/512) when y,
 * grad_out and grad_y are 32-byte aligned and H % 16 == 0, else 8*ceil(H/256) -- then
 * adds the 32 lane sums by a 5-level butterfly: its error is at most (m + 5) * 2^-24 *
 * sum_h |grad_out * y| (first order).  n_units and unit_count are ignored when row_token
 * is NULL.
 */
int combine_scatter_backward(const uint16_t *y, int64_t n_rows, const float *gates,
                             const int32_t *comb_row, int64_t N, int k,
                             const int32_t *row_token, const uint8_t *row_kmask,
                             int64_t n_units, const int32_t *unit_count,
                             const uint16_t *grad_out, int64_t H,
                             uint16_t *grad_y, float *grad_gates,
                             int32_t *err_flag, coact_stream_t stream);

/*
 * plan_dispatch_noalloc -- plan_dispatch without a caller-provided workspace.
 * No counterpart in the papers: it exists for callers that cannot allocate device
 * memory, such as code running inside a runtime that owns all device memory through its
 * own pool or a fixed memory plan and forbids stray allocations, or a latency-critical
 * caller that cannot afford cudaMalloc's implicit device-wide synchronisation.  It
 * computes exactly what plan_dispatch computes (same arguments and outputs, minus
 * workspace / workspace_bytes) and allocates nothing: its scratch is a file-scope
 * device array of the library, sized for N <= COACT_NOALLOC_MAX_TOKENS and R <= 64
 * (about 560 KB), which every GPU that loads the library holds until the process exits.
 *  - N > COACT_NOALLOC_MAX_TOKENS returns COACT_ERR_UNSUPPORTED before anything is
 *    enqueued; use plan_dispatch with a workspace for larger batches.
 *  - The first call on each device looks up the scratch array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call before any
 *    stream capture.  The address is kept per CUDA context: after a device reset (a new
 *    context, in which the library's module is loaded again) the first call looks it up
 *    again, so make that call outside a capture too.
 *  - All calls on a device share the one scratch array, and it keeps the last call's
 *    contents.  Nothing in it needs clearing (every entry a call reads is written
 *    earlier in the same call), but calls that overlap on the GPU -- e.g. two streams at
 *    once -- race on it: order such calls on one stream.
 */
#define COACT_NOALLOC_MAX_TOKENS 262144
int plan_dispatch_noalloc(const int32_t *ids, int64_t N, int k, int E,
                          const int32_t *expert_rank, int R,
                          const int32_t *rank_node, int n_nodes,
                          const int32_t *src_rank,
                          int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                          uint64_t *rank_mask,
                          int32_t *row_token, uint8_t *row_kmask, int64_t row_capacity,
                          int32_t *send_row, int32_t *comb_row,
                          int64_t *stats, int32_t *src_dst,
                          int32_t *err_flag, coact_stream_t stream);

/*
 * Two-hop dispatch.  Cobalt, English abstract: the communication-aware task assignment
 * "routes tokens to fewer remote nodes".  Hop 1 sends each token once to each destination
 * NODE (an ordinary plan_dispatch at node granularity: expert -> node map, home node, R =
 * n_nodes); hop 2 forwards each node-level row inside the node to the token's ranks there
 * (the rank-level plan).  These three calls connect the two plans.
 *
 * coact_compose_map -- out[i] = b[a[i]] for i < n (device arrays; e.g. expert -> rank ->
 * node with a = expert_rank, b = rank_node; or token home rank -> home node).  An a[i]
 * outside [0, nb) gives out[i] = -1 and COACT_EFLAG_ID_RANGE.
 */
int coact_compose_map(const int32_t *a, int64_t n, const int32_t *b, int64_t nb, int32_t *out,
                      int32_t *err_flag, coact_stream_t stream);

/*
 * plan_forward -- which hop-1 row feeds each hop-2 row.
 *   fwd_src[d] = the node-level row of (t, node(r)) for the rank-level row d of token t on
 *                rank r (d < D = rank_offsets[R]);  -1 for D <= d < row_capacity
 * ids, expert_rank, rank_node, n_nodes: as given to the rank-level plan_dispatch;
 * send_row / rank_offsets: that plan's outputs; node_send_row: the node-level plan's
 * send_row (int32 [N,k]) for the same ids.  fwd_src: int32 [row_capacity].  Row indices
 * at or beyond row_capacity set COACT_EFLAG_ROW_RANGE; invalid tokens are skipped.
 */
int plan_forward(const int32_t *ids, int64_t N, int k, int E, const int32_t *expert_rank, int R,
                 const int32_t *rank_node, int n_nodes, const int32_t *send_row,
                 const int32_t *rank_offsets, const int32_t *node_send_row, int32_t *fwd_src,
                 int64_t row_capacity, int32_t *err_flag, coact_stream_t stream);

/*
 * forward_gather -- the intra-node forward of hop 2:  dst[d] = src[fwd_src[d]] for every
 * d < n_rows with fwd_src[d] >= 0 (bf16 rows of H; other rows untouched).  src: the
 * hop-1 send buffer [n_src_rows, H]; dst: the rank-level send buffer [n_rows, H].  An
 * fwd_src entry at or beyond n_src_rows sets COACT_EFLAG_ROW_RANGE and is skipped.
 * Composition: forward_gather(dispatch_gather(x, node plan), plan_forward(...)) equals
 * dispatch_gather(x, rank plan) row for row.
 */
int forward_gather(const uint16_t *src, int64_t n_src_rows, int64_t H, const int32_t *fwd_src,
                   int64_t n_rows, uint16_t *dst, int32_t *err_flag, coact_stream_t stream);

/*
 * forward_gather_tokens -- forward_gather's rows in token order: for each token t, its
 * rank rows d = send_row[t, j] >= 0 (the rank plan's [N, k]) are grouped by their hop-1
 * row fwd_src[d]; each hop-1 row is read once and written to every rank row it feeds, so
 * the forward reads Dn hop-1 rows instead of D.  Results equal forward_gather's for every
 * rank row a token reaches (all d < D); other rows untouched.  A send_row entry below -1
 * or >= n_rows, or an fwd_src entry >= n_src_rows, sets COACT_EFLAG_ROW_RANGE and is
 * skipped.
 */
int forward_gather_tokens(const uint16_t *src, int64_t n_src_rows, int64_t H,
                          const int32_t *send_row, int64_t N, int k, const int32_t *fwd_src,
                          int64_t n_rows, uint16_t *dst, int32_t *err_flag, coact_stream_t stream);

/*
 * Expert parallelism across GPUs (one process per GPU; EP rank s plans its own tokens for
 * all R destination ranks).  Cobalt / Zyphra, English abstracts: every MoE layer exchanges
 * tokens all-to-all to the GPUs holding their experts and combines the results back.
 * These two calls fuse that exchange into the data movement through per-rank buffer
 * tables -- on a GPU system, the peers' NVLink-mapped buffers (e.g. symmetric memory);
 * plain device pointers work the same way on one GPU.  With C[s][r] = rows and A[s][r] =
 * assignments that source s sends to rank r (rank_counts / diff(asg_offsets) of s's
 * plan), source s writes at row offsets off[r] = sum_{s'<s} C[s'][r] and reads back at
 * sum_{s'<s} A[s'][r]; every destination buffer then holds exactly the rank-r segment the
 * single-GPU plan of all sources' tokens would produce (sources contiguous in token
 * order).  Ordering across GPUs (all writes done before the experts read, all expert
 * outputs written before the combine reads) is the caller's barrier.
 *
 * dispatch_gather_peer -- for this source's plan (send_row [N,k], rank_offsets [R+1]):
 *   row d of rank r's segment goes to dst_bases[r] + (dst_row_offset[r] + d - rank_offsets[r]) * H
 * dst_bases: DEVICE array of R uint64 device addresses (bf16 [dst_capacity[r], H] each);
 * dst_row_offset, dst_capacity: DEVICE int32 [R].  A row outside [0, dst_capacity[r]) or a
 * NULL base sets COACT_EFLAG_ROW_RANGE and is skipped.  x: bf16 [N,H], 16-byte aligned.
 */
int dispatch_gather_peer(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row, int k,
                         const int32_t *rank_offsets, int R, const uint64_t *dst_bases,
                         const int32_t *dst_row_offset, const int32_t *dst_capacity,
                         int32_t *err_flag, coact_stream_t stream);

/*
 * combine_scatter_peer -- combine_scatter reading the expert outputs from the ranks that
 * computed them: assignment row a of rank r's segment (asg_offsets [R+1] of this source's
 * plan) is read at y_bases[r] + (y_row_offset[r] + a - asg_offsets[r]) * H.  Same fp32
 * fma chain, output types and flags as combine_scatter; y_bases / y_row_offset /
 * y_capacity: DEVICE arrays as above.  gates may be NULL (every weight 1): with send_row
 * for comb_row and rank_offsets for asg_offsets this is dispatch_gather_backward reading
 * each row from the rank that holds it -- the way back of the pre-reduced combine (the
 * partial rows) and of the dispatch's gradient.  A -1 entry is skipped silently.
 */
int combine_scatter_peer(const uint64_t *y_bases, const int32_t *y_row_offset,
                         const int32_t *y_capacity, const int32_t *asg_offsets, int R,
                         const float *gates, const int32_t *comb_row, int64_t N, int k, int64_t H,
                         void *out, int out_dtype, int32_t *err_flag, coact_stream_t stream);

/*
 * plan_row_meta -- what travels with each send row under expert parallelism besides the
 * row itself.  Cobalt / Zyphra, English abstracts: each token goes to the ranks holding
 * its experts (each rank once), which run them and send the results back to be combined;
 * a deduplicated row serves one or more of the token's k slots.  For
 * d < n_rows = min(row_capacity, rank_offsets[R]) (read on the device) and j < k, with
 * t = row_token[d] and r the rank whose segment [rank_offsets[r], rank_offsets[r+1])
 * holds d:
 *   bit j of row_kmask[d] set:  row_experts[d,j] = ids[t,j]      (the expert to run)
 *                               row_gates[d,j]   = gates[t,j]    (for a combine there)
 *                               row_slots[d,j]   = comb_row[t,j] + slot_base[r]
 *   otherwise:                  -1, 0.0f, -1
 * slot_base: DEVICE int32 [R] or NULL (0).  With slot_base[r] = (assignment rows that
 * earlier sources send rank r) - asg_offsets[r], row_slots[d,j] is the position of slot
 * j's expert output in rank r's expanded receive order -- the comb_row the receiving
 * rank's own combine or backward takes.  Inputs are the plan's outputs (row_token,
 * row_kmask [row_capacity], rank_offsets [R+1], comb_row [N,k]) and the router's ids
 * int32 / gates fp32 [N,k]; outputs [row_capacity, k] (rows >= n_rows untouched), each
 * optional (NULL: not computed; its input may then be NULL).  A row whose token is
 * outside [0, N) gets -1 / 0 / -1 and sets COACT_EFLAG_ROW_RANGE.
 */
int plan_row_meta(const int32_t *row_token, const uint8_t *row_kmask, int64_t row_capacity,
                  const int32_t *rank_offsets, int R,
                  const int32_t *ids, const float *gates, const int32_t *comb_row,
                  int64_t N, int k, const int32_t *slot_base,
                  int32_t *row_experts, float *row_gates, int32_t *row_slots,
                  int32_t *err_flag, coact_stream_t stream);

/*
 * gather_row_slots -- the way back of one value per (send row, slot) to token order, e.g.
 * the gate gradients computed where the experts ran, returned in send-row order:
 *   out[t,j] = vals[d,j] for the send row d of token t (one of its send_row[t, j0] >= 0)
 *              whose row_kmask[d] holds bit j,
 *   out[t,j] = 0 where none does (slots of invalid tokens).
 * vals: DEVICE fp32 [n_rows, k]; send_row int32 [N,k] and row_kmask uint8 [>= n_rows] of
 * the plan; out: DEVICE fp32 [N,k], every entry written.  A send row outside [0, n_rows)
 * is skipped and sets COACT_EFLAG_ROW_RANGE.
 */
int gather_row_slots(const float *vals, int64_t n_rows, const int32_t *send_row,
                     const uint8_t *row_kmask, int64_t N, int k, float *out,
                     int32_t *err_flag, coact_stream_t stream);

/*
 * shuffle_reduce_scatter -- token shuffling fused into the post-attention reduce-scatter.
 * Zyphra, English abstract: under sequence parallelism each token moves, during the
 * reduce-scatter that follows attention, to the GPU predicted to hold its next-layer
 * experts.  The P ranks each hold a partial attention output for all N tokens (bf16
 * [N, H] at part_bases[q]: DEVICE array of P uint64 device addresses -- the peers'
 * NVLink-mapped buffers on a GPU group, local buffers on one GPU); this call writes
 *   out[i] = sum over q = 0..P-1 of part_q[row_token[i]]   for i < n_out
 * per element an fp32 add chain in rank order from +0.0f, stored fp32 (out_dtype 1) or
 * rounded to bf16 nearest-even (out_dtype 0); out: [n_out, H].  row_token: the tokens of
 * this rank's output rows -- the row_token segment [rank_offsets[r], rank_offsets[r+1])
 * of plan_dispatch over ids = home [N, 1], E = R, expert_rank = identity, i.e. the tokens
 * predicted to live on rank r in ascending order (home from predict_home).  A row_token
 * outside [0, N) gives a zero row and COACT_EFLAG_ROW_RANGE; a NULL or misaligned (not
 * 16-byte) partial base is skipped with COACT_EFLAG_ROW_RANGE.  1 <= P <= 64.  Ordering
 * across GPUs (partials written before this call reads them) is the caller's barrier.
 */
int shuffle_reduce_scatter(const uint64_t *part_bases, int P, int64_t N, int64_t H,
                           const int32_t *row_token, int64_t n_out, void *out, int out_dtype,
                           int32_t *err_flag, coact_stream_t stream);

/* Bytes of device workspace predict_home needs (E1*R int64 scores). */
size_t predict_home_workspace_bytes(int E1, int R);

/*
 * predict_home -- token shuffling's home-rank prediction.
 * Zyphra, English abstract: when sequence parallelism shards tokens across the EP
 * group, each token is moved to the GPU predicted to hold its next-layer experts.
 * Prediction from cross-layer counts C12 (coact_count in cross mode over a calibration
 * batch):
 *   score(t, r) = sum_j sum_{b : expert_rank2[b] == r} C12[ids1[t,j] * E2 + b]
 *   home[t]     = argmax_r score(t, r), ties to the lowest r
 * ids1: int32 [N, k1] (layer-1 ids); C12: int64 [E1*E2]; expert_rank2: int32 [E2];
 * home: int32 [N] (then usable as plan_dispatch's src_rank).  workspace: at least
 * predict_home_workspace_bytes(E1, R) bytes.  Tokens with invalid ids get home = -1
 * and set their flag; layer-2 experts with a rank outside [0, R) set
 * COACT_EFLAG_ID_RANGE and are ignored.
 */
int predict_home(const int32_t *ids1, int64_t N, int k1, int E1,
                 const int64_t *C12, int E2, const int32_t *expert_rank2, int R,
                 int32_t *home, void *workspace, size_t workspace_bytes,
                 int32_t *err_flag, coact_stream_t stream);

/*
 * coact_place_correlated -- correlated expert placement (HOST function).
 * Zyphra, English abstract: experts that are often selected together go on the same
 * GPU, which with the once-per-GPU dispatcher removes dispatched rows; Cobalt, English
 * abstract: co-activated experts are co-located to cut cross-node traffic.  The pages
 * give no algorithm; this is a plain greedy over the pair counts:
 *   weight(a,b) = pair[a*E+b] + pair[b*E+a] for a < b, pairs with weight > 0 visited by
 *   weight descending (ties: a, then b ascending); two unplaced experts go together to
 *   the lowest rank with two free slots, an unplaced expert joins its placed partner if
 *   that rank has a free slot; remaining experts, ascending id, fill the lowest rank
 *   with a free slot.  Every rank receives exactly E/R experts.
 * pair: HOST int64 [E*E] (e.g. a copy of coact_count's output); expert_rank: HOST
 * int32 [E] output.  Requires E % R == 0.  Synchronous; no CUDA call.
 */
int coact_place_correlated(const int64_t *pair, int E, int R, int32_t *expert_rank);

/*
 * coact_rebalance_ranks -- intra-node load rebalancing (HOST function).
 * Cobalt, English abstract: a two-stage layout planner co-locates frequently co-activated
 * experts on the same node (stage 1: coact_place_correlated with R = n_nodes gives expert ->
 * node) and adjusts the layout inside each node to rebalance workloads (stage 2: this
 * call).  The pages give no algorithm; this is the longest-first greedy: experts by load
 * descending (ties: lower id), each to the least-loaded rank of its node with a free slot
 * (ties: lower rank).  loads: HOST int64 [E] (coact_count's per-expert loads);
 * expert_node: HOST int32 [E]; rank_node: HOST int32 [R]; expert_rank: HOST int32 [E]
 * output.  Requires E % R == 0 and every node to hold exactly (its ranks) x E/R experts
 * (COACT_ERR_INVALID otherwise).  Synchronous; no CUDA call.
 */
int coact_rebalance_ranks(const int64_t *loads, const int32_t *expert_node, int E,
                          const int32_t *rank_node, int R, int32_t *expert_rank);

/*
 * rebalance_ranks -- the same greedy on the device, for Cobalt's "per-step intra-node
 * adjustment" (English abstract) without a host round trip: the loads coact_count left on
 * the device go straight to a placement plan_dispatch can take.  Within each node, its
 * experts by load descending (ties: lower id) each take the node's least loaded rank
 * with a free slot (E/R slots per rank; ties: lower rank).  loads: DEVICE int64 [E];
 * expert_node: DEVICE int32 [E]; rank_node: DEVICE int32 [R] in [0, n_nodes);
 * expert_rank: DEVICE int32 [E] (out).  Needs E % R == 0 (host check).  An expert whose
 * node is outside [0, n_nodes) or has no free slot left (a node layout that does not fit
 * its ranks) gets -1 and sets COACT_EFLAG_ID_RANGE, as does a rank whose node is outside
 * [0, n_nodes) (it then takes no expert).  One CTA; no host synchronisation.
 */
int rebalance_ranks(const int64_t *loads, const int32_t *expert_node, int E,
                    const int32_t *rank_node, int R, int n_nodes, int32_t *expert_rank,
                    int32_t *err_flag, coact_stream_t stream);

/*
 * coact_place_replicas -- a replica layout from co-activation and workload statistics
 * (host code).  Cobalt, English abstract: EP distributes expert replicas across GPUs; the
 * planner follows co-activation and workload statistics.  Reading taken: an expert's load
 * is shared equally by its replicas (units of 1/840); `budget` times, the most loaded
 * rank holding a replicable expert (fewer than max_rep replicas, some rank without one)
 * gives its largest such share a new replica, on a node holding no replica of that
 * expert if such a node still has a rank,
 * the node with the largest co-activation sum_f pair[e][f] + pair[f][e] over the experts f
 * whose replica 0 lives there, on that node's least loaded rank (ties: lower id).  pair:
 * HOST int64 [E, E]; loads: HOST int64 [E]; expert_rank: HOST int32 [E] (replica 0);
 * rank_node: HOST int32 [R]; out: rep_rank HOST int32 [E, max_rep] (-1 padded), n_rep
 * HOST int32 [E] -- the tables assign_replicas takes.  Returns the number of replicas
 * added (>= 0), or a negative status.
 */
int coact_place_replicas(const int64_t *pair, const int64_t *loads, const int32_t *expert_rank,
                         int E, const int32_t *rank_node, int R, int budget, int max_rep,
                         int32_t *rep_rank, int32_t *n_rep);

#ifdef __cplusplus
}
#endif

#endif /* COACT_H */
