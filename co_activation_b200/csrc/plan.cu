// plan_dispatch: the deduplicated dispatch layout.
//
// Zyphra (arxivdaily 2610.09372), English abstract: "a dispatcher that sends each token
// to each GPU once" -- one send row per (token, destination rank) instead of one per
// (token, expert).  Cobalt (arxivdaily 2609.36959), English abstract: routing tokens to
// fewer remote nodes -- node-level statistics of the same plan.
//
// Launches, none of which waits on another block (a cooperative single-launch variant
// with two bounded grid barriers was measured on B200: slower on N = 16K tokens, 6 us
// faster on 64-128K, so it was dropped):
//  1. k_plan_tiles   one thread per token, 256-token tiles: per-token rank mask, per-tile
//                    per-rank row and assignment counts (per-warp bit planes of the
//                    tokens' rank counts, transposed across the warp; no atomics) and
//                    per-tile statistics partials.
//  2. k_plan_scan    R + 1 blocks: block r turns rank r's per-tile counts into exclusive
//                    per-tile bases (in place) and a total; the last block reduces the
//                    statistics partials and clears src_dst.
//     (skipped when R * n_tiles <= COACT_PLAN_SMALL_MAX: k_plan_scatter<SMALL> then sums
//     the per-tile counts itself, which costs less than a launch at these sizes)
//  3. k_plan_scatter one thread per token again: rank offsets from the totals, stable
//                    in-tile positions from the same transposed bit planes (popcounts
//                    of the lane sets below this lane: rows, and count bits weighted by
//                    2^q: assignments), then row_token / row_kmask / send_row /
//                    comb_row / rank_mask, and the src x dst split matrix.  It does its
//                    in-tile work before waiting on its predecessor, and triggers no
//                    early launch of its own successor.
// Positions depend only on token order, so every output is deterministic.
#include <algorithm>

#include <mutex>

#include "common.cuh"

namespace coact {
namespace {

#if defined(COACT_PLAN_TILE)
constexpr int kTile = COACT_PLAN_TILE;     // experiment builds (a multiple of 32, <= 1024)
#else
constexpr int kTile = 256;                 // tokens per tile, one per thread
#endif
constexpr int kTileWarps = kTile / 32;
constexpr int kScanThreads = 1024;
constexpr int kStatSlots = 6;              // per-tile partials (see TileStat)
enum TileStat { TS_REMOTE_ROWS, TS_XNODE_ROWS, TS_NODE_ROWS, TS_LOCAL_ASG, TS_XNODE_ASG, TS_VALID_ASG };

struct Workspace {
    int32_t *tile_rows;   // [R][n_tiles]  counts, then exclusive bases (in place)
    int32_t *tile_asg;    // [R][n_tiles]
    int64_t *tile_stats;  // [n_tiles][kStatSlots]
    int32_t *tot;         // [2R] rows per rank, assignments per rank
};

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t workspace_layout(int64_t N, int R, Workspace *ws, void *base) {
    const int64_t n_tiles = ceil_div(N, kTile);
    const size_t b_rows = align256(sizeof(int32_t) * (size_t)R * n_tiles);
    const size_t b_stats = align256(sizeof(int64_t) * kStatSlots * (size_t)n_tiles);
    const size_t b_tot = align256(sizeof(int32_t) * 2 * (size_t)R);
    if (ws) {
        char *p = static_cast<char *>(base);
        ws->tile_rows = reinterpret_cast<int32_t *>(p);
        ws->tile_asg = reinterpret_cast<int32_t *>(p + b_rows);
        ws->tile_stats = reinterpret_cast<int64_t *>(p + 2 * b_rows);
        ws->tot = reinterpret_cast<int32_t *>(p + 2 * b_rows + b_stats);
    }
    return 2 * b_rows + b_stats + b_tot;
}

// Token t's per-slot ranks and home rank; returns validation bits (0 = valid).  The rank
// of slot j is slot_rank[t*K + j] when slot_rank is given (expert replicas), else
// expert_rank[ids[t,j]].
template <int K>
__device__ __forceinline__ int load_token(const int32_t *__restrict__ ids,
                                          const int32_t *__restrict__ expert_rank,
                                          const int32_t *__restrict__ slot_rank,
                                          const int32_t *__restrict__ src_rank, int64_t t,
                                          int64_t N, int E, int R, int (&rk)[K], int &src) {
    int e[K];
    int f = load_ids<K>(ids, t, E, e);
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (slot_rank)
            rk[j] = __ldg(slot_rank + t * K + j);
        else
            rk[j] = (f & COACT_EFLAG_ID_RANGE) ? 0 : __ldg(expert_rank + e[j]);
        if ((unsigned)rk[j] >= (unsigned)R) f |= COACT_EFLAG_ID_RANGE;
    }
    src = src_rank ? __ldg(src_rank + t) : (int)((t * R) / N);
    if ((unsigned)src >= (unsigned)R) f |= COACT_EFLAG_SRC_RANK;
    return f;
}

// rank -> node table and node -> rank-set table in shared memory.  A node id outside
// [0, n_nodes) raises COACT_EFLAG_ID_RANGE and is read as node 0.
__device__ __forceinline__ int fetch_node(const int32_t *__restrict__ rank_node, int R) {
    const int tid = threadIdx.x;
    return (tid < R && rank_node) ? __ldg(rank_node + tid) : 0;
}

// nd: this thread's fetch_node() value (issued early so its latency overlaps other loads).
__device__ __forceinline__ void load_nodes(int nd, int R, int n_nodes, int *s_node,
                                           unsigned long long *s_node_ranks, int32_t *err) {
    const int tid = threadIdx.x;
    if (tid < 64) {
        if (tid < R && (unsigned)nd >= (unsigned)n_nodes) {
            raise_flag(err, COACT_EFLAG_ID_RANGE);
            nd = 0;
        }
        s_node[tid] = tid < R ? nd : 0;
        s_node_ranks[tid] = 0;
    }
    __syncthreads();
    if (tid < R) atomicOr(&s_node_ranks[s_node[tid]], 1ull << tid);
    __syncthreads();
}

// ---- per-warp rank tables by bit planes
//
// A warp holds 32 tokens, one per lane, each with its K slot ranks.  Every per-rank count
// the planner needs -- rows (lanes holding rank r), assignments (slots on rank r), and
// their exclusive prefixes over the lanes -- comes from one table: for rank r and bit q,
// the set of lanes whose slot count c_r has bit q set.  Each lane first writes its own
// counts as NP bit planes over the ranks (bit r of plane q = bit q of c_r, NW 32-bit words
// for R <= 32 * NW), then a warp bit-matrix transpose per plane word turns them into the
// per-rank lane sets, held by lane r % 32.  The cost is independent of how many ranks the
// warp touches (a loop over the ranks, with a ballot per rank and count bit, costs ~75
// instructions per rank: ~4,600 per warp at R = 64, k = 8).

// Bits needed to hold a count of 0..K.
template <int K>
constexpr int plane_bits() { return K >= 8 ? 4 : K >= 4 ? 3 : K >= 2 ? 2 : 1; }

// This lane's per-rank slot counts as bit planes: bit (r & 31) of p[q][r >> 5] is bit q
// of #{j : rk[j] == r}.  All zero when !ok.
// Built by adding one-hot rank vectors with a ripple carry through the planes (the count
// never exceeds K < 2^NP, so the last carry is always zero).
template <int K, int NW>
__device__ __forceinline__ void count_planes(const int (&rk)[K], bool ok,
                                             uint32_t (&p)[plane_bits<K>()][NW]) {
    constexpr int NP = plane_bits<K>();
#pragma unroll
    for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int w = 0; w < NW; ++w) p[q][w] = 0;
    if (!ok) return;
#pragma unroll
    for (int j = 0; j < K; ++j) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            uint32_t carry = (rk[j] >> 5) == w ? 1u << (rk[j] & 31) : 0u;
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const uint32_t c = p[q][w] & carry;
                p[q][w] ^= carry;
                carry = c;
            }
        }
    }
}

// 32 x 32 bit-matrix transpose across the warp: lane i passes row i (bit j = entry (i, j))
// and gets back column i (bit j = entry (j, i)).  Each of the five butterfly steps swaps
// the two off-diagonal s x s blocks inside every 2s x 2s block (an exchange with lane
// i ^ s); together they swap the row and column index bits.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
    constexpr uint32_t kHi[5] = {0xFFFF0000u, 0xFF00FF00u, 0xF0F0F0F0u, 0xCCCCCCCCu, 0xAAAAAAAAu};
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int s = 16 >> i;
        const uint32_t hi = kHi[i];
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, s);
        x = (lane & s) ? ((x & hi) | ((y & hi) >> s)) : ((x & ~hi) | ((y & ~hi) << s));
    }
    return x;
}

// Count planes -> per-rank lane sets in place: afterwards p[q][w] on lane l is the set of
// lanes whose count of rank 32*w + l has bit q set.
template <int K, int NW>
__device__ __forceinline__ void transpose_planes(uint32_t (&p)[plane_bits<K>()][NW], int lane) {
#pragma unroll
    for (int q = 0; q < plane_bits<K>(); ++q)
#pragma unroll
        for (int w = 0; w < NW; ++w) p[q][w] = warp_transpose32(p[q][w], lane);
}

// From the lane sets of rank 32*w + lane: the warp's rows on it (lanes holding it) and
// assignments on it (the sum of the lanes' counts).
template <int K, int NW>
__device__ __forceinline__ void rank_totals(const uint32_t (&p)[plane_bits<K>()][NW], int w,
                                            uint32_t &lanes, int &rows, int &asg) {
    lanes = 0;
    asg = 0;
#pragma unroll
    for (int q = 0; q < plane_bits<K>(); ++q) {
        lanes |= p[q][w];
        asg += __popc(p[q][w]) << q;
    }
    rows = __popc(lanes);
}

template <int K, int NW>
__global__ void __launch_bounds__(kTile)
    k_plan_tiles(const int32_t *__restrict__ ids, int64_t N, int E,
                 const int32_t *__restrict__ expert_rank, const int32_t *__restrict__ slot_rank,
                 int R,
                 const int32_t *__restrict__ rank_node, int n_nodes,
                 const int32_t *__restrict__ src_rank, int n_tiles, Workspace ws,
                 int32_t *__restrict__ src_dst, int32_t *__restrict__ err) {
    __shared__ int s_node[64];
    __shared__ unsigned long long s_node_ranks[64];
    __shared__ int s_wrows[kTileWarps][64];
    __shared__ int s_wasg[kTileWarps][64];
    __shared__ long long s_stat[kTileWarps][kStatSlots];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    if (src_dst && blockIdx.x == 0)   // cleared here; the scatter kernel accumulates into it
        for (int i = tid; i < R * R; i += kTile) src_dst[i] = 0;
    // the node table's load and the token's loads are in flight together
    const int nd = fetch_node(rank_node, R);
    const int64_t t = (int64_t)blockIdx.x * kTile + tid;
    int rk[K];
    int src = 0;
    bool ok = false;
    int flags = 0;
    if (t < N) {
        flags = load_token<K>(ids, expert_rank, slot_rank, src_rank, t, N, E, R, rk, src);
        ok = flags == 0;
    }
    load_nodes(nd, R, n_nodes, s_node, s_node_ranks, err);
    unsigned long long mask = 0;
    int st[kStatSlots] = {0, 0, 0, 0, 0, 0};
    if (ok) {
        const int nsrc = s_node[src];
        unsigned long long nmask = 0;
#pragma unroll
        for (int j = 0; j < K; ++j) {
            mask |= 1ull << rk[j];
            const int nd = s_node[rk[j]];
            nmask |= 1ull << nd;
            st[TS_LOCAL_ASG] += rk[j] == src;
            st[TS_XNODE_ASG] += nd != nsrc;
        }
        st[TS_REMOTE_ROWS] = __popcll(mask & ~(1ull << src));
        st[TS_XNODE_ROWS] = __popcll(mask & ~s_node_ranks[nsrc]);
        st[TS_NODE_ROWS] = __popcll(nmask & ~(1ull << nsrc));
        st[TS_VALID_ASG] = K;
    }
    // per-rank counts of this warp (every rank < R written): rows = lanes holding the
    // rank, asg = slots on it; lane l holds ranks l and 32 + l
    uint32_t pl[plane_bits<K>()][NW];
    count_planes<K, NW>(rk, ok, pl);
    transpose_planes<K, NW>(pl, lane);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int r = 32 * w + lane;
        uint32_t lanes;
        int rows, asg;
        rank_totals<K, NW>(pl, w, lanes, rows, asg);
        if (r < R) {
            s_wrows[warp][r] = rows;
            s_wasg[warp][r] = asg;
        }
    }
#pragma unroll
    for (int i = 0; i < kStatSlots; ++i) {
        const int v = __reduce_add_sync(0xffffffffu, st[i]);
        if (lane == 0) s_stat[warp][i] = v;
    }
    raise_flag_warp(err, flags);
    __syncthreads();
    if (tid < R) {
        int rows = 0, asg = 0;
#pragma unroll
        for (int w = 0; w < kTileWarps; ++w) {
            rows += s_wrows[w][tid];
            asg += s_wasg[w][tid];
        }
        ws.tile_rows[(int64_t)tid * n_tiles + blockIdx.x] = rows;
        ws.tile_asg[(int64_t)tid * n_tiles + blockIdx.x] = asg;
    }
    if (tid < kStatSlots) {
        long long v = 0;
#pragma unroll
        for (int w = 0; w < kTileWarps; ++w) v += s_stat[w][tid];
        ws.tile_stats[(int64_t)blockIdx.x * kStatSlots + tid] = v;
    }
}

// Exclusive scan of one int per thread over the block; returns the prefix and sets
// *total.  All threads must call.
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < nw) s_warp[lane] = wi - w;     // exclusive per-warp base
        if (lane == 31) s_warp[32] = wi;          // block total
    }
    __syncthreads();
    const int out = s_warp[warp] + inc - v;
    *total = s_warp[32];
    __syncthreads();
    return out;
}

__global__ void __launch_bounds__(kScanThreads)
    k_plan_scan(int64_t N, int K, int R, int n_tiles, Workspace ws, int64_t *__restrict__ stats,
                int32_t *__restrict__ src_dst) {
    __shared__ int s_warp[33];
    __shared__ long long s_red[kStatSlots][32];
    pdl_wait();
    pdl_trigger();
    if ((int)blockIdx.x < R) {
        const int r = blockIdx.x;
        for (int which = 0; which < 2; ++which) {
            int32_t *row = (which == 0 ? ws.tile_rows : ws.tile_asg) + (int64_t)r * n_tiles;
            int carry = 0;
            for (int c0 = 0; c0 < n_tiles; c0 += kScanThreads) {
                const int i = c0 + threadIdx.x;
                const int v = i < n_tiles ? row[i] : 0;
                int tot;
                const int ex = block_excl_scan(v, s_warp, &tot);
                if (i < n_tiles) row[i] = carry + ex;
                carry += tot;
            }
            if (threadIdx.x == 0) ws.tot[which * R + r] = carry;
        }
        return;
    }
    // statistics block
    long long acc[kStatSlots] = {0, 0, 0, 0, 0, 0};
    for (int i = threadIdx.x; i < n_tiles; i += kScanThreads)
#pragma unroll
        for (int s = 0; s < kStatSlots; ++s) acc[s] += ws.tile_stats[(int64_t)i * kStatSlots + s];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int s = 0; s < kStatSlots; ++s) {
        long long v = acc[s];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) s_red[s][warp] = v;
    }
    __syncthreads();
    if (threadIdx.x < kStatSlots) {
        long long v = 0;
        for (int w = 0; w < kScanThreads / 32; ++w) v += s_red[threadIdx.x][w];
        s_red[threadIdx.x][0] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        stats[COACT_STAT_NAIVE_ROWS] = N * K;
        stats[COACT_STAT_REMOTE_ROWS] = s_red[TS_REMOTE_ROWS][0];
        stats[COACT_STAT_CROSSNODE_ROWS] = s_red[TS_XNODE_ROWS][0];
        stats[COACT_STAT_NODE_DEDUP_ROWS] = s_red[TS_NODE_ROWS][0];
        stats[COACT_STAT_LOCAL_ASG] = s_red[TS_LOCAL_ASG][0];
        stats[COACT_STAT_REMOTE_ASG] = s_red[TS_VALID_ASG][0] - s_red[TS_LOCAL_ASG][0];
        stats[COACT_STAT_CROSSNODE_ASG] = s_red[TS_XNODE_ASG][0];
    }
    if (src_dst)   // only when no tiles ran (N == 0); otherwise k_plan_tiles cleared it
        for (int i = threadIdx.x; i < R * R; i += kScanThreads) src_dst[i] = 0;
}

// Rank offsets from per-rank totals (R <= 64: two ranks per lane of warp 0), then this
// tile's base per rank.  tot_row/tot_asg and before_row/before_asg give, per rank, the
// totals over all tiles and the sums over the tiles before this one.  Block 0 also
// writes the offset outputs.
__device__ __forceinline__ void rank_bases(int R, int tile, const int *tot_row,
                                           const int *tot_asg, const int *before_row,
                                           const int *before_asg, int *s_rbase, int *s_abase,
                                           int32_t *rank_counts, int32_t *rank_offsets,
                                           int32_t *asg_offsets, int64_t *stats) {
    const int lane = threadIdx.x & 31;
    const int r0 = lane, r1 = lane + 32;
    for (int which = 0; which < 2; ++which) {
        const int *tot = which == 0 ? tot_row : tot_asg;
        const int *before = which == 0 ? before_row : before_asg;
        const int v0 = r0 < R ? tot[r0] : 0, v1 = r1 < R ? tot[r1] : 0;
        int i0 = v0, i1 = v1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u0 = __shfl_up_sync(0xffffffffu, i0, o);
            const int u1 = __shfl_up_sync(0xffffffffu, i1, o);
            if (lane >= o) {
                i0 += u0;
                i1 += u1;
            }
        }
        const int total0 = __shfl_sync(0xffffffffu, i0, 31);
        const int total = total0 + __shfl_sync(0xffffffffu, i1, 31);
        const int e0 = i0 - v0, e1 = total0 + i1 - v1;
        int *sbase = which == 0 ? s_rbase : s_abase;
        if (r0 < R) sbase[r0] = e0 + before[r0];
        if (r1 < R) sbase[r1] = e1 + before[r1];
        if (tile == 0) {
            int32_t *offs = which == 0 ? rank_offsets : asg_offsets;
            if (r0 < R) offs[r0] = e0;
            if (r1 < R) offs[r1] = e1;
            if (lane == 0) offs[R] = total;
            if (which == 0) {
                if (r0 < R) rank_counts[r0] = v0;
                if (r1 < R) rank_counts[r1] = v1;
                if (lane == 0) stats[COACT_STAT_DEDUP_ROWS] = total;
            }
        }
    }
}

// SMALL: the scan kernel is skipped (R * n_tiles small); every block sums the raw
// per-tile counts itself and block 0 reduces the statistics.  Otherwise the per-tile
// counts have been scanned in place by k_plan_scan and ws.tot holds the totals.
// Everything before pdl_wait() reads only this call's inputs (safe: the predecessor is
// this call's own k_plan_tiles or k_plan_scan, see pdl_wait).
template <int K, bool SMALL, int NW>
__global__ void __launch_bounds__(kTile)
    k_plan_scatter(const int32_t *__restrict__ ids, int64_t N, int E,
                   const int32_t *__restrict__ expert_rank, const int32_t *__restrict__ slot_rank,
                   int R,
                   const int32_t *__restrict__ src_rank, int n_tiles, Workspace ws,
                   int32_t *__restrict__ rank_counts, int32_t *__restrict__ rank_offsets,
                   int32_t *__restrict__ asg_offsets, unsigned long long *__restrict__ rank_mask,
                   int32_t *__restrict__ row_token, uint8_t *__restrict__ row_kmask, int64_t cap,
                   int32_t *__restrict__ send_row, int32_t *__restrict__ comb_row,
                   int64_t *__restrict__ stats, int32_t *__restrict__ src_dst,
                   int32_t *__restrict__ err) {
    __shared__ int s_rbase[64], s_abase[64];
    __shared__ int s_wrows[kTileWarps][64];
    __shared__ int s_wasg[kTileWarps][64];
    __shared__ uint32_t s_lanes[kTileWarps][plane_bits<K>()][32 * NW];  // per-warp lane sets
    __shared__ uint32_t s_pre[(K + 1) / 2][kTile];  // per-slot in-warp prefixes, 16 bits each
    __shared__ int s_tot[2][64], s_before[2][64];
    __shared__ long long s_stat[kTileWarps][kStatSlots];
    extern __shared__ int s_sd[];  // [R*R] when src_dst != NULL

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x;
    // The last kernel of the call does not trigger its dependents: they launch when it
    // completes.  Launched earlier, the next kernel's CTAs (the dispatch gather) would
    // share SMs with this kernel's blocks and inherit the shared-memory carveout chosen
    // for them (~164 KB of 228 at R = 64) for as long as they keep those SMs busy -- the
    // whole gather -- and the gather's 32-byte loads in flight need the L1 capacity
    // (on B200, 131,072 tokens with k = 8 over 64 ranks and rows of H = 7168: the
    // count + plan + gather + combine step took 4.47 ms instead of 4.06).
    if (src_dst)
        for (int i = tid; i < R * R; i += kTile) s_sd[i] = 0;
    __syncthreads();

    // ---- in-tile work: reads only the call's inputs
    const int64_t t = (int64_t)tile * kTile + tid;
    int rk[K];
    int src = 0;
    bool ok = false;
    int flags = 0;
    if (t < N) ok = load_token<K>(ids, expert_rank, slot_rank, src_rank, t, N, E, R, rk, src) == 0;
    unsigned long long mask = 0;
    if (ok) {
#pragma unroll
        for (int j = 0; j < K; ++j) mask |= 1ull << rk[j];
    }
    // lanes with the same home rank, for the src x dst split counts
    const unsigned same_src = __match_any_sync(0xffffffffu, ok ? src : -1);

    // per-rank lane sets of this warp (lane l: ranks l and 32 + l), per-warp totals (every
    // rank < R written) and the sets themselves for the per-slot prefixes below
    uint32_t pl[plane_bits<K>()][NW];
    count_planes<K, NW>(rk, ok, pl);
    transpose_planes<K, NW>(pl, lane);
    uint32_t holders[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int r = 32 * w + lane;
        int rows, asg;
        rank_totals<K, NW>(pl, w, holders[w], rows, asg);
        if (r < R) {
            s_wrows[warp][r] = rows;
            s_wasg[warp][r] = asg;
        }
#pragma unroll
        for (int q = 0; q < plane_bits<K>(); ++q) s_lanes[warp][q][r] = pl[q][w];
    }
    // src x dst split counts: for each group of valid lanes sharing a home rank (usually
    // one per warp), its rows per destination rank
    if (src_dst) {
        unsigned rest = __ballot_sync(0xffffffffu, ok);
        while (rest) {
            const int leader = __ffs(rest) - 1;
            const unsigned grp = __shfl_sync(0xffffffffu, same_src, leader);
            const int s = __shfl_sync(0xffffffffu, src, leader);
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const int r = 32 * w + lane;
                const int n = __popc(holders[w] & grp);
                if (r < R && n) atomicAdd(&s_sd[s * R + r], n);
            }
            rest &= ~grp;
        }
    }
    __syncwarp();
    // per slot, 16 bits (two slots a word, kept in shared memory across the wait below):
    // in-warp row prefix (< 32) | in-warp assignment prefix (< 256) << 8, from the lanes
    // below this one in the lane sets of the slot's rank
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int j2 = 0; j2 < (K + 1) / 2; ++j2) {
        uint32_t packed = 0;
#pragma unroll
        for (int h = 0; h < 2 && 2 * j2 + h < K; ++h) {
            const int r = ok ? rk[2 * j2 + h] : 0;
            uint32_t below = 0;
            int ap = 0;
#pragma unroll
            for (int q = 0; q < plane_bits<K>(); ++q) {
                const uint32_t m = s_lanes[warp][q][r] & lt;
                below |= m;
                ap += __popc(m) << q;
            }
            packed |= (uint32_t)(__popc(below) | (ap << 8)) << (16 * h);
        }
        s_pre[j2][tid] = packed;
    }
    __syncthreads();
    if (tid < R) {
        int run_r = 0, run_a = 0;
#pragma unroll
        for (int w = 0; w < kTileWarps; ++w) {
            const int vr = s_wrows[w][tid], va = s_wasg[w][tid];
            s_wrows[w][tid] = run_r;
            s_wasg[w][tid] = run_a;
            run_r += vr;
            run_a += va;
        }
    }

    // ---- cross-tile bases: need the predecessor's results
    pdl_wait();
    if (SMALL) {
        // rank r's row and assignment counts read together (one round trip), then reduced
        for (int r = warp; r < R; r += kTileWarps) {
            const int32_t *cr = ws.tile_rows + (int64_t)r * n_tiles;
            const int32_t *ca = ws.tile_asg + (int64_t)r * n_tiles;
            int tot[2] = {0, 0}, before[2] = {0, 0};
            for (int i = lane; i < n_tiles; i += 32) {
                const int vr = cr[i], va = ca[i];
                tot[0] += vr;
                tot[1] += va;
                before[0] += i < tile ? vr : 0;
                before[1] += i < tile ? va : 0;
            }
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const int t_all = __reduce_add_sync(0xffffffffu, tot[which]);
                const int t_before = __reduce_add_sync(0xffffffffu, before[which]);
                if (lane == 0) {
                    s_tot[which][r] = t_all;
                    s_before[which][r] = t_before;
                }
            }
        }
        if (tile == 0) {
            long long acc[kStatSlots] = {0, 0, 0, 0, 0, 0};
            for (int i = tid; i < n_tiles; i += kTile)
#pragma unroll
                for (int q = 0; q < kStatSlots; ++q) acc[q] += ws.tile_stats[(int64_t)i * kStatSlots + q];
#pragma unroll
            for (int q = 0; q < kStatSlots; ++q) {
                long long v = acc[q];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) s_stat[warp][q] = v;
            }
        }
    } else if (warp == 0) {
        for (int r = lane; r < R; r += 32) {
            s_tot[0][r] = ws.tot[r];
            s_tot[1][r] = ws.tot[R + r];
            s_before[0][r] = tile < n_tiles ? ws.tile_rows[(int64_t)r * n_tiles + tile] : 0;
            s_before[1][r] = tile < n_tiles ? ws.tile_asg[(int64_t)r * n_tiles + tile] : 0;
        }
    }
    __syncthreads();
    if (warp == 0)
        rank_bases(R, tile, s_tot[0], s_tot[1], s_before[0], s_before[1], s_rbase, s_abase,
                   rank_counts, rank_offsets, asg_offsets, stats);
    if (SMALL && tile == 0 && tid == 0) {
        long long tot[kStatSlots] = {0, 0, 0, 0, 0, 0};
        for (int w = 0; w < kTileWarps; ++w)
            for (int q = 0; q < kStatSlots; ++q) tot[q] += s_stat[w][q];
        stats[COACT_STAT_NAIVE_ROWS] = N * K;
        stats[COACT_STAT_REMOTE_ROWS] = tot[TS_REMOTE_ROWS];
        stats[COACT_STAT_CROSSNODE_ROWS] = tot[TS_XNODE_ROWS];
        stats[COACT_STAT_NODE_DEDUP_ROWS] = tot[TS_NODE_ROWS];
        stats[COACT_STAT_LOCAL_ASG] = tot[TS_LOCAL_ASG];
        stats[COACT_STAT_REMOTE_ASG] = tot[TS_VALID_ASG] - tot[TS_LOCAL_ASG];
        stats[COACT_STAT_CROSSNODE_ASG] = tot[TS_XNODE_ASG];
    }
    __syncthreads();

    if (t < N) {
        if (!ok) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                send_row[t * K + j] = -1;
                comb_row[t * K + j] = -1;
            }
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int r = rk[j];
                unsigned km = 0;
#pragma unroll
                for (int jj = 0; jj < K; ++jj) km |= (unsigned)(rk[jj] == r) << jj;
                const unsigned below = km & ((1u << j) - 1);
                const uint32_t pj = (s_pre[j / 2][tid] >> (16 * (j % 2))) & 0xffffu;
                comb_row[t * K + j] = s_abase[r] + s_wasg[warp][r] + (int)(pj >> 8) + __popc(below);
                int sr = -1;
                if (below == 0) {
                    const int64_t row = (int64_t)s_rbase[r] + s_wrows[warp][r] + (int)(pj & 0xff);
                    if (row < cap) {
                        row_token[row] = (int32_t)t;
                        row_kmask[row] = (uint8_t)km;
                        sr = (int)row;
                    } else {
                        flags |= COACT_EFLAG_CAPACITY;
                    }
                }
                send_row[t * K + j] = sr;
            }
        }
        if (rank_mask) rank_mask[t] = mask;
    }
    raise_flag_warp(err, flags);
    if (src_dst) {
        for (int i = tid; i < R * R; i += kTile) {
            const int v = s_sd[i];
            if (v) atomicAdd(src_dst + i, v);
        }
    }
}

#ifndef COACT_PLAN_SMALL_MAX
#define COACT_PLAN_SMALL_MAX 4096  // R * n_tiles up to which the scan kernel is skipped
#endif

template <int K, int NW>
int launch_plan(const int32_t *ids, int64_t N, int E, const int32_t *expert_rank,
                const int32_t *slot_rank, int R,
                const int32_t *rank_node, int n_nodes, const int32_t *src_rank,
                int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                uint64_t *rank_mask, int32_t *row_token, uint8_t *row_kmask, int64_t cap,
                int32_t *send_row, int32_t *comb_row, int64_t *stats, int32_t *src_dst,
                const Workspace &ws, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
    (void)di;
    const int n_tiles = (int)ceil_div(N, kTile);
    const size_t sd_smem = src_dst ? sizeof(int) * R * R : 0;
    auto *rm = reinterpret_cast<unsigned long long *>(rank_mask);
    if (n_tiles > 0 && (int64_t)R * n_tiles <= COACT_PLAN_SMALL_MAX) {
        if (int s = launch_pdl(k_plan_tiles<K, NW>, n_tiles, kTile, 0, st, ids, N, E, expert_rank, slot_rank, R,
                               rank_node, n_nodes, src_rank, n_tiles, ws, src_dst, err))
            return s;
        return launch_pdl(k_plan_scatter<K, true, NW>, n_tiles, kTile, sd_smem, st, ids, N, E,
                          expert_rank, slot_rank, R, src_rank, n_tiles, ws, rank_counts, rank_offsets,
                          asg_offsets, rm, row_token, row_kmask, cap, send_row, comb_row, stats,
                          src_dst, err);
    }
    if (n_tiles > 0)
        if (int s = launch_pdl(k_plan_tiles<K, NW>, n_tiles, kTile, 0, st, ids, N, E, expert_rank, slot_rank, R,
                               rank_node, n_nodes, src_rank, n_tiles, ws, src_dst, err))
            return s;
    if (int s = launch_pdl(k_plan_scan, R + 1, kScanThreads, 0, st, N, K, R, n_tiles, ws, stats,
                           n_tiles > 0 ? nullptr : src_dst))
        return s;
    return launch_pdl(k_plan_scatter<K, false, NW>, std::max(n_tiles, 1), kTile, sd_smem, st, ids, N,
                      E, expert_rank, slot_rank, R, src_rank, n_tiles, ws, rank_counts, rank_offsets,
                      asg_offsets, rm, row_token, row_kmask, cap, send_row, comb_row, stats,
                      src_dst, err);
}

// R <= 32: one 32-bit word per bit plane; R <= 64: two.
template <int K>
int launch_plan_any(const int32_t *ids, int64_t N, int E, const int32_t *expert_rank,
                    const int32_t *slot_rank, int R, const int32_t *rank_node, int n_nodes,
                    const int32_t *src_rank, int32_t *rank_counts, int32_t *rank_offsets,
                    int32_t *asg_offsets, uint64_t *rank_mask, int32_t *row_token,
                    uint8_t *row_kmask, int64_t cap, int32_t *send_row, int32_t *comb_row,
                    int64_t *stats, int32_t *src_dst, const Workspace &ws, int32_t *err,
                    cudaStream_t st, const DeviceInfo &di) {
    auto *run = R > 32 ? launch_plan<K, 2> : launch_plan<K, 1>;
    return run(ids, N, E, expert_rank, slot_rank, R, rank_node, n_nodes, src_rank, rank_counts,
               rank_offsets, asg_offsets, rank_mask, row_token, row_kmask, cap, send_row,
               comb_row, stats, src_dst, ws, err, st, di);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" size_t plan_dispatch_workspace_bytes(int64_t N, int k, int E, int R) {
    (void)k;
    (void)E;
    if (N < 0 || R < 1 || R > COACT_MAX_R) return 0;
    return workspace_layout(N, R, nullptr, nullptr);
}

namespace coact {
namespace {

// plan_dispatch and plan_dispatch_slots: the rank of each slot comes from expert_rank
// (per expert, per_slot false) or slot_rank (per slot, per_slot true).
int plan_entry(const int32_t *ids, int64_t N, int k, int E, const int32_t *expert_rank,
               const int32_t *slot_rank, bool per_slot, int R, const int32_t *rank_node, int n_nodes,
               const int32_t *src_rank, int32_t *rank_counts, int32_t *rank_offsets,
               int32_t *asg_offsets, uint64_t *rank_mask, int32_t *row_token, uint8_t *row_kmask,
               int64_t row_capacity, int32_t *send_row, int32_t *comb_row, int64_t *stats,
               int32_t *src_dst, void *workspace, size_t workspace_bytes, int32_t *err_flag,
               coact_stream_t stream) {
    if (N < 0 || row_capacity < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R)
        return COACT_ERR_UNSUPPORTED;
    if (rank_node && (n_nodes < 1 || n_nodes > 64)) return COACT_ERR_UNSUPPORTED;
    if (!rank_node) n_nodes = 1;
    if (N > (int64_t)INT32_MAX / k || row_capacity > (int64_t)INT32_MAX) return COACT_ERR_UNSUPPORTED;
    if (per_slot ? (N > 0 && !slot_rank) : !expert_rank) return COACT_ERR_INVALID;
    if (!rank_counts || !rank_offsets || !asg_offsets || !stats) return COACT_ERR_INVALID;
    if (N > 0 && (!ids || !send_row || !comb_row)) return COACT_ERR_INVALID;
    if (row_capacity > 0 && (!row_token || !row_kmask)) return COACT_ERR_INVALID;
    const size_t need = workspace_layout(N, R, nullptr, nullptr);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return COACT_ERR_WORKSPACE;
    Workspace ws;
    workspace_layout(N, R, &ws, workspace);
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_PLAN_CASE(KK)                                                                        \
    case KK:                                                                                       \
        return launch_plan_any<KK>(ids, N, E, expert_rank, slot_rank, R, rank_node, n_nodes, src_rank, \
                               rank_counts, rank_offsets, asg_offsets, rank_mask, row_token,       \
                               row_kmask, row_capacity, send_row, comb_row, stats, src_dst, ws,    \
                               err_flag, st, di);
    switch (k) {
        COACT_PLAN_CASE(1)
        COACT_PLAN_CASE(2)
        COACT_PLAN_CASE(3)
        COACT_PLAN_CASE(4)
        COACT_PLAN_CASE(5)
        COACT_PLAN_CASE(6)
        COACT_PLAN_CASE(7)
        COACT_PLAN_CASE(8)
    }
#undef COACT_PLAN_CASE
    return COACT_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace coact

extern "C" int plan_dispatch(const int32_t *ids, int64_t N, int k, int E, const int32_t *expert_rank,
                             int R, const int32_t *rank_node, int n_nodes, const int32_t *src_rank,
                             int32_t *rank_counts, int32_t *rank_offsets, int32_t *asg_offsets,
                             uint64_t *rank_mask, int32_t *row_token, uint8_t *row_kmask,
                             int64_t row_capacity, int32_t *send_row, int32_t *comb_row,
                             int64_t *stats, int32_t *src_dst, void *workspace,
                             size_t workspace_bytes, int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("plan_dispatch");
    return plan_entry(ids, N, k, E, expert_rank, nullptr, false, R, rank_node, n_nodes, src_rank,
                      rank_counts, rank_offsets, asg_offsets, rank_mask, row_token, row_kmask,
                      row_capacity, send_row, comb_row, stats, src_dst, workspace, workspace_bytes,
                      err_flag, stream);
}

extern "C" int plan_dispatch_slots(const int32_t *ids, int64_t N, int k, int E,
                                   const int32_t *slot_rank, int R, const int32_t *rank_node,
                                   int n_nodes, const int32_t *src_rank, int32_t *rank_counts,
                                   int32_t *rank_offsets, int32_t *asg_offsets, uint64_t *rank_mask,
                                   int32_t *row_token, uint8_t *row_kmask, int64_t row_capacity,
                                   int32_t *send_row, int32_t *comb_row, int64_t *stats,
                                   int32_t *src_dst, void *workspace, size_t workspace_bytes,
                                   int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("plan_dispatch_slots");
    return plan_entry(ids, N, k, E, nullptr, slot_rank, true, R, rank_node, n_nodes,
                      src_rank, rank_counts, rank_offsets, asg_offsets, rank_mask, row_token,
                      row_kmask, row_capacity, send_row, comb_row, stats, src_dst, workspace,
                      workspace_bytes, err_flag, stream);
}

// ------------------------------------------------------------------ no-allocation variant
//
// plan_dispatch_noalloc: plan_dispatch for callers that cannot allocate device memory
// -- code running inside a runtime that owns every byte of device memory through its
// own pool or a fixed memory plan and forbids stray allocations, or a latency-critical
// caller that cannot afford cudaMalloc's implicit device-wide synchronisation.  Its
// scratch is a file-scope device array sized for COACT_NOALLOC_MAX_TOKENS tokens and
// COACT_MAX_R ranks, which every GPU that loads this library holds until exit.

namespace coact {
namespace {

constexpr size_t align256c(size_t b) { return (b + 255) & ~size_t(255); }
constexpr int64_t kNoallocTiles = (COACT_NOALLOC_MAX_TOKENS + kTile - 1) / kTile;
constexpr size_t kNoallocScratchBytes =
    2 * align256c(sizeof(int32_t) * (size_t)COACT_MAX_R * kNoallocTiles) +
    align256c(sizeof(int64_t) * kStatSlots * (size_t)kNoallocTiles) +
    align256c(sizeof(int32_t) * 2 * (size_t)COACT_MAX_R);

// In host code this name is only a host-side stand-in, never a device address: the
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_plan_scratch[kNoallocScratchBytes];

struct ScratchAddr {
    std::mutex m;
    unsigned long long ctx = 0;  // context the address belongs to
    void *addr = nullptr;
};
ScratchAddr g_plan_scratch_addr[kMaxDevices];

// Device address of g_plan_scratch in the current context of the current device, looked
// up once per device and again whenever the context changes (a device reset unloads the
// module, and the array may come back at another address).
int noalloc_scratch(const DeviceInfo &di, void **out) {
    ScratchAddr &slot = g_plan_scratch_addr[di.device];
    std::lock_guard<std::mutex> lock(slot.m);
    if (!slot.addr || slot.ctx != di.ctx) {
        void *p = nullptr;
        if (cudaError_t e = cudaGetSymbolAddress(&p, g_plan_scratch)) return cuda_fail(e);
        if (!p) return COACT_ERR_CUDA;
        slot.addr = p;
        slot.ctx = di.ctx;
    }
    *out = slot.addr;
    return COACT_OK;
}

}  // namespace
}  // namespace coact

extern "C" int plan_dispatch_noalloc(const int32_t *ids, int64_t N, int k, int E,
                                     const int32_t *expert_rank, int R, const int32_t *rank_node,
                                     int n_nodes, const int32_t *src_rank, int32_t *rank_counts,
                                     int32_t *rank_offsets, int32_t *asg_offsets,
                                     uint64_t *rank_mask, int32_t *row_token, uint8_t *row_kmask,
                                     int64_t row_capacity, int32_t *send_row, int32_t *comb_row,
                                     int64_t *stats, int32_t *src_dst, int32_t *err_flag,
                                     coact_stream_t stream) {
    COACT_RANGE("plan_dispatch_noalloc");
    if (N < 0 || row_capacity < 0) return COACT_ERR_INVALID;
    if (N > COACT_NOALLOC_MAX_TOKENS) return COACT_ERR_UNSUPPORTED;
    if (k < 1 || k > COACT_MAX_K || E < 2 || E > COACT_MAX_E || R < 1 || R > COACT_MAX_R)
        return COACT_ERR_UNSUPPORTED;
    if (rank_node && (n_nodes < 1 || n_nodes > 64)) return COACT_ERR_UNSUPPORTED;
    if (!rank_node) n_nodes = 1;
    if (N > (int64_t)INT32_MAX / k || row_capacity > (int64_t)INT32_MAX) return COACT_ERR_UNSUPPORTED;
    if (!expert_rank || !rank_counts || !rank_offsets || !asg_offsets || !stats)
        return COACT_ERR_INVALID;
    if (N > 0 && (!ids || !send_row || !comb_row)) return COACT_ERR_INVALID;
    if (row_capacity > 0 && (!row_token || !row_kmask)) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    void *scratch = nullptr;
    if (int s = noalloc_scratch(di, &scratch)) return s;
    if (workspace_layout(N, R, nullptr, nullptr) > kNoallocScratchBytes) return COACT_ERR_UNSUPPORTED;
    Workspace ws;
    workspace_layout(N, R, &ws, scratch);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define COACT_PLAN_NOALLOC_CASE(KK)                                                                \
    case KK:                                                                                       \
        return launch_plan_any<KK>(ids, N, E, expert_rank, nullptr, R, rank_node, n_nodes, src_rank,   \
                               rank_counts, rank_offsets, asg_offsets, rank_mask, row_token,       \
                               row_kmask, row_capacity, send_row, comb_row, stats, src_dst, ws,    \
                               err_flag, st, di);
    switch (k) {
        COACT_PLAN_NOALLOC_CASE(1)
        COACT_PLAN_NOALLOC_CASE(2)
        COACT_PLAN_NOALLOC_CASE(3)
        COACT_PLAN_NOALLOC_CASE(4)
        COACT_PLAN_NOALLOC_CASE(5)
        COACT_PLAN_NOALLOC_CASE(6)
        COACT_PLAN_NOALLOC_CASE(7)
        COACT_PLAN_NOALLOC_CASE(8)
    }
#undef COACT_PLAN_NOALLOC_CASE
    return COACT_ERR_UNSUPPORTED;
}
