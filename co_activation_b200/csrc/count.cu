// coact_count: expert co-activation pair counts and per-expert loads.
//
// Cobalt (arxivdaily 2609.36959), English abstract: pairs of experts co-activated by
// single tokens and per-expert workload statistics feed the expert layout planner.
// Zyphra (arxivdaily 2610.09372), English abstract: a few expert pairs are selected
// together by many tokens; layer-to-layer correlation (cross mode).
//
// Two kernels:
//  * k_count_smem -- each block privatises the strict upper triangle of the E x E count
//    matrix (E*(E-1)/2 u32 bins, 130 KB at E = 256) plus E load bins in shared memory,
//    adds its tokens' pairs with shared atomics, then flushes every non-zero bin to both
//    halves of the int64 matrix with one global atomic each.  Used when the triangle
//    fits and each block sees enough pairs to amortise its zero/flush pass.  (A
//    warp-aggregated variant -- lanes with the same bin merged by __match_any_sync --
//    exists as AGG = true; on B200 it measured 1.4-3x slower than plain shared atomics
//    even on the Zipf-skewed configurations, so it is off.)
//  * k_count_global -- one global 64-bit atomic per ordered pair, for E too large for
//    shared memory or inputs too small to amortise a private histogram.
// Cross mode (ids2 != NULL) counts ids x ids2 into an E x E2 matrix, privatised in
// shared memory when E*E2 bins fit.
#include <algorithm>

#include "common.cuh"

namespace coact {
namespace {

constexpr int kCountThreads = 1024;
constexpr int kNone = -1;
using ull = unsigned long long;

__device__ __forceinline__ int tri_index(int a, int b, int E) {
    // strict upper triangle, row-major: row a starts at a*(2E-a-1)/2
    const int lo = min(a, b), hi = max(a, b);
    return lo * (2 * E - lo - 1) / 2 + (hi - lo - 1);
}

template <int K, bool AGG>
__global__ void __launch_bounds__(kCountThreads)
    k_count_smem(const int32_t *__restrict__ ids, int64_t N, int E, ull *__restrict__ pair,
                 ull *__restrict__ loads, int32_t *__restrict__ err) {
    extern __shared__ uint32_t sh[];
    const int nbins = E * (E - 1) / 2;
    uint32_t *tri = sh;
    uint32_t *sload = sh + nbins;
    for (int i = threadIdx.x; i < nbins + E; i += blockDim.x) sh[i] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    const int lane = threadIdx.x & 31;
    int flags = 0;
    // The warp takes 32 consecutive tokens per step, so the loop trip count is
    // warp-uniform and the warp-collective match below sees all 32 lanes.
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = gwarp * 32; base < N; base += nwarps * 32) {
        const int64_t t = base + lane;
        int e[K];
        bool ok = false;
        if (t < N) {
            const int f = load_ids<K>(ids, t, E, e);
            flags |= f;
            ok = (f == 0);
        }
        if (ok) {
#pragma unroll
            for (int j = 0; j < K; ++j) atomicAdd(&sload[e[j]], 1u);
        }
#pragma unroll
        for (int j = 0; j < K; ++j)
#pragma unroll
            for (int jj = j + 1; jj < K; ++jj) {
                const int key = ok ? tri_index(e[j], e[jj], E) : kNone;
                if (AGG) {
                    const unsigned m = __match_any_sync(0xffffffffu, key);
                    if (key != kNone && lane == __ffs(m) - 1) atomicAdd(&tri[key], (unsigned)__popc(m));
                } else if (key != kNone) {
                    atomicAdd(&tri[key], 1u);
                }
            }
    }
    raise_flag_warp(err, flags);
    __syncthreads();

    // Flush: every ordered pair (a, b), a != b, takes the count of its triangle bin.
    const int EE = E * E;
    for (int i = threadIdx.x; i < EE; i += blockDim.x) {
        const int a = i / E, b = i - a * E;
        if (a == b) continue;
        const uint32_t v = tri[tri_index(a, b, E)];
        if (v) atomicAdd(pair + i, (ull)v);
    }
    if (loads)
        for (int i = threadIdx.x; i < E; i += blockDim.x) {
            const uint32_t v = sload[i];
            if (v) atomicAdd(loads + i, (ull)v);
        }
}

template <int K>
__global__ void __launch_bounds__(256)
    k_count_global(const int32_t *__restrict__ ids, int64_t N, int E, ull *__restrict__ pair,
                   ull *__restrict__ loads, int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < N; t += stride) {
        int e[K];
        const int f = load_ids<K>(ids, t, E, e);
        flags |= f;
        if (f) continue;
#pragma unroll
        for (int j = 0; j < K; ++j) {
            if (loads) atomicAdd(loads + e[j], 1ull);
#pragma unroll
            for (int jj = 0; jj < K; ++jj)
                if (jj != j) atomicAdd(pair + (int64_t)e[j] * E + e[jj], 1ull);
        }
    }
    if (flags && err) atomicOr(err, flags);
}

// Cross-layer counts: C[a*E2 + b] += 1 for every slot pair of ids (K slots) x ids2
// (k2 slots).  SMEM = privatised E x E2 histogram in shared memory.
template <int K, bool SMEM>
__global__ void __launch_bounds__(512)
    k_count_cross(const int32_t *__restrict__ ids, const int32_t *__restrict__ ids2, int k2,
                  int64_t N, int E, int E2, ull *__restrict__ C, ull *__restrict__ loads,
                  int32_t *__restrict__ err) {
    extern __shared__ uint32_t sh[];
    const int nb = SMEM ? E * E2 : 0;
    if (SMEM)
        for (int i = threadIdx.x; i < nb + E; i += blockDim.x) sh[i] = 0;
    pdl_wait();
    pdl_trigger();
    if (SMEM) __syncthreads();
    int flags = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < N; t += stride) {
        int e[K];
        int f = load_ids<K>(ids, t, E, e);
        int e2[COACT_MAX_K];
#pragma unroll
        for (int j = 0; j < COACT_MAX_K; ++j) {
            e2[j] = j < k2 ? __ldg(ids2 + t * k2 + j) : 0;
            if (j < k2 && (unsigned)e2[j] >= (unsigned)E2) f |= COACT_EFLAG_ID_RANGE;
        }
#pragma unroll
        for (int j = 1; j < COACT_MAX_K; ++j)
#pragma unroll
            for (int jj = 0; jj < j; ++jj)
                if (j < k2 && e2[j] == e2[jj]) f |= COACT_EFLAG_DUP_ID;
        flags |= f;
        if (f) continue;
#pragma unroll
        for (int j = 0; j < K; ++j) {
            if (loads) {
                if (SMEM) atomicAdd(&sh[nb + e[j]], 1u);
                else atomicAdd(loads + e[j], 1ull);
            }
#pragma unroll
            for (int jj = 0; jj < COACT_MAX_K; ++jj) {
                if (jj >= k2) break;
                const int idx = e[j] * E2 + e2[jj];
                if (SMEM) atomicAdd(&sh[idx], 1u);
                else atomicAdd(C + idx, 1ull);
            }
        }
    }
    if (flags && err) atomicOr(err, flags);
    if (SMEM) {
        __syncthreads();
        for (int i = threadIdx.x; i < nb; i += blockDim.x) {
            const uint32_t v = sh[i];
            if (v) atomicAdd(C + i, (ull)v);
        }
        if (loads)
            for (int i = threadIdx.x; i < E; i += blockDim.x) {
                const uint32_t v = sh[nb + i];
                if (v) atomicAdd(loads + i, (ull)v);
            }
    }
}

// Blocks for a privatised histogram: enough pairs per block to amortise the zero and
// flush passes over `bins` bins, capped by what fits on the GPU at once.
#ifndef COACT_COUNT_MIN_PER_BLOCK
#define COACT_COUNT_MIN_PER_BLOCK 2048
#endif
#ifndef COACT_COUNT_BINS_FACTOR
#define COACT_COUNT_BINS_FACTOR 1
#endif
int hist_blocks(int64_t N, int64_t pairs_per_token, int64_t bins, int resident) {
    const int64_t total = N * pairs_per_token;
    const int64_t per_block =
        std::max<int64_t>(COACT_COUNT_BINS_FACTOR * bins, COACT_COUNT_MIN_PER_BLOCK);
    const int64_t want = std::max<int64_t>(1, ceil_div(total, per_block));
    return (int)std::min<int64_t>(want, resident);
}

template <int K>
int count_self(const int32_t *ids, int64_t N, int E, ull *pair, ull *loads, int32_t *err,
               cudaStream_t st, const DeviceInfo &di) {
    const int64_t nbins = (int64_t)E * (E - 1) / 2;
    const size_t smem = (size_t)(nbins + E) * sizeof(uint32_t);
    const int64_t ppt = (int64_t)K * (K - 1) / 2;
    bool use_smem = K > 1 && smem <= (size_t)di.smem_optin;
    // tiny inputs: a private histogram would cost more to clear than to fill
    if (N * ppt < 2 * nbins) use_smem = false;
#if defined(COACT_COUNT_PATH)
    use_smem = K > 1 && smem <= (size_t)di.smem_optin && COACT_COUNT_PATH != 0;  // experiments
#endif
#ifndef COACT_COUNT_AGG
#define COACT_COUNT_AGG false  // measured on B200: match_any costs more than it saves
#endif
    if (use_smem) {
        auto kern = k_count_smem<K, COACT_COUNT_AGG>;
        static SmemOptIn opt;
        if (int s = ensure_smem(kern, smem, opt, di)) return s;
        const int per_sm = blocks_per_sm(kCountThreads, smem, di);
        const int blocks = hist_blocks(N, ppt, nbins, per_sm * di.sm_count);
        return launch_pdl(kern, blocks, kCountThreads, smem, st, ids, N, E, pair, loads, err);
    } else {
        const int blocks = (int)std::min<int64_t>(ceil_div(N, 256), (int64_t)di.sm_count * 8);
        return launch_pdl(k_count_global<K>, blocks, 256, 0, st, ids, N, E, pair, loads, err);
    }
}

template <int K>
int count_cross(const int32_t *ids, const int32_t *ids2, int k2, int64_t N, int E, int E2,
                ull *C, ull *loads, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
    const int64_t nb = (int64_t)E * E2;
    const size_t smem = (size_t)(nb + E) * sizeof(uint32_t);
    const bool use_smem = smem <= (size_t)di.smem_optin && N * K * k2 >= 2 * nb;
    if (use_smem) {
        auto kern = k_count_cross<K, true>;
        static SmemOptIn opt;
        if (int s = ensure_smem(kern, smem, opt, di)) return s;
        const int per_sm = blocks_per_sm(512, smem, di);
        const int blocks = hist_blocks(N, (int64_t)K * k2, nb, per_sm * di.sm_count);
        return launch_pdl(kern, blocks, 512, smem, st, ids, ids2, k2, N, E, E2, C, loads, err);
    } else {
        const int blocks = (int)std::min<int64_t>(ceil_div(N, 512), (int64_t)di.sm_count * 4);
        return launch_pdl(k_count_cross<K, false>, blocks, 512, 0, st, ids, ids2, k2, N, E, E2, C,
                          loads, err);
    }
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int coact_count(const int32_t *ids, int64_t N, int k, int E, const int32_t *ids2, int k2,
                           int E2, int64_t *pair, int64_t *loads, int32_t *err_flag,
                           coact_stream_t stream) {
    COACT_RANGE("coact_count");
    if (N < 0 || !pair || (N > 0 && !ids)) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K || E < 2 || E > COACT_MAX_E) return COACT_ERR_UNSUPPORTED;
    if (ids2 && (k2 < 1 || k2 > COACT_MAX_K || E2 < 2 || E2 > COACT_MAX_E))
        return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX / COACT_MAX_K) return COACT_ERR_UNSUPPORTED;
    if (N == 0) return COACT_OK;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    ull *P = reinterpret_cast<ull *>(pair);
    ull *L = reinterpret_cast<ull *>(loads);
#define COACT_COUNT_CASE(KK)                                                                 \
    case KK:                                                                                 \
        return ids2 ? count_cross<KK>(ids, ids2, k2, N, E, E2, P, L, err_flag, st, di)       \
                    : count_self<KK>(ids, N, E, P, L, err_flag, st, di);
    switch (k) {
        COACT_COUNT_CASE(1)
        COACT_COUNT_CASE(2)
        COACT_COUNT_CASE(3)
        COACT_COUNT_CASE(4)
        COACT_COUNT_CASE(5)
        COACT_COUNT_CASE(6)
        COACT_COUNT_CASE(7)
        COACT_COUNT_CASE(8)
    }
#undef COACT_COUNT_CASE
    return COACT_ERR_UNSUPPORTED;
}
