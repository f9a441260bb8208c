// predict_home: token shuffling's home-rank prediction.
//
// Zyphra (arxivdaily 2610.09372), English abstract: when sequence parallelism shards
// tokens across the EP group, each token is moved to the GPU predicted to hold its
// next-layer experts; the experts a token picks at one layer predict those at the next.
//
//   S[a][r]     = sum_{b : expert_rank2[b] == r} C12[a][b]      (k_rank_scores)
//   home[t]     = argmax_r sum_j S[ids1[t,j]][r], ties -> lowest r  (k_predict_home)
// Integer arithmetic throughout, so the result is exact and deterministic.
#include <algorithm>

#include "common.cuh"

namespace coact {
namespace {

__global__ void __launch_bounds__(256)
    k_rank_scores(const int64_t *__restrict__ C12, int E1, int E2,
                  const int32_t *__restrict__ expert_rank2, int R, int64_t *__restrict__ S,
                  int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)E1 * R) return;
    const int a = (int)(i / R), r = (int)(i - (int64_t)a * R);
    int64_t s = 0;
    int flags = 0;
    for (int b = 0; b < E2; ++b) {
        const int rb = __ldg(expert_rank2 + b);
        if ((unsigned)rb >= (unsigned)R) flags = COACT_EFLAG_ID_RANGE;
        if (rb == r) s += __ldg(C12 + (int64_t)a * E2 + b);
    }
    S[i] = s;
    if (flags && r == 0) raise_flag(err, flags);
}

template <int K>
__global__ void __launch_bounds__(256)
    k_predict_home(const int32_t *__restrict__ ids1, int64_t N, int E1,
                   const int64_t *__restrict__ S, int R, int32_t *__restrict__ home,
                   int32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    int flags = 0;
    if (t < N) {
        int e[K];
        flags = load_ids<K>(ids1, t, E1, e);
        int best = -1;
        if (!flags) {
            int64_t best_score = -1;
            for (int r = 0; r < R; ++r) {
                int64_t sc = 0;
#pragma unroll
                for (int j = 0; j < K; ++j) sc += __ldg(S + (int64_t)e[j] * R + r);
                if (sc > best_score) {
                    best_score = sc;
                    best = r;
                }
            }
        }
        home[t] = best;
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" size_t predict_home_workspace_bytes(int E1, int R) {
    if (E1 < 1 || R < 1) return 0;
    return sizeof(int64_t) * (size_t)E1 * (size_t)R;
}

extern "C" int predict_home(const int32_t *ids1, int64_t N, int k1, int E1, const int64_t *C12,
                            int E2, const int32_t *expert_rank2, int R, int32_t *home,
                            void *workspace, size_t workspace_bytes, int32_t *err_flag,
                            coact_stream_t stream) {
    COACT_RANGE("predict_home");
    if (N < 0) return COACT_ERR_INVALID;
    if (k1 < 1 || k1 > COACT_MAX_K || E1 < 2 || E1 > COACT_MAX_E || E2 < 2 || E2 > COACT_MAX_E ||
        R < 1 || R > COACT_MAX_R)
        return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX / k1) return COACT_ERR_UNSUPPORTED;
    if (!C12 || !expert_rank2 || (N > 0 && (!ids1 || !home))) return COACT_ERR_INVALID;
    if (!workspace || workspace_bytes < predict_home_workspace_bytes(E1, R) || !aligned16(workspace))
        return COACT_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int64_t *S = static_cast<int64_t *>(workspace);
    const int64_t cells = (int64_t)E1 * R;
    if (int s = launch_pdl(k_rank_scores, (int)ceil_div(cells, 256), 256, 0, st, C12, E1, E2,
                           expert_rank2, R, S, err_flag))
        return s;
    if (N == 0) return COACT_OK;
    const int blocks = (int)ceil_div(N, 256);
#define COACT_PREDICT_CASE(KK)                                                                   \
    case KK:                                                                                     \
        return launch_pdl(k_predict_home<KK>, blocks, 256, 0, st, ids1, N, E1, S, R, home,        \
                          err_flag);
    switch (k1) {
        COACT_PREDICT_CASE(1)
        COACT_PREDICT_CASE(2)
        COACT_PREDICT_CASE(3)
        COACT_PREDICT_CASE(4)
        COACT_PREDICT_CASE(5)
        COACT_PREDICT_CASE(6)
        COACT_PREDICT_CASE(7)
        COACT_PREDICT_CASE(8)
    }
#undef COACT_PREDICT_CASE
    return COACT_ERR_UNSUPPORTED;
}
