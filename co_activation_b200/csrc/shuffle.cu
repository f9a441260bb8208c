// shuffle_reduce_scatter: token shuffling fused into the post-attention reduce-scatter.
//
// Zyphra (arxivdaily 2610.09372), English abstract: when sequence parallelism shards the
// tokens across the EP group, each token is moved to the GPU predicted to hold its
// next-layer experts during the reduce-scatter that follows attention.  The P ranks of
// the group each hold a partial attention output for all N tokens; rank r's output rows
// are the tokens whose predicted home is r (row_token: the dispatch plan of every token
// to its home rank alone, i.e. grouped by rank in ascending token order), each the sum of
// the P partial rows:
//   out[i] = sum over q = 0..P-1 of part_q[row_token[i]]   (fp32 adds in rank order, +0)
// then fp32 or bf16 round-to-nearest-even.  On a GPU group, part_bases holds the peers'
// partial buffers (NVLink-mapped, e.g. symmetric memory) and every rank reads its own
// rows from every peer; on one GPU, P local buffers.  Plain 16-byte loads through the
// base pointers: no TMA multicast, no waits between ranks (the caller's barrier orders
// the partials' writes before this kernel).
//
// k_shuffle_reduce: one warp per output row; each lane owns 8 hidden elements per 16-byte
// column chunk and keeps U chunks x G partial rows of loads in flight, adding the groups
// of G partials in rank order.  HBM traffic: P*n_out*H*2 read + n_out*H*(2|4) written.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace coact {
namespace {

template <int U, int G, bool F32>
__global__ void __launch_bounds__(256)
    k_shuffle_reduce(const unsigned long long *__restrict__ bases, int P, int64_t N, int64_t H16,
                     const int32_t *__restrict__ row_token, int64_t n_out, void *__restrict__ out,
                     int32_t *__restrict__ err) {
    __shared__ unsigned long long s_base[COACT_MAX_R];
    pdl_wait();
    pdl_trigger();
    int flags = 0;
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
        unsigned long long b = __ldg(bases + q);
        if (b == 0 || (b & 15u)) {          // absent or misaligned partial: skipped, flagged
            if (blockIdx.x == 0) flags |= COACT_EFLAG_ROW_RANGE;
            b = 0;
        }
        s_base[q] = b;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = gwarp; i < n_out; i += nwarps) {
        const int t = __ldg(row_token + i);
        const bool ok = t >= 0 && (int64_t)t < N;
        if (!ok) flags |= COACT_EFLAG_ROW_RANGE;
        for (int64_t c0 = 0; c0 < H16; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[u][e] = 0.0f;
            if (ok) {
                for (int q0 = 0; q0 < P; q0 += G) {
                    uint4 v[U][G];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int64_t c = c0 + u * 32 + lane;
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const int q = q0 + g;
                            if (c < H16 && q < P && s_base[q])
                                v[u][g] = ld_stream(reinterpret_cast<const uint4 *>(s_base[q]) +
                                                    (int64_t)t * H16 + c);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int64_t c = c0 + u * 32 + lane;
                        if (c >= H16) continue;
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const int q = q0 + g;
                            if (q >= P || !s_base[q]) continue;
                            const uint32_t w[4] = {v[u][g].x, v[u][g].y, v[u][g].z, v[u][g].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acc[u][2 * e] = __fadd_rn(acc[u][2 * e], bf16lo(w[e]));
                                acc[u][2 * e + 1] = __fadd_rn(acc[u][2 * e + 1], bf16hi(w[e]));
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + u * 32 + lane;
                if (c >= H16) continue;
                if (F32) {
                    float4 *o = reinterpret_cast<float4 *>(out) + (i * H16 + c) * 2;
                    __stcs(o, make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]));
                    __stcs(o + 1, make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]));
                } else {
                    uint4 p;
                    uint32_t *pw = &p.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h2 =
                            __floats2bfloat162_rn(acc[u][2 * e], acc[u][2 * e + 1]);
                        pw[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    st_stream(reinterpret_cast<uint4 *>(out) + i * H16 + c, p);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

}  // namespace
}  // namespace coact

using namespace coact;

extern "C" int shuffle_reduce_scatter(const uint64_t *part_bases, int P, int64_t N, int64_t H,
                                      const int32_t *row_token, int64_t n_out, void *out,
                                      int out_dtype, int32_t *err_flag, coact_stream_t stream) {
    COACT_RANGE("shuffle_reduce_scatter");
    if (N < 0 || H < 0 || n_out < 0) return COACT_ERR_INVALID;
    if (P < 1 || P > COACT_MAX_R || (out_dtype != 0 && out_dtype != 1)) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N > (int64_t)INT32_MAX) return COACT_ERR_UNSUPPORTED;
    if (n_out == 0 || H == 0) return COACT_OK;
    if (!part_bases || !row_token || !out) return COACT_ERR_INVALID;
    if (!aligned16(out)) return COACT_ERR_INVALID;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    const int64_t H16 = H / 8;
    const int blocks = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(n_out, 8), (int64_t)di.sm_count * 8));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto *b = reinterpret_cast<const unsigned long long *>(part_bases);
    return out_dtype
               ? launch_pdl(k_shuffle_reduce<2, 4, true>, blocks, 256, 0, st, b, P, N, H16,
                            row_token, n_out, out, err_flag)
               : launch_pdl(k_shuffle_reduce<2, 4, false>, blocks, 256, 0, st, b, P, N, H16,
                            row_token, n_out, out, err_flag);
}
