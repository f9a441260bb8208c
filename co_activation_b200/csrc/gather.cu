// dispatch_gather: fill the per-rank send buffers, token-major.
//
// Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English
// abstracts: tokens are exchanged by all-to-all so each reaches the ranks that hold its
// experts -- with the deduplicated dispatcher, each rank once.  Here a rank's send
// segment is a region of this GPU's memory.
//
// Each x row is read from HBM once and written to every distinct destination row, so
// the algorithmic traffic is (N + D) * H * 2 bytes (+ N*k*4 for send_row).
//  * k_gather_v16 (default) -- one warp per token: vector loads of the x row into
//    registers, then streaming stores of them to each destination row.  Chunks are 32
//    bytes (one 256-bit access per lane) when the rows and both buffers are 32-byte
//    aligned, else 16 bytes; 2 (resp. 4) chunks per lane in flight on long rows.  The
//    kernel is specialised per k: a token's k destination rows are resolved once with k
//    shuffles and the store loop is unrolled and warp-uniform (no per-chunk shuffle or
//    data-dependent loop, which kept the MIO queue full).  The grid has one warp per
//    token up to 128 CTAs of 8 warps per SM (3-6 resident): tokens have different
//    fan-outs, and with one token per warp the CTA scheduler balances them to the end,
//    where a grid-stride loop over several tokens per warp leaves a tail.  Measured on
//    B200, 131,072 tokens of 14 KB rows, k = 8 (D = 4.33 rows per token) in the step:
//    1,677 us with the earlier 16-byte kernel (one kernel for all k, 8 CTAs per SM),
//    1,591-1,607 us with this kernel at 16 CTAs per SM, 1,550 us with one token per warp.
//    As a build option (-DCOACT_GATHER_PREFETCH_BYTES), each warp can warm L2 with the x
//    rows it will copy first before its wait on the predecessor (bulk L2 prefetch); it
//    measured without gain on the current kernel and is off.
//  * k_gather_bulk (entry point dispatch_gather_tma) -- TMA bulk copies.  One warp per
//    CTA; lane 0 streams rows into a ring of shared-memory stages with cp.async.bulk
//    (global -> shared, completion on an mbarrier), then lanes j < k each issue the
//    cp.async.bulk store of the staged row to destination j.  No multicast: every load
//    reads this GPU's own memory once.  Measured on B200 it is 2-5% slower than the
//    vector path (4-14 KB rows), also next to a concurrent GEMM: the gather is bound by
//    HBM bandwidth, so its lighter SM footprint does not buy overlap.
// All mbarrier waits are bounded by a wall-clock limit; on expiry the kernel raises
// COACT_EFLAG_TIMEOUT, drains its own copies and returns.
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace coact {
namespace {

// ------------------------------------------------------------------ vector path

// One warp per token; Hv chunks of type V per row.  K > 0: the token's K destination
// rows are resolved once (K shuffles) and the store loop is unrolled and warp-uniform;
// K == 0: k destinations at run time, walked with a ballot mask.  n_prefetch: tokens
// [0, n_prefetch) have their x rows warmed into L2 before the wait on the predecessor
// (each warp its own tokens, in the order it copies them), so that while a
// latency-bound predecessor (the plan) runs, HBM already streams x.
template <int K, typename V, int UNROLL>
__global__ void __launch_bounds__(256)
    k_gather_v16(const V *__restrict__ x, int64_t N, int64_t Hv,
                 const int32_t *__restrict__ send_row, int k, V *__restrict__ send, int64_t cap,
                 int64_t n_prefetch, int32_t *__restrict__ err) {
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    if (lane == 0)
        for (int64_t t = gwarp; t < n_prefetch; t += nwarps)
            prefetch_l2_bulk(x + t * Hv, (uint32_t)(Hv * sizeof(V)));
    pdl_wait();
    pdl_trigger();
    const int kk = K > 0 ? K : k;
    int flags = 0;
    for (int64_t t = gwarp; t < N; t += nwarps) {
        // destinations: lane j < k reads send_row[t, j]
        int dl = -1;
        if (lane < kk) {
            dl = __ldg(send_row + t * kk + lane);
            if (dl >= 0 && (int64_t)dl >= cap) {
                flags |= COACT_EFLAG_ROW_RANGE;
                dl = -1;
            }
        }
        int d[K > 0 ? K : 1];
        if (K > 0) {
#pragma unroll
            for (int j = 0; j < (K > 0 ? K : 1); ++j) d[j] = __shfl_sync(0xffffffffu, dl, j);
        }
        const unsigned dmask = __ballot_sync(0xffffffffu, dl >= 0);
        const V *src = x + t * Hv + lane;
        for (int64_t c0 = 0; c0 < Hv; c0 += 32 * UNROLL) {
            V v[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                if (c0 + u * 32 + lane < Hv) v[u] = ld_chunk<V>(src + c0 + u * 32);
            if (K > 0) {
#pragma unroll
                for (int j = 0; j < (K > 0 ? K : 1); ++j) {
                    if (d[j] < 0) continue;
                    V *dst = send + (int64_t)d[j] * Hv + lane + c0;
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u)
                        if (c0 + u * 32 + lane < Hv) st_chunk(dst + u * 32, v[u]);
                }
            } else {
                unsigned m = dmask;
                while (m) {
                    const int j = __ffs(m) - 1;
                    m &= m - 1;
                    V *dst = send + (int64_t)__shfl_sync(0xffffffffu, dl, j) * Hv + lane + c0;
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u)
                        if (c0 + u * 32 + lane < Hv) st_chunk(dst + u * 32, v[u]);
                }
            }
        }
    }
    raise_flag_warp(err, flags);
}

// ------------------------------------------------------------------ bulk (TMA) path

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of the mbarrier; gives up after `limit_ns` of wall clock.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63) == 63 && globaltimer_ns() - t0 > limit_ns) return false;
    }
}

#if defined(COACT_GATHER_EVICT_FIRST)
// L2 policy for data touched exactly once (x rows, send rows): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
#endif

__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void *src, uint32_t bytes,
                                          uint32_t bar) {
#if defined(COACT_GATHER_EVICT_FIRST)
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(dst_smem),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy_evict_first())
        : "memory");
#else
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst_smem),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
#endif
}

__device__ __forceinline__ void bulk_store(void *dst, uint32_t src_smem, uint32_t bytes) {
#if defined(COACT_GATHER_EVICT_FIRST)
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(
                     dst),
                 "r"(src_smem), "r"(bytes), "l"(policy_evict_first())
                 : "memory");
#else
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(src_smem), "r"(bytes)
                 : "memory");
#endif
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate copy
constexpr int kBulkHeader = 128;                   // mbarriers live in the first 128 bytes

// One warp per CTA.  Token i of this CTA is t = blockIdx.x + i * gridDim.x and uses
// stage i % S.  Lane 0 owns the mbarriers and the loads; lane j < k owns the store of
// destination j and its bulk groups.
template <int S>
__global__ void __launch_bounds__(32)
    k_gather_bulk(const uint16_t *__restrict__ x, int64_t N, uint32_t row_bytes,
                  const int32_t *__restrict__ send_row, int k, uint16_t *__restrict__ send,
                  int64_t cap, int32_t *__restrict__ err) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x;
    const uint32_t bars = smem_u32(smem);
    const uint32_t bufs = smem_u32(smem + kBulkHeader);
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t n_mine = N > first ? (N - 1 - first) / step + 1 : 0;
    const char *xb = reinterpret_cast<const char *>(x);
    char *sb = reinterpret_cast<char *>(send);

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) mbar_init(bars + 8 * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
        for (int64_t i = 0; i < n_mine && i < S; ++i) {
            const uint32_t bar = bars + 8 * (uint32_t)i;
            mbar_expect_tx(bar, row_bytes);
            bulk_load(bufs + (uint32_t)i * row_bytes, xb + (first + i * step) * (int64_t)row_bytes,
                      row_bytes, bar);
        }
    }
    __syncwarp();

    int flags = 0;
    int64_t loaded = n_mine < S ? n_mine : S;  // tokens whose load was issued
    int dnext = (lane < k && n_mine > 0) ? __ldg(send_row + first * k + lane) : -1;
    int64_t i = 0;
    for (; i < n_mine; ++i) {
        const int s = (int)(i % S);
        const uint32_t parity = (uint32_t)((i / S) & 1);
        const int d = dnext;
        if (lane < k && i + 1 < n_mine) dnext = __ldg(send_row + (first + (i + 1) * step) * k + lane);
        bool ready = true;
        if (lane == 0) ready = mbar_wait_bounded(bars + 8 * s, parity, kWaitLimitNs);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) {
            flags |= COACT_EFLAG_TIMEOUT;
            break;
        }
        // every lane observes the completed phase before reading the stage
        mbar_try_wait(bars + 8 * s, parity);
        fence_proxy_async_smem();
        if (lane < k && d >= 0) {
            if ((int64_t)d < cap) {
                bulk_store(sb + (int64_t)d * row_bytes, bufs + (uint32_t)s * row_bytes, row_bytes);
            } else {
                flags |= COACT_EFLAG_ROW_RANGE;
            }
        }
        bulk_commit();
        // token i-1's stores have finished reading its stage once at most the newest
        // group (token i's) is outstanding; refill that stage with token i-1+S
        bulk_wait_read<1>();
        __syncwarp();
        if (lane == 0 && i >= 1 && loaded < n_mine) {
            const int sp = (int)((i - 1) % S);
            const uint32_t bar = bars + 8 * sp;
            mbar_expect_tx(bar, row_bytes);
            bulk_load(bufs + (uint32_t)sp * row_bytes,
                      xb + (first + loaded * step) * (int64_t)row_bytes, row_bytes, bar);
            ++loaded;
        }
        __syncwarp();
    }
    if (i < n_mine && lane == 0) {
        // gave up: wait (bounded) for the loads still in flight before the CTA exits
        for (int64_t q = i; q < loaded; ++q)
            mbar_wait_bounded(bars + 8 * (uint32_t)(q % S), (uint32_t)((q / S) & 1), kWaitLimitNs);
    }
    bulk_wait_all();
    raise_flag_warp(err, flags);
}

template <int S>
int launch_bulk(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row, int k,
                uint16_t *send, int64_t cap, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
    const uint32_t row_bytes = (uint32_t)(H * 2);
    const size_t smem = kBulkHeader + (size_t)S * row_bytes;
    auto kern = k_gather_bulk<S>;
    static SmemOptIn opt;
    if (int s = ensure_smem(kern, smem, opt, di)) return s;
    const int per_sm = blocks_per_sm(32, smem, di);
    // at least S tokens per CTA so the ring fills, but every SM busy
    const int64_t want = std::max<int64_t>(1, ceil_div(N, 2 * S));
    const int blocks = (int)std::min<int64_t>(want, (int64_t)per_sm * di.sm_count);
    return launch_pdl(kern, blocks, 32, smem, st, x, N, row_bytes, send_row, k, send, cap, err);
}

int launch_v16(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row, int k,
               uint16_t *send, int64_t cap, int32_t *err, cudaStream_t st, const DeviceInfo &di) {
#ifndef COACT_GATHER_PER_SM
#define COACT_GATHER_PER_SM 128  // CTAs per SM in the grid at most (0: one resident wave)
#endif
#ifndef COACT_GATHER_UNROLL
#define COACT_GATHER_UNROLL 4  // chunk loads in flight per lane on long rows
#endif
#ifndef COACT_GATHER_VEC
#define COACT_GATHER_VEC 32  // widest chunk: 32 (256-bit accesses where aligned) or 16
#endif
#ifndef COACT_GATHER_KT
#define COACT_GATHER_KT 1  // 1: kernels specialised per k (unrolled destinations); 0: one kernel
#endif
#ifndef COACT_GATHER_PREFETCH_BYTES
// x bytes warmed into L2 before the wait (0: none).  With the earlier 16-byte gather, 16-32
// MB took ~1% off config 1's step behind its plan; with the current kernel it gains nothing
// (config 1: 72.1 vs 72.2 us, config 3: 4,069 vs 4,070 us per step) and on config 3 costs
// ~7% extra DRAM reads (prefetched lines evicted by the write stream before use) -> off.
#define COACT_GATHER_PREFETCH_BYTES 0ll
#endif
    // the bulk prefetch takes a 32-bit size: rows beyond 16 MB are not prefetched
    const int64_t n_pf =
        H * 2 > (1 << 24) ? 0 : std::min<int64_t>(N, (int64_t)(COACT_GATHER_PREFETCH_BYTES) / (H * 2));
    const bool wide = COACT_GATHER_VEC == 32 && H % 16 == 0 && aligned32(x) && aligned32(send);
    auto go = [&](auto kern, auto *xv, auto *sv, int64_t Hv) {
        return launch_pdl(kern, grid_for(kern, N, COACT_GATHER_PER_SM, di), 256, 0, st, xv, N, Hv,
                          send_row, k, sv, cap, n_pf, err);
    };
    auto with_k = [&](auto k_tag) {
        constexpr int KK = decltype(k_tag)::value;
        if (wide) {
            const Row32 *xv = reinterpret_cast<const Row32 *>(x);
            Row32 *sv = reinterpret_cast<Row32 *>(send);
            const int64_t Hv = H / 16;
            if (Hv <= 32) return go(k_gather_v16<KK, Row32, 1>, xv, sv, Hv);
            return go(k_gather_v16<KK, Row32, (COACT_GATHER_UNROLL + 1) / 2>, xv, sv, Hv);
        }
        const uint4 *xv = reinterpret_cast<const uint4 *>(x);
        uint4 *sv = reinterpret_cast<uint4 *>(send);
        const int64_t Hv = H / 8;
        if (Hv <= 32) return go(k_gather_v16<KK, uint4, 1>, xv, sv, Hv);
        return go(k_gather_v16<KK, uint4, COACT_GATHER_UNROLL>, xv, sv, Hv);
    };
#if COACT_GATHER_KT
    switch (k) {
        case 1: return with_k(std::integral_constant<int, 1>{});
        case 2: return with_k(std::integral_constant<int, 2>{});
        case 3: return with_k(std::integral_constant<int, 3>{});
        case 4: return with_k(std::integral_constant<int, 4>{});
        case 5: return with_k(std::integral_constant<int, 5>{});
        case 6: return with_k(std::integral_constant<int, 6>{});
        case 7: return with_k(std::integral_constant<int, 7>{});
        case 8: return with_k(std::integral_constant<int, 8>{});
    }
    return COACT_ERR_UNSUPPORTED;
#else
    return with_k(std::integral_constant<int, 0>{});
#endif
}

}  // namespace
}  // namespace coact

using namespace coact;

namespace coact {
namespace {

int gather_args(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row, int k,
                uint16_t *send, int64_t row_capacity) {
    if (N < 0 || H < 0 || row_capacity < 0) return COACT_ERR_INVALID;
    if (k < 1 || k > COACT_MAX_K) return COACT_ERR_UNSUPPORTED;
    if (H % 8 != 0) return COACT_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return -100;  // nothing to do
    if (!x || !send_row || (row_capacity > 0 && !send)) return COACT_ERR_INVALID;
    if (!aligned16(x) || (send && !aligned16(send))) return COACT_ERR_INVALID;
    if (N > (int64_t)INT32_MAX / k || row_capacity > (int64_t)INT32_MAX) return COACT_ERR_UNSUPPORTED;
    return COACT_OK;
}

}  // namespace
}  // namespace coact

extern "C" int dispatch_gather(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row,
                               int k, uint16_t *send, int64_t row_capacity, int32_t *err_flag,
                               coact_stream_t stream) {
    COACT_RANGE("dispatch_gather");
    const int a = gather_args(x, N, H, send_row, k, send, row_capacity);
    if (a == -100) return COACT_OK;
    if (a) return a;
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#if defined(COACT_GATHER_PATH)
    if (COACT_GATHER_PATH != 0 && H * 2 >= 1024 && H * 2 <= 32768) {  // experiment builds only
        if (H * 2 <= 4096)
            return launch_bulk<8>(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
        return launch_bulk<4>(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
    }
#endif
    return launch_v16(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
}

extern "C" int dispatch_gather_tma(const uint16_t *x, int64_t N, int64_t H, const int32_t *send_row,
                                   int k, uint16_t *send, int64_t row_capacity, int32_t *err_flag,
                                   coact_stream_t stream) {
    COACT_RANGE("dispatch_gather_tma");
    const int a = gather_args(x, N, H, send_row, k, send, row_capacity);
    if (a == -100) return COACT_OK;
    if (a) return a;
    if (H * 2 > 32768) return COACT_ERR_UNSUPPORTED;   // one row per shared-memory stage
    DeviceInfo di;
    if (int s = device_info(&di)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (H * 2 <= 4096)
        return launch_bulk<8>(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
    if (H * 2 <= 16384)
        return launch_bulk<4>(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
    return launch_bulk<2>(x, N, H, send_row, k, send, row_capacity, err_flag, st, di);
}
