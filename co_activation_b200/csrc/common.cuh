// Internal helpers shared by the library's kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#if defined(COACT_NVTX)
#include <nvtx3/nvToolsExt.h>
#endif
#include <utility>

#include "coact.h"

namespace coact {

constexpr int kWarp = 32;

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ void raise_flag(int32_t *err, int bits) {
    if (bits && err) atomicOr(err, bits);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// bf16 bit pattern -> fp32 (exact: bf16 is the top half of an fp32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Streaming 16-byte global accesses: data touched once, do not keep it in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4 *p, const uint4 &v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Row chunks of 16 bytes (uint4) or 32 bytes (Row32: one 256-bit access per lane, half the
// memory instructions of 16-byte chunks; only for rows and buffers that are 32-byte
// aligned, which the host checks before choosing it).
struct alignas(32) Row32 {
    uint32_t w[8];
};

template <typename V>
__device__ __forceinline__ V ld_chunk(const V *p);
template <>
__device__ __forceinline__ uint4 ld_chunk<uint4>(const uint4 *p) {
    return ld_stream(p);
}
template <>
__device__ __forceinline__ Row32 ld_chunk<Row32>(const Row32 *p) {
    Row32 v;
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                   "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_chunk(uint4 *p, const uint4 &v) { st_stream(p, v); }
__device__ __forceinline__ void st_chunk(Row32 *p, const Row32 &v) {
    asm volatile("st.global.cs.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
                 "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
                 "r"(v.w[7])
                 : "memory");
}

// 32-bit word q of a chunk (q a compile-time constant after unrolling)
__device__ __forceinline__ uint32_t chunk_word(const uint4 &v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t chunk_word(const Row32 &v, int q) { return v.w[q]; }
__device__ __forceinline__ void set_chunk_word(uint4 &v, int q, uint32_t x) {
    if (q == 0) v.x = x;
    else if (q == 1) v.y = x;
    else if (q == 2) v.z = x;
    else v.w = x;
}
__device__ __forceinline__ void set_chunk_word(Row32 &v, int q, uint32_t x) { v.w[q] = x; }

// Asks the copy engine of the SM (TMA) to bring [p, p + bytes) of this GPU's memory into
// L2; p 16-byte aligned, bytes a multiple of 16.  A hint with no completion: nothing is
// returned, no mbarrier is involved and nothing needs waiting for.  L2 is where every
// access to this GPU's memory meets, so a line fetched before its last writer finished
// is updated there by that write, never served stale.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Loads token t's K expert ids (row t of an int32 [N, K] array) and returns the
// validation bits: COACT_EFLAG_ID_RANGE for an id outside [0, E), COACT_EFLAG_DUP_ID
// for an id that repeats within the token.  0 means the token is valid.
template <int K>
__device__ __forceinline__ int load_ids(const int32_t *__restrict__ ids, int64_t t, int E,
                                        int (&e)[K]) {
    int f = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        e[j] = __ldg(ids + t * K + j);
        if ((unsigned)e[j] >= (unsigned)E) f |= COACT_EFLAG_ID_RANGE;
    }
#pragma unroll
    for (int j = 1; j < K; ++j)
#pragma unroll
        for (int jj = 0; jj < j; ++jj)
            if (e[j] == e[jj]) f |= COACT_EFLAG_DUP_ID;
    return f;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// OR of `bits` over the warp, raised once by lane 0 (all lanes must call).
__device__ __forceinline__ void raise_flag_warp(int32_t *err, int bits) {
    const unsigned all = __reduce_or_sync(0xffffffffu, (unsigned)bits);
    if (all && (threadIdx.x & 31) == 0 && err) atomicOr(err, (int)all);
}

// Programmatic dependent launch.  Every library kernel is launched with programmatic
// stream serialisation: it may start while the previous kernel on the stream drains,
// and it reads no global input written by that kernel until pdl_wait() returns (the
// previous grid has completed and its writes are visible).  A kernel that is not the
// last of its call calls pdl_trigger() only AFTER its own pdl_wait(), so when the next
// kernel of the same call starts, every kernel before it has completed: such a kernel
// may read the call's inputs before waiting.  The first kernel of a call reads no
// global memory before pdl_wait() (it may warm L2 with prefetch_l2_bulk, which reads
// nothing into the program).  The last kernel of plan_dispatch triggers nothing: its
// successor launches when it completes (see k_plan_scatter).
__device__ __forceinline__ void pdl_wait() {
#if !defined(COACT_NO_PDL)
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

__device__ __forceinline__ void pdl_trigger() {
#if !defined(COACT_NO_PDL)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

// ------------------------------------------------------------------ host helpers

// Per-device attributes, queried once per device.
struct DeviceInfo {
    int device;
    int sm_count;
    int smem_optin;   // max dynamic shared memory per block (opt-in)
    int smem_per_sm;  // shared memory per SM
    // Id of the current CUDA context (unique for the life of the process; 0 if the driver
    // cannot tell).  Per-context state -- a kernel's shared-memory opt-in, the device
    // address of a __device__ array -- is cached under it, so a device reset (which ends
    // the context and unloads the module) makes the next call set it up again.
    unsigned long long ctx;
};
int device_info(DeviceInfo *out);  // returns COACT_OK or COACT_ERR_CUDA

constexpr int kMaxDevices = 64;

// Largest dynamic shared-memory size already opted in, per device, for one kernel.
// The CUDA error behind the last COACT_ERR_CUDA of this host thread (coact_last_cuda_error).
// A failed call is recorded here and consumed (cudaGetLastError), so it is not reported
// again by an unrelated later check.
int cuda_fail(cudaError_t e);

struct SmemOptIn {
    std::atomic<int> bytes[kMaxDevices];
    std::atomic<unsigned long long> ctx[kMaxDevices];
};

// Opts `kernel` in to `bytes` of dynamic shared memory on the current device once per
// context; later calls only read the cache, so a stream capture sees launches alone.
// (Two threads racing here at most repeat the idempotent attribute call.)
template <typename F>
int ensure_smem(F kernel, size_t bytes, SmemOptIn &cache, const DeviceInfo &di) {
    if (bytes <= 48 * 1024) return COACT_OK;
    if (bytes > (size_t)di.smem_optin) return COACT_ERR_UNSUPPORTED;
    std::atomic<int> &slot = cache.bytes[di.device];
    std::atomic<unsigned long long> &ctx = cache.ctx[di.device];
    if (ctx.load(std::memory_order_acquire) == di.ctx &&
        slot.load(std::memory_order_relaxed) >= (int)bytes)
        return COACT_OK;
    if (cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)bytes))
        return cuda_fail(e);
    if (ctx.load(std::memory_order_relaxed) != di.ctx) slot.store(0, std::memory_order_relaxed);
    slot.store(std::max(slot.load(std::memory_order_relaxed), (int)bytes),
               std::memory_order_relaxed);
    ctx.store(di.ctx, std::memory_order_release);
    return COACT_OK;
}

// Resident blocks per SM for a kernel limited by threads and shared memory (for the
// kernels sized with it, which use few enough registers that registers never bind).
inline int blocks_per_sm(int threads, size_t smem, const DeviceInfo &di) {
    int by_threads = 2048 / threads;
    int by_smem = smem ? (int)(di.smem_per_sm / (smem + 1024)) : 32;
    int b = by_threads < by_smem ? by_threads : by_smem;
    b = b < 32 ? b : 32;
    return b > 0 ? b : 1;
}

inline int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? COACT_OK : cuda_fail(e);
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Grid for a grid-stride kernel of 256-thread CTAs over `units` work items, 8 per CTA
// (one per warp): at most `per_sm` CTAs per SM, where per_sm <= 0 means the CTAs of
// `kernel` that fit on an SM at once (one wave, every CTA resident from the start).
template <typename... KArgs>
int grid_for(void (*kernel)(KArgs...), int64_t units, int per_sm, const DeviceInfo &di) {
    if (per_sm <= 0) {
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, 256, 0) != cudaSuccess ||
            occ < 1) {
            (void)cudaGetLastError();
            occ = 1;
        }
        per_sm = occ;
    }
    const int64_t b = std::min<int64_t>(ceil_div(units, 8), (int64_t)di.sm_count * per_sm);
    return (int)(b > 1 ? b : 1);
}

// Launches `kernel` on `stream` with programmatic stream serialisation (see pdl_wait).
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
               Args &&...args) {
#if defined(COACT_CARVEOUT)   // experiment builds: preferred shared-memory carveout, percent
    if (cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             COACT_CARVEOUT))
        return cuda_fail(e);
#endif
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
#if defined(COACT_NO_PDL)
    cfg.numAttrs = 0;
#else
    cfg.attrs = attr;
    cfg.numAttrs = 1;
#endif
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    return e == cudaSuccess ? COACT_OK : cuda_fail(e);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// NVTX range around each C-ABI call, for timeline profilers (builds with -DCOACT_NVTX; the
// NVTX v3 headers are header-only and cost nothing when no tool is attached).
#if defined(COACT_NVTX)
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
#define COACT_RANGE(name) ::coact::NvtxRange coact_nvtx_range_(name)
#else
#define COACT_RANGE(name) ((void)0)
#endif


}  // namespace coact
