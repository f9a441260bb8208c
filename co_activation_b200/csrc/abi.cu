// Status strings, ABI version and the per-device attribute cache.
#include <cuda.h>  // the driver's types for cuCtxGetId, resolved at run time (no -lcuda)

#include "common.cuh"

namespace coact {

namespace {
thread_local int g_last_cuda = 0;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_optin[kMaxDevices];
std::atomic<int> g_smem_sm[kMaxDevices];
}  // namespace

int cuda_fail(cudaError_t e) {
    g_last_cuda = (int)e;
    (void)cudaGetLastError();
    return COACT_ERR_CUDA;
}

namespace {
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// cuCtxGetId through the runtime's driver entry-point lookup, once per process; NULL if
// this driver does not provide it (the context id then reads 0 everywhere).
CtxGetIdFn ctx_get_id_fn() {
    static const CtxGetIdFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<CtxGetIdFn>(p);
    }();
    return fn;
}
}  // namespace

int device_info(DeviceInfo *out) {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return COACT_ERR_UNSUPPORTED;
    int sms = g_sm_count[dev].load(std::memory_order_relaxed);
    int smem = g_smem_optin[dev].load(std::memory_order_relaxed);
    int smem_sm = g_smem_sm[dev].load(std::memory_order_relaxed);
    if (sms <= 0 || smem <= 0 || smem_sm <= 0) {
        cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (!e) e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (!e) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        if (e) return cuda_fail(e);
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
        g_smem_optin[dev].store(smem, std::memory_order_relaxed);
        g_smem_sm[dev].store(smem_sm, std::memory_order_relaxed);
    }
    unsigned long long ctx = 0;
    if (CtxGetIdFn f = ctx_get_id_fn()) {
        if (f(nullptr, &ctx) != CUDA_SUCCESS) {
            // no current context (e.g. right after a device reset): make the device's
            // primary context current, as any runtime call would, and ask again
            if (cudaError_t e = cudaSetDevice(dev)) return cuda_fail(e);
            if (f(nullptr, &ctx) != CUDA_SUCCESS) ctx = 0;
        }
    }
    out->device = dev;
    out->ctx = ctx;
    out->sm_count = sms;
    out->smem_optin = smem;
    out->smem_per_sm = smem_sm;
    return COACT_OK;
}

}  // namespace coact

extern "C" const char *coact_strerror(int status) {
    switch (status) {
        case COACT_OK: return "ok";
        case COACT_ERR_INVALID: return "invalid argument (NULL pointer, negative size or misaligned buffer)";
        case COACT_ERR_UNSUPPORTED: return "argument outside the supported limits";
        case COACT_ERR_CUDA: return "CUDA launch or attribute query failed";
        case COACT_ERR_WORKSPACE: return "workspace missing or too small";
        case COACT_ERR_TIMEOUT: return "a bounded device wait gave up";
        default: return "unknown status";
    }
}

extern "C" int coact_abi_version(void) { return COACT_ABI_VERSION; }

extern "C" int coact_last_cuda_error(void) { return coact::g_last_cuda; }
