// api.cu -- status strings, version, the sticky device error word, the
// per-context cache of device-symbol addresses, and the diagnostic of the
// bounded device waits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"

// First error code recorded by any kernel of the library on this device
// (0 = none).  Kernels never trap; they record here and skip the access.
__device__ int dsa_device_error_word_storage = 0;

namespace dsa {
namespace {

PFN_cuCtxGetCurrent_v4000 ctx_get_current_fn() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    return fn;
}

void *current_context() {
    auto fn = ctx_get_current_fn();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

SymbolCache g_error_word_cache;

}  // namespace

void *symbol_address(const void *symbol, SymbolCache *cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= SymbolCache::kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(cache->mutex);
    void *ctx = current_context();
    if (cache->ptr[dev] && ctx && ctx == cache->ctx[dev]) return cache->ptr[dev];
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return nullptr;
    cache->ptr[dev] = p;
    cache->ctx[dev] = current_context();     // the runtime's context now exists
    return p;
}

int *device_error_word() {
    return static_cast<int *>(symbol_address(&dsa_device_error_word_storage, &g_error_word_cache));
}

}  // namespace dsa

extern "C" const char *dsa_status_string(dsa_status status) {
    switch (status) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case DSA_ERR_CUDA: return "CUDA runtime or launch error";
        case DSA_ERR_TIMEOUT: return "bounded device wait expired";
        case DSA_ERR_DEVICE: return "device-side check failed";
        case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

extern "C" int dsa_version(void) { return 100; }

extern "C" dsa_status dsa_get_device_error(dsa_stream_t stream, int32_t *device_status) {
    if (!device_status) return DSA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int *word = dsa::device_error_word();
    if (!word) return DSA_ERR_CUDA;
    int host = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemcpy(&host, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (host != 0 && cudaMemset(word, 0, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
    *device_status = host;
    return DSA_OK;
}

namespace {

// One CTA waits on a shared-memory barrier through the wait routine every
// kernel of the library uses, with the given budget; nobody arrives unless
// `complete`, so the wait either succeeds at once or expires and records
// DSA_ERR_TIMEOUT.
__global__ void __launch_bounds__(32) wait_selftest_kernel(long long budget, int complete, int *err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        dsa::tc::mbar_init(&bar, 1);
        abort_flag = 0;
        dsa::tc::fence_mbar_init();
    }
    __syncthreads();
    if (complete && threadIdx.x == 0) dsa::tc::mbar_arrive(&bar);
    dsa::tc::mbar_wait(&bar, 0, err, &abort_flag, budget);
    __syncthreads();
}

}  // namespace

extern "C" dsa_status dsa_wait_selftest(int64_t budget_cycles, int complete, dsa_stream_t stream) {
    if (budget_cycles < 1 || budget_cycles > dsa::tc::kWaitBudget) return DSA_ERR_INVALID_ARG;
    int *err = dsa::device_error_word();
    if (!err) return DSA_ERR_CUDA;
    wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (long long)budget_cycles, complete, err);
    return dsa::launch_status();
}
