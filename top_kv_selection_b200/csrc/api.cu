// api.cu -- status strings, version and the sticky device error word.
#include "common.cuh"

// First error code recorded by any kernel of the library on this device
// (0 = none).  Kernels never trap; they record here and skip the access.
__device__ int dsa_device_error_word_storage = 0;

namespace dsa {

int *device_error_word() {
    static int *cached[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cached[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, dsa_device_error_word_storage) != cudaSuccess) return nullptr;
        cached[dev] = static_cast<int *>(p);
    }
    return cached[dev];
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
