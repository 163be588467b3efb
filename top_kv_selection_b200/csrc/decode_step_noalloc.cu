// decode_step_noalloc.cu -- the decode step for callers that cannot allocate.
//
// dsa_decode_step needs a caller-provided workspace.  Some callers cannot get
// one: a plugin that runs inside another engine's memory pool and may not call
// cudaMalloc, code that is launched while someone else's CUDA graph is being
// captured (an allocation there would break the capture), or a small C host
// that links only this library.  dsa_decode_step_noalloc takes the same inputs
// and outputs and runs the same kernels, with the scratch memory taken from a
// fixed array that belongs to this file: DSA_NOALLOC_SCRATCH_BYTES of device
// memory that every GPU which loads this code keeps until the process exits.
//
// The array's host-side name is only a stand-in for the symbol, not a device
// address, so the host code below resolves the real address once per device
// (with that device current) and hands it to the kernels as a pointer.
#include "common.cuh"

static __device__ __align__(256) unsigned char dsa_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

namespace {

dsa::SymbolCache g_scratch_cache;

// Device address of the scratch array on the current device, resolved on the
// first call for that device (and again if the device's context was replaced).
dsa_status scratch_address(void **out) {
    void *p = dsa::symbol_address(dsa_noalloc_scratch, &g_scratch_cache);
    if (!p) return DSA_ERR_CUDA;
    *out = p;
    return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_decode_step_noalloc(const float *q_idx, const float *w,
                                              const float *k_new, uint8_t *k_cache,
                                              float *k_scale, int64_t t_max, const void *kv_cache,
                                              const void *q_mla, int B, int H, int D, int Hq,
                                              int dc, int dr, int64_t T, int index_topk,
                                              float softmax_scale, float sm_scale, dsa_dtype dt,
                                              int32_t *idx, void *out, float *lse,
                                              dsa_stream_t stream) {
    const size_t need =
        dsa_decode_step_workspace_size(B, H, D, T, index_topk, Hq, dc, dr, dt);
    if (need > (size_t)DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const dsa_status st = scratch_address(&scratch);
    if (st != DSA_OK) return st;
    return dsa_decode_step(q_idx, w, k_new, k_cache, k_scale, t_max, kv_cache, q_mla, B, H, D,
                           Hq, dc, dr, T, index_topk, softmax_scale, sm_scale, dt, idx, out, lse,
                           scratch, (size_t)DSA_NOALLOC_SCRATCH_BYTES, stream);
}
