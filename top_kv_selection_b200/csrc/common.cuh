// common.cuh -- internal helpers shared by the libdsa CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <mutex>

#include "dsa.h"

namespace dsa {

// ---------------------------------------------------------------- host side
// Device address of a __device__ variable (its host-side name is only a
// stand-in) on the current device, cached per device together with the CUDA
// context it was resolved in: a new context (after cudaDeviceReset, say)
// resolves it again.  Thread-safe.  Returns nullptr if the runtime cannot
// resolve it.
struct SymbolCache {
    static constexpr int kMaxDevices = 64;
    std::mutex mutex;
    void *ctx[kMaxDevices] = {nullptr};
    void *ptr[kMaxDevices] = {nullptr};
};
void *symbol_address(const void *symbol, SymbolCache *cache);

// Device pointer of the sticky error word of the current device (the word
// lives in api.cu).  Returns nullptr if the runtime cannot resolve it.
int *device_error_word();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline dsa_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

inline int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// -------------------------------------------------------------- device side
__device__ __forceinline__ void record_error(int *word, int code) {
    if (word) atomicCAS(word, 0, code);
}

// Loads of a preceding kernel's output (or of anything written in the same
// stream order) after griddepcontrol.wait: L2-coherent (.cg), and volatile so
// that the compiler keeps them after the wait (a non-coherent __ldg may be
// moved above it).
__device__ __forceinline__ uint32_t ld_cg_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ float ld_cg_f32(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Order-preserving map from an fp32 score to an unsigned key: a > b as floats
// <=> key(a) > key(b).  -0 maps to the key of +0; NaN maps to 0, below -inf.
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;   // NaN
    if ((u & 0x7fffffffu) == 0u) u = 0u;              // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// e4m3 code -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __nv_fp8_e4m3 v;
    v.__x = c;
    return static_cast<float>(v);
}

// Four packed e4m3 codes (little-endian in a 32-bit word) -> fp32.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float &a, float &b, float &c, float &d) {
    __nv_fp8x2_e4m3 lo, hi;
    lo.__x = static_cast<__nv_fp8x2_storage_t>(w & 0xffffu);
    hi.__x = static_cast<__nv_fp8x2_storage_t>(w >> 16);
    float2 l = static_cast<float2>(lo);
    float2 h = static_cast<float2>(hi);
    a = l.x; b = l.y; c = h.x; d = h.y;
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// ------------------------------------------------ internal launchers (no checks)
dsa_status launch_indexer_quant(const void *x, dsa_dtype x_dtype, int64_t n_rows, int64_t n_vec,
                                int d, uint8_t *out_fp8, int64_t out_row_stride, float *out_scale,
                                int64_t scale_row_stride, cudaStream_t stream);

dsa_status launch_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                               const uint8_t *k_cache, const float *k_scale, int64_t t_max, int B,
                               int S, int H, int D, int64_t start_pos, int64_t T,
                               float softmax_scale, float *scores, cudaStream_t stream,
                               int compress = 1);

// Decode step: rotate + quantise the new queries and key inside the scorer,
// append the key at T-1, score positions 0..T-1 of each sequence.  With
// row_hist ([B][decode_hist_chunks()][kHistBins]), each of the scorer's CTAs
// also counts its scores by the top 12 bits of their key and writes that
// histogram, every bin, into its own slot, for the decode top-k (topk.cu),
// which sums a row's slots; nothing needs zeroing first.
constexpr int kHistBins = 4096;
int decode_hist_chunks(int B, int H, int D, int64_t T);
dsa_status launch_decode_scores(const float *q_raw, const float *w, const float *k_new,
                                uint8_t *k_cache, float *k_scale, int64_t t_max, int B, int H,
                                int D, int64_t T, float softmax_scale, float *scores,
                                cudaStream_t stream, uint32_t *row_hist = nullptr);

size_t topk_workspace_bytes(int B, int S, int64_t T, int k);
// prefetch_rows: optional cache whose rows at the selected positions are
// requested into L2 as they are selected (row (b, t) at prefetch_rows +
// (b * prefetch_t_max + t) * prefetch_row_bytes; bytes a multiple of 16).
// compress: the scores are over compressed entries of this many tokens; row s
// keeps the best of its (start_pos + s + 1) / compress available entries.
// row_hist / hist_chunks: the decode step's top-k (S = 1, start_pos = T - 1,
// T up to 262144) takes the decode scorer's per-CTA histograms of the scores'
// top 12 key bits ([B][hist_chunks][kHistBins]) and runs one cluster per row
// that reads the scores once; without them the general cluster kernel runs.
dsa_status launch_topk_select(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                              int k, int32_t *idx, void *ws, cudaStream_t stream,
                              const void *prefetch_rows = nullptr, int64_t prefetch_t_max = 0,
                              int prefetch_row_bytes = 0, const uint32_t *row_hist = nullptr,
                              int hist_chunks = 0, int compress = 1);

size_t sparse_mla_workspace_bytes(int B, int S, int Hq, int dc, int dr, int k, dsa_dtype dt);
bool sparse_mla_tc_supported(int Hq, int dc, int dr, int k, dsa_dtype dt);
size_t sparse_mla_tc_workspace_bytes(int B, int S, int k);
dsa_status launch_sparse_mla_tc(const void *q, const void *kv, int64_t t_max, const int32_t *idx,
                                int B, int S, int k, int64_t start_pos, float sm_scale, void *out,
                                float *lse, void *ws, cudaStream_t stream);
bool sparse_mla_fp8_tc_supported(int Hq, int dc, int dr, int k);
dsa_status launch_sparse_mla_fp8_tc(const void *q, const uint8_t *kv8, int64_t t_max,
                                    const int32_t *idx, int B, int S, int k, int64_t start_pos,
                                    float sm_scale, void *out, float *lse, void *ws,
                                    cudaStream_t stream);
// FP8 latent cache (latent_fp8.cu): 656-byte rows at the V3.2 shapes
bool latent_fp8_shape_ok(int dc, int dr);
size_t sparse_mla_fp8_workspace_bytes(int B, int S, int Hq, int dc, int dr, int k);
dsa_status launch_sparse_mla_fp8(const void *q, const uint8_t *kv_fp8, int64_t t_max,
                                 const int32_t *idx, int B, int S, int Hq, int dc, int dr, int k,
                                 int64_t start_pos, float sm_scale, void *out, float *lse,
                                 void *workspace, cudaStream_t stream);
dsa_status launch_sparse_mla(const void *q, const void *kv, int64_t t_max, const int32_t *idx,
                             int B, int S, int Hq, int dc, int dr, int k, int64_t start_pos,
                             float sm_scale, dsa_dtype dt, void *out, float *lse, void *ws,
                             cudaStream_t stream);

}  // namespace dsa
