// indexer_quant.cu -- rotate_activation + act_quant of indexer queries and keys.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward: queries
// and keys are rotated (rotate_activation) and quantised blockwise to FP8
// (act_quant), and the key's codes and scale are written into the caches at
// positions start_pos .. end_pos-1.
//
// One warp rotates and quantises one d-vector entirely in registers (see
// quant.cuh for the butterfly order and the rounding).
// The pass is HBM-bound: 4*d (fp32) or 2*d (bf16) bytes in, d + 4 bytes out
// per vector.
#include "common.cuh"
#include "quant.cuh"

namespace dsa {
namespace {

template <int D, typename Tin>
__global__ void __launch_bounds__(256)
indexer_quant_kernel(const Tin *__restrict__ x, int64_t n_rows, int64_t n_vec,
                     uint8_t *__restrict__ out, int64_t out_row_stride,
                     float *__restrict__ out_scale, int64_t scale_row_stride) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t total = n_rows * n_vec;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); v < total;
         v += warps) {
        float r[E];
        load_lane_slice<D, Tin>(x + v * D, r);
        float s;
        const uint32_t packed = rotate_quant_warp<D>(r, &s);
        const int64_t row = v / n_vec, vi = v - row * n_vec;
        uint8_t *dst = out + row * out_row_stride + vi * D + lane * E;
        if constexpr (E == 4) *reinterpret_cast<uint32_t *>(dst) = packed;
        else *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(packed);
        if (lane == 0) out_scale[row * scale_row_stride + vi] = s;
    }
}

template <int D, typename Tin>
dsa_status launch_d(const void *x, int64_t n_rows, int64_t n_vec, uint8_t *out,
                    int64_t out_row_stride, float *out_scale, int64_t scale_row_stride,
                    cudaStream_t stream) {
    const int64_t total = n_rows * n_vec;
    const int warps_per_block = 8;
    int64_t blocks = (total + warps_per_block - 1) / warps_per_block;
    const int64_t cap = (int64_t)num_sms() * 64;
    if (blocks > cap) blocks = cap;
    indexer_quant_kernel<D, Tin><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(
        static_cast<const Tin *>(x), n_rows, n_vec, out, out_row_stride, out_scale,
        scale_row_stride);
    return launch_status();
}

}  // namespace

dsa_status launch_indexer_quant(const void *x, dsa_dtype x_dtype, int64_t n_rows, int64_t n_vec,
                                int d, uint8_t *out_fp8, int64_t out_row_stride, float *out_scale,
                                int64_t scale_row_stride, cudaStream_t stream) {
    if (n_rows * n_vec == 0) return DSA_OK;
    const bool bf = x_dtype == DSA_BF16;
    if (d == 128)
        return bf ? launch_d<128, __nv_bfloat16>(x, n_rows, n_vec, out_fp8, out_row_stride,
                                                 out_scale, scale_row_stride, stream)
                  : launch_d<128, float>(x, n_rows, n_vec, out_fp8, out_row_stride, out_scale,
                                         scale_row_stride, stream);
    return bf ? launch_d<64, __nv_bfloat16>(x, n_rows, n_vec, out_fp8, out_row_stride, out_scale,
                                            scale_row_stride, stream)
              : launch_d<64, float>(x, n_rows, n_vec, out_fp8, out_row_stride, out_scale,
                                    scale_row_stride, stream);
}

}  // namespace dsa

extern "C" dsa_status dsa_indexer_quant(const void *x, dsa_dtype x_dtype, int64_t n_rows,
                                        int64_t n_vec, int d, uint8_t *out_fp8,
                                        int64_t out_row_stride, float *out_scale,
                                        int64_t scale_row_stride, dsa_stream_t stream) {
    if (n_rows < 0 || n_vec < 0) return DSA_ERR_INVALID_ARG;
    if (x_dtype != DSA_F32 && x_dtype != DSA_BF16) return DSA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return DSA_ERR_UNSUPPORTED;
    if (n_rows == 0 || n_vec == 0) return DSA_OK;
    if (!x || !out_fp8 || !out_scale) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(x) || !dsa::aligned16(out_fp8) || (reinterpret_cast<uintptr_t>(out_scale) & 3))
        return DSA_ERR_INVALID_ARG;
    if (n_rows > 1) {
        if (out_row_stride < n_vec * d || (out_row_stride & 15) || scale_row_stride < n_vec)
            return DSA_ERR_INVALID_ARG;
    }
    return dsa::launch_indexer_quant(x, x_dtype, n_rows, n_vec, d, out_fp8, out_row_stride,
                                     out_scale, scale_row_stride,
                                     reinterpret_cast<cudaStream_t>(stream));
}
