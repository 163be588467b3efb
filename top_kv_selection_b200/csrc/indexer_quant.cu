// indexer_quant.cu -- rotate_activation + act_quant of indexer queries and keys.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward
// (q = rotate_activation(q); k = rotate_activation(k); act_quant(., block_size);
//  k_cache[:, start_pos:end_pos] = k_fp8; k_scale_cache[...] = k_scale).
//
// One warp rotates and quantises one d-vector entirely in registers:
//   lane L holds elements [E*L, E*L + E), E = d / 32.
//   Butterfly stage h pairs element i with i ^ h: for h < E both live in the
//   lane's registers, otherwise in lane L ^ (h / E) at the same register slot.
//   The lower element becomes a + b and the upper a - b, in fp32, stages in
//   the order h = 1, 2, 4, ..., d/2, so the result is bit-identical to the
//   straightforward in-place transform.  Then one multiply by fp32(d^-1/2),
//   a warp max of |x|, scale = max(amax, 1e-4) / 448 and the e4m3 codes of
//   x / scale (round to nearest even, saturate to +-448).
// The pass is HBM-bound: 4*d (fp32) or 2*d (bf16) bytes in, d + 4 bytes out
// per vector.
#include "common.cuh"

namespace dsa {
namespace {

// Two fp32 -> two e4m3 codes packed as (lo | hi << 8); the first PTX source
// operand fills the upper byte.
__device__ __forceinline__ uint32_t e4m3x2_rn_sat(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D> struct HadamardScale;
template <> struct HadamardScale<64> { static constexpr float value = 0.125f; };
// nearest fp32 to 128^-1/2 = sqrt(2)/16: 0x3DB504F3
template <> struct HadamardScale<128> { static constexpr float value = 0x1.6a09e6p-4f; };

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
        const Tin *src = x + v * D + lane * E;
        if constexpr (E == 4 && sizeof(Tin) == 4) {
            float4 t = *reinterpret_cast<const float4 *>(src);
            r[0] = t.x; r[1] = t.y; r[2] = t.z; r[3] = t.w;
        } else if constexpr (E == 2 && sizeof(Tin) == 4) {
            float2 t = *reinterpret_cast<const float2 *>(src);
            r[0] = t.x; r[1] = t.y;
        } else {
#pragma unroll
            for (int e = 0; e < E; e++) r[e] = to_f32<Tin>(src[e]);
        }
        // butterflies inside the lane
#pragma unroll
        for (int h = 1; h < E; h <<= 1) {
#pragma unroll
            for (int e = 0; e < E; e++) {
                if (e & h) continue;
                float a = r[e], b = r[e + h];
                r[e] = a + b;
                r[e + h] = a - b;
            }
        }
        // butterflies across lanes
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int e = 0; e < E; e++) {
                float p = __shfl_xor_sync(0xffffffffu, r[e], m);
                r[e] = upper ? (p - r[e]) : (r[e] + p);
            }
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) {
            r[e] = r[e] * HadamardScale<D>::value;
            amax = fmaxf(amax, fabsf(r[e]));
        }
        amax = warp_max(amax);
        const float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < E; e += 2)
            packed |= e4m3x2_rn_sat(__fdiv_rn(r[e], s), __fdiv_rn(r[e + 1], s)) << (8 * e);
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
