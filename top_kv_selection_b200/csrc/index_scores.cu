// index_scores.cu -- fp8_index scoring with the weight fold and the causal mask.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward:
//   weights = weights_proj(x) * n_heads^-1/2; weights = weights * q_scale * softmax_scale
//   index_score = fp8_index(q_fp8, weights, k_cache, k_scale); index_score += mask
// and the diagram's I(t,s) = sum_j w_j ReLU(q_j . k_s).
//
// General kernel: one CTA scores 128 consecutive tokens of one query row
// (b, s); each thread owns one token, decodes its FP8 key into registers and
// runs the per-head dot products against the query tile held in shared
// memory (fp32, read as broadcasts).  The weight fold is computed once per CTA.
#include "common.cuh"

namespace dsa {
namespace {

constexpr int kTokPerCta = 128;

template <int D>
__global__ void __launch_bounds__(kTokPerCta)
index_scores_simt_kernel(const uint8_t *__restrict__ q_fp8, const float *__restrict__ q_scale,
                         const float *__restrict__ w, const uint8_t *__restrict__ k_cache,
                         const float *__restrict__ k_scale, int64_t t_max, int S, int H,
                         int64_t start_pos, int64_t T, float head_scale, float softmax_scale,
                         float *__restrict__ scores) {
    extern __shared__ float smem[];
    float *qs = smem;                 // [H][D] decoded query codes
    float *wf = smem + H * D;         // [H] folded weights
    const int64_t row = blockIdx.x;   // b * S + s
    const int64_t b = row / S, s = row - b * S;
    const uint8_t *qrow = q_fp8 + row * H * D;
    for (int i = threadIdx.x; i < H * D; i += blockDim.x) qs[i] = e4m3_to_f32(qrow[i]);
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        float t = __fmul_rn(w[row * H + h], head_scale);
        t = __fmul_rn(t, q_scale[row * H + h]);
        wf[h] = __fmul_rn(t, softmax_scale);
    }
    __syncthreads();

    const int64_t t = (int64_t)blockIdx.y * kTokPerCta + threadIdx.x;
    if (t >= T) return;
    float *dst = scores + row * T + t;
    if (t > start_pos + s) {
        *dst = -INFINITY;
        return;
    }
    float kf[D];
    const uint4 *krow = reinterpret_cast<const uint4 *>(k_cache + (b * t_max + t) * D);
#pragma unroll
    for (int c = 0; c < D / 16; c++) {
        uint4 v = __ldg(krow + c);
        e4m3x4_to_f32(v.x, kf[16 * c + 0], kf[16 * c + 1], kf[16 * c + 2], kf[16 * c + 3]);
        e4m3x4_to_f32(v.y, kf[16 * c + 4], kf[16 * c + 5], kf[16 * c + 6], kf[16 * c + 7]);
        e4m3x4_to_f32(v.z, kf[16 * c + 8], kf[16 * c + 9], kf[16 * c + 10], kf[16 * c + 11]);
        e4m3x4_to_f32(v.w, kf[16 * c + 12], kf[16 * c + 13], kf[16 * c + 14], kf[16 * c + 15]);
    }
    float acc = 0.f;
    for (int h = 0; h < H; h++) {
        const float4 *qh = reinterpret_cast<const float4 *>(qs + h * D);
        float dot = 0.f;
#pragma unroll
        for (int d4 = 0; d4 < D / 4; d4++) {
            float4 q4 = qh[d4];
            dot = fmaf(q4.x, kf[4 * d4 + 0], dot);
            dot = fmaf(q4.y, kf[4 * d4 + 1], dot);
            dot = fmaf(q4.z, kf[4 * d4 + 2], dot);
            dot = fmaf(q4.w, kf[4 * d4 + 3], dot);
        }
        acc = fmaf(wf[h], fmaxf(dot, 0.f), acc);
    }
    *dst = k_scale[b * t_max + t] * acc;
}

}  // namespace

dsa_status launch_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                               const uint8_t *k_cache, const float *k_scale, int64_t t_max, int B,
                               int S, int H, int D, int64_t start_pos, int64_t T,
                               float softmax_scale, float *scores, cudaStream_t stream) {
    if ((int64_t)B * S * T == 0) return DSA_OK;
    const float head_scale = (float)(1.0 / sqrt((double)H));
    const size_t smem = (size_t)H * D * sizeof(float) + (size_t)H * sizeof(float);
    dim3 grid((unsigned)(B * S), (unsigned)((T + kTokPerCta - 1) / kTokPerCta));
    if (D == 128) {
        cudaFuncSetAttribute(index_scores_simt_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        index_scores_simt_kernel<128><<<grid, kTokPerCta, smem, stream>>>(
            q_fp8, q_scale, w, k_cache, k_scale, t_max, S, H, start_pos, T, head_scale,
            softmax_scale, scores);
    } else {
        cudaFuncSetAttribute(index_scores_simt_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        index_scores_simt_kernel<64><<<grid, kTokPerCta, smem, stream>>>(
            q_fp8, q_scale, w, k_cache, k_scale, t_max, S, H, start_pos, T, head_scale,
            softmax_scale, scores);
    }
    return launch_status();
}

}  // namespace dsa

extern "C" dsa_status dsa_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                                       const uint8_t *k_cache, const float *k_scale,
                                       int64_t t_max, int B, int S, int H, int D,
                                       int64_t start_pos, int64_t T, float softmax_scale,
                                       float *scores, dsa_stream_t stream) {
    if (B < 0 || S < 0 || T < 0 || start_pos < 0 || H < 1) return DSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
    if (H > 256) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S * T == 0) return DSA_OK;
    if (T > t_max || start_pos + S > T) return DSA_ERR_INVALID_ARG;
    if ((T + 127) / 128 > 65535) return DSA_ERR_UNSUPPORTED;
    if (!q_fp8 || !q_scale || !w || !k_cache || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q_fp8) || !dsa::aligned16(k_cache)) return DSA_ERR_INVALID_ARG;
    return dsa::launch_index_scores(q_fp8, q_scale, w, k_cache, k_scale, t_max, B, S, H, D,
                                    start_pos, T, softmax_scale, scores,
                                    reinterpret_cast<cudaStream_t>(stream));
}
