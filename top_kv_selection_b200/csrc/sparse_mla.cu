// sparse_mla.cu -- sparse latent attention (MQA mode) over the selected rows.
//
// Pages: "DeepSeek Sparse Attention, one decode step in one layer (V3.2 sizes)"
// (core attention in MQA mode: 128 heads over the 2048 gathered latents, each
// latent row is key and value) and the MLA prefill excerpt of "DeepSeek-V3.2-Exp
// - Causal mask" (an index mask that is -inf everywhere except at the selected
// positions, plus the causal mask, added to the scores; softmax; value mix).  The latent row is [c | k_pe]
// (wkv_a output order); the query is already in latent space.
//
// bf16 at the V3.2 shapes (128 heads, 512 + 64) runs the tensor-core kernel of
// sparse_mla_tc.cu.  SIMT kernel (the fp32 test mode and other shapes):
// a warp owns one head of one query row and walks the selected rows with an
// online softmax; lane l holds dims l, l+32, ... of the query and of the
// output accumulator.
#include "common.cuh"

namespace dsa {
namespace {

constexpr int kHeadsPerCta = 8;
constexpr int kMaxDqkPerLane = 18;   // dc + dr <= 576
constexpr int kMaxDcPerLane = 16;    // dc <= 512

template <typename T>
__global__ void __launch_bounds__(32 * kHeadsPerCta)
sparse_mla_simt_kernel(const T *__restrict__ q, const T *__restrict__ kv, int64_t t_max,
                       const int32_t *__restrict__ idx, int S, int Hq, int dc, int dr, int k,
                       int64_t start_pos, float sm_scale, T *__restrict__ out,
                       float *__restrict__ lse, int *err) {
    const int lane = threadIdx.x & 31;
    const int head = blockIdx.y * kHeadsPerCta + (threadIdx.x >> 5);
    const int64_t row = blockIdx.x;                 // b * S + s
    if (head >= Hq) return;
    const int64_t b = row / S, s = row - b * S;
    const int dqk = dc + dr;
    const int nq = (dqk + 31) / 32;
    const int nc = dc / 32;

    float qr[kMaxDqkPerLane];
    const T *qh = q + (row * Hq + head) * dqk;
#pragma unroll
    for (int i = 0; i < kMaxDqkPerLane; i++) {
        const int d = lane + 32 * i;
        qr[i] = (i < nq && d < dqk) ? to_f32<T>(qh[d]) : 0.f;
    }
    float o[kMaxDcPerLane];
#pragma unroll
    for (int i = 0; i < kMaxDcPerLane; i++) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int32_t *sel = idx + row * k;
    const int64_t limit = start_pos + s;
    for (int j = 0; j < k; j++) {
        const int32_t t = sel[j];
        if (t < 0 || (int64_t)t > limit) continue;
        if ((int64_t)t >= t_max) {
            if (lane == 0) record_error(err, DSA_ERR_DEVICE);
            continue;
        }
        const T *c = kv + (b * t_max + t) * dqk;
        float cr[kMaxDqkPerLane];
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxDqkPerLane; i++) {
            const int d = lane + 32 * i;
            cr[i] = (i < nq && d < dqk) ? to_f32<T>(c[d]) : 0.f;
            part = fmaf(qr[i], cr[i], part);
        }
        const float z = warp_sum(part) * sm_scale;
        const float m_new = fmaxf(m, z);
        const float corr = expf(m - m_new);
        const float p = expf(z - m_new);
        l = l * corr + p;
#pragma unroll
        for (int i = 0; i < kMaxDcPerLane; i++)
            if (i < nc) o[i] = fmaf(p, cr[i], o[i] * corr);
        m = m_new;
    }
    T *oh = out + (row * Hq + head) * dc;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxDcPerLane; i++)
        if (i < nc) oh[lane + 32 * i] = from_f32<T>(o[i] * inv);
    if (lse && lane == 0) lse[row * Hq + head] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

size_t sparse_mla_workspace_bytes(int B, int S, int Hq, int dc, int dr, int k, dsa_dtype dt) {
    if (sparse_mla_tc_supported(Hq, dc, dr, k, dt)) return sparse_mla_tc_workspace_bytes(B, S, k);
    return 0;
}

dsa_status launch_sparse_mla(const void *q, const void *kv, int64_t t_max, const int32_t *idx,
                             int B, int S, int Hq, int dc, int dr, int k, int64_t start_pos,
                             float sm_scale, dsa_dtype dt, void *out, float *lse, void *ws,
                             cudaStream_t stream) {
    if ((int64_t)B * S * Hq == 0) return DSA_OK;
    if (sparse_mla_tc_supported(Hq, dc, dr, k, dt))
        return launch_sparse_mla_tc(q, kv, t_max, idx, B, S, k, start_pos, sm_scale, out, lse, ws,
                                    stream);
    dim3 grid((unsigned)(B * S), (unsigned)((Hq + kHeadsPerCta - 1) / kHeadsPerCta));
    int *err = device_error_word();
    if (dt == DSA_BF16)
        sparse_mla_simt_kernel<__nv_bfloat16><<<grid, 32 * kHeadsPerCta, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(kv), t_max,
            idx, S, Hq, dc, dr, k, start_pos, sm_scale, static_cast<__nv_bfloat16 *>(out), lse,
            err);
    else
        sparse_mla_simt_kernel<float><<<grid, 32 * kHeadsPerCta, 0, stream>>>(
            static_cast<const float *>(q), static_cast<const float *>(kv), t_max, idx, S, Hq, dc,
            dr, k, start_pos, sm_scale, static_cast<float *>(out), lse, err);
    return launch_status();
}

}  // namespace dsa

extern "C" size_t dsa_sparse_mla_attn_workspace_size(int B, int S, int Hq, int dc, int dr, int k,
                                                     dsa_dtype dt) {
    if (B <= 0 || S <= 0 || Hq <= 0 || k <= 0) return 0;
    return dsa::sparse_mla_workspace_bytes(B, S, Hq, dc, dr, k, dt);
}

extern "C" dsa_status dsa_sparse_mla_attn(const void *q, const void *kv_cache, int64_t t_max,
                                          const int32_t *idx, int B, int S, int Hq, int dc,
                                          int dr, int k, int64_t start_pos, float sm_scale,
                                          dsa_dtype dt, void *out, float *lse, void *workspace,
                                          size_t workspace_bytes, dsa_stream_t stream) {
    if (B < 0 || S < 0 || Hq < 0 || k < 1 || start_pos < 0 || dc < 0 || dr < 0)
        return DSA_ERR_INVALID_ARG;
    if (dt != DSA_F32 && dt != DSA_BF16) return DSA_ERR_INVALID_ARG;
    if (dc == 0 || dc % 32 != 0 || dc > 512 || dr % 8 != 0 || dc + dr > 576)
        return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S * Hq == 0) return DSA_OK;
    if (start_pos + S > t_max) return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * t_max > INT32_MAX || (int64_t)B * S * Hq > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    if (!q || !kv_cache || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q) || !dsa::aligned16(kv_cache) || !dsa::aligned16(out))
        return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::sparse_mla_workspace_bytes(B, S, Hq, dc, dr, k, dt);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DSA_ERR_WORKSPACE;
    return dsa::launch_sparse_mla(q, kv_cache, t_max, idx, B, S, Hq, dc, dr, k, start_pos,
                                  sm_scale, dt, out, lse, workspace,
                                  reinterpret_cast<cudaStream_t>(stream));
}
