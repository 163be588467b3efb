// latent_fp8.cu -- the FP8 latent cache: quantising latent rows into it, and
// sparse attention over it.
//
// Page: the diagram "DeepSeek Sparse Attention, one decode step in one layer
// (V3.2 sizes)": latents cached as "FP8 + bf16 RoPE", 656 B per row.  Row
// layout: [dc e4m3 codes | dc/128 fp32 scales | dr bf16 rotary values]; the
// latent part is quantised in blocks of 128 exactly as act_quant does (scale
// max(amax, 1e-4) / 448, code e4m3_rn_satfinite(x / scale), both divisions
// correctly rounded), the rotary part is rounded to bf16.
//
// Attention over the FP8 cache: at the V3.2 shapes (128 heads, 512 + 64) the
// tensor-core kernel of sparse_mla_tc.cu decodes each latent chunk while
// gathering it.  Other shapes run in two launches: a gather pass decodes each
// query row's selected rows (code * block scale, rounded to bf16; the rotary
// part copied) into a workspace, one row per selection slot, and the bf16
// sparse attention of sparse_mla.cu then attends over it with every query row
// as its own sequence and slot j at position j.
#include <cuda_fp8.h>

#include "common.cuh"
#include "quant.cuh"

namespace dsa {
namespace {

__host__ __device__ constexpr int64_t row_bytes(int dc, int dr) {
    return (int64_t)dc + (int64_t)(dc / 128) * 4 + (int64_t)dr * 2;
}

// One warp per latent row: lane l holds latent values [16l, 16l + 16) (8
// lanes per 128-block) and rotary values [2l, 2l + 2).
template <typename Tin>
__global__ void __launch_bounds__(256)
latent_quant_kernel(const Tin *__restrict__ kv, int64_t n_rows, int64_t n_vec, int dc, int dr,
                    uint8_t *__restrict__ out, int64_t out_row_stride) {
    const int lane = threadIdx.x & 31;
    const int dqk = dc + dr;
    const int64_t rb = row_bytes(dc, dr);
    const int64_t total = n_rows * n_vec;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const bool has_c = lane * 16 < dc;
    for (int64_t v = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); v < total;
         v += warps) {
        const Tin *src = kv + v * dqk;
        float x[16];
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 16; e++) {
            x[e] = has_c ? to_f32<Tin>(src[lane * 16 + e]) : 0.f;
            amax = fmaxf(amax, fabsf(x[e]));
        }
        // max over the 8 lanes of this lane's 128-block
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
        const float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
        const float rs = __frcp_rn(s);
        const int64_t row = v / n_vec, vi = v - row * n_vec;
        uint8_t *dst = out + row * out_row_stride + vi * rb;
        if (has_c) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; j++)
                w[j] = e4m3x2_rn_sat(div_rn_by(x[4 * j], s, rs), div_rn_by(x[4 * j + 1], s, rs)) |
                       e4m3x2_rn_sat(div_rn_by(x[4 * j + 2], s, rs), div_rn_by(x[4 * j + 3], s, rs)) << 16;
            uint32_t *d32 = reinterpret_cast<uint32_t *>(dst + lane * 16);
#pragma unroll
            for (int j = 0; j < 4; j++) d32[j] = w[j];
            if ((lane & 7) == 0) *reinterpret_cast<float *>(dst + dc + 4 * (lane >> 3)) = s;
        }
        if (2 * lane < dr) {
            const __nv_bfloat162 r2 = __floats2bfloat162_rn(to_f32<Tin>(src[dc + 2 * lane]),
                                                            to_f32<Tin>(src[dc + 2 * lane + 1]));
            *reinterpret_cast<__nv_bfloat162 *>(dst + dc + dc / 32 + 4 * lane) = r2;
        }
    }
}

// One warp per (query row, selection slot): decodes the selected FP8 row into
// slot j of the row's workspace block, or marks the slot empty (-1).
__global__ void __launch_bounds__(256)
latent_gather_kernel(const uint8_t *__restrict__ kv, int64_t t_max, const int32_t *__restrict__ idx,
                     int64_t rows, int S, int k, int dc, int dr, int64_t start_pos,
                     __nv_bfloat16 *__restrict__ g_rows, int32_t *__restrict__ g_idx, int *err) {
    const int lane = threadIdx.x & 31;
    const int dqk = dc + dr;
    const int64_t rb = row_bytes(dc, dr);
    const int64_t total = rows * k;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < total;
         u += warps) {
        const int64_t r = u / k;
        const int j = (int)(u - r * k);
        const int64_t b = r / S, s = r - b * S;
        const int32_t t = idx[u];
        bool valid = t >= 0 && (int64_t)t <= start_pos + s;
        if (valid && (int64_t)t >= t_max) {
            if (lane == 0) record_error(err, DSA_ERR_DEVICE);
            valid = false;
        }
        if (lane == 0) g_idx[u] = valid ? j : -1;
        if (!valid) continue;
        const uint8_t *src = kv + (b * t_max + t) * rb;
        __nv_bfloat16 *dst = g_rows + u * dqk;
        if (lane * 16 < dc) {
            const float sc = *reinterpret_cast<const float *>(src + dc + 4 * (lane >> 3));
            const uint32_t *c32 = reinterpret_cast<const uint32_t *>(src + lane * 16);
            uint32_t o[8];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint32_t w = c32[q];
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                        static_cast<__nv_fp8x2_storage_t>((w >> (16 * h)) & 0xFFFFu), __NV_E4M3);
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(f.x * sc, f.y * sc);
                    o[2 * q + h] = *reinterpret_cast<const uint32_t *>(&v2);
                }
            }
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + lane * 16);
            d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
            d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
        if (2 * lane < dr)
            reinterpret_cast<uint32_t *>(dst + dc)[lane] =
                reinterpret_cast<const uint32_t *>(src + dc + dc / 32)[lane];
    }
}

bool fp8_shape_ok(int dc, int dr) {
    return dc >= 128 && dc <= 512 && dc % 128 == 0 && dr >= 0 && dr <= 64 && dr % 8 == 0 &&
           dc + dr <= 576;
}

int64_t grid_for(int64_t warps_needed) {
    int64_t blocks = (warps_needed + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 32;
    if (blocks > cap) blocks = cap;
    return blocks > 0 ? blocks : 1;
}

struct Fp8Ws {
    size_t rows_bytes, idx_bytes, attn_bytes;
    size_t total() const { return rows_bytes + idx_bytes + attn_bytes; }
};

Fp8Ws fp8_workspace(int B, int S, int Hq, int dc, int dr, int k, bool tc) {
    const int64_t rows = (int64_t)B * S;
    Fp8Ws w;
    if (tc) {
        w.rows_bytes = 0;
        w.idx_bytes = 0;
        w.attn_bytes = sparse_mla_tc_workspace_bytes(B, S, k);
        return w;
    }
    w.rows_bytes = align_up((size_t)rows * k * (dc + dr) * sizeof(__nv_bfloat16), 256);
    w.idx_bytes = align_up((size_t)rows * k * sizeof(int32_t), 256);
    w.attn_bytes = sparse_mla_workspace_bytes((int)rows, 1, Hq, dc, dr, k, DSA_BF16);
    return w;
}

}  // namespace

bool latent_fp8_shape_ok(int dc, int dr) { return fp8_shape_ok(dc, dr); }

size_t sparse_mla_fp8_workspace_bytes(int B, int S, int Hq, int dc, int dr, int k) {
    return fp8_workspace(B, S, Hq, dc, dr, k, sparse_mla_fp8_tc_supported(Hq, dc, dr, k)).total();
}

dsa_status launch_sparse_mla_fp8(const void *q, const uint8_t *kv_fp8, int64_t t_max,
                                 const int32_t *idx, int B, int S, int Hq, int dc, int dr, int k,
                                 int64_t start_pos, float sm_scale, void *out, float *lse,
                                 void *workspace, cudaStream_t st) {
    // the decode-in-gather kernel reads rows with 16-byte loads (the entry
    // point requires a 16-byte aligned cache for these shapes)
    if (sparse_mla_fp8_tc_supported(Hq, dc, dr, k))
        return launch_sparse_mla_fp8_tc(q, kv_fp8, t_max, idx, B, S, k, start_pos, sm_scale, out,
                                        lse, workspace, st);
    const Fp8Ws w = fp8_workspace(B, S, Hq, dc, dr, k, false);
    char *ws = static_cast<char *>(workspace);
    __nv_bfloat16 *g_rows = reinterpret_cast<__nv_bfloat16 *>(ws);
    int32_t *g_idx = reinterpret_cast<int32_t *>(ws + w.rows_bytes);
    void *attn_ws = w.attn_bytes ? ws + w.rows_bytes + w.idx_bytes : nullptr;
    const int64_t rows = (int64_t)B * S;
    latent_gather_kernel<<<(unsigned)grid_for(rows * k), 256, 0, st>>>(
        kv_fp8, t_max, idx, rows, S, k, dc, dr, start_pos, g_rows, g_idx, device_error_word());
    const dsa_status e = launch_status();
    if (e != DSA_OK) return e;
    // every query row is a sequence of k decoded rows; slot j sits at position j
    return launch_sparse_mla(q, g_rows, k, g_idx, (int)rows, 1, Hq, dc, dr, k, k - 1, sm_scale,
                             DSA_BF16, out, lse, attn_ws, st);
}

}  // namespace dsa

extern "C" int64_t dsa_latent_row_bytes(int dc, int dr) { return dsa::row_bytes(dc, dr); }

extern "C" dsa_status dsa_latent_quant(const void *kv, dsa_dtype x_dtype, int64_t n_rows,
                                       int64_t n_vec, int dc, int dr, uint8_t *out,
                                       int64_t out_row_stride, dsa_stream_t stream) {
    if (n_rows < 0 || n_vec < 0) return DSA_ERR_INVALID_ARG;
    if (x_dtype != DSA_F32 && x_dtype != DSA_BF16) return DSA_ERR_INVALID_ARG;
    if (!dsa::fp8_shape_ok(dc, dr)) return DSA_ERR_UNSUPPORTED;
    if (n_rows == 0 || n_vec == 0) return DSA_OK;
    if (!kv || !out) return DSA_ERR_INVALID_ARG;
    const int64_t rb = dsa::row_bytes(dc, dr);
    if ((reinterpret_cast<uintptr_t>(kv) & 3) || (reinterpret_cast<uintptr_t>(out) & 3))
        return DSA_ERR_INVALID_ARG;
    if (n_rows > 1 && (out_row_stride < n_vec * rb || (out_row_stride & 3)))
        return DSA_ERR_INVALID_ARG;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const unsigned blocks = (unsigned)dsa::grid_for(n_rows * n_vec);
    if (x_dtype == DSA_BF16)
        dsa::latent_quant_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(kv), n_rows, n_vec, dc, dr, out, out_row_stride);
    else
        dsa::latent_quant_kernel<float><<<blocks, 256, 0, st>>>(
            static_cast<const float *>(kv), n_rows, n_vec, dc, dr, out, out_row_stride);
    return dsa::launch_status();
}

extern "C" size_t dsa_sparse_mla_attn_fp8_workspace_size(int B, int S, int Hq, int dc, int dr,
                                                         int k) {
    if (B <= 0 || S <= 0 || Hq <= 0 || k <= 0 || !dsa::fp8_shape_ok(dc, dr)) return 0;
    return dsa::sparse_mla_fp8_workspace_bytes(B, S, Hq, dc, dr, k);
}

extern "C" dsa_status dsa_sparse_mla_attn_fp8(const void *q, const uint8_t *kv_fp8, int64_t t_max,
                                              const int32_t *idx, int B, int S, int Hq, int dc,
                                              int dr, int k, int64_t start_pos, float sm_scale,
                                              void *out, float *lse, void *workspace,
                                              size_t workspace_bytes, dsa_stream_t stream) {
    if (B < 0 || S < 0 || Hq < 0 || k < 1 || start_pos < 0) return DSA_ERR_INVALID_ARG;
    if (!dsa::fp8_shape_ok(dc, dr)) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S * Hq == 0) return DSA_OK;
    if (start_pos + S > t_max) return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * S * k > INT32_MAX || (int64_t)B * S * Hq > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    if (!q || !kv_fp8 || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q) || !dsa::aligned16(out) || (reinterpret_cast<uintptr_t>(kv_fp8) & 3) ||
        (reinterpret_cast<uintptr_t>(idx) & 3))
        return DSA_ERR_INVALID_ARG;
    if (dsa::sparse_mla_fp8_tc_supported(Hq, dc, dr, k) && !dsa::aligned16(kv_fp8))
        return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::sparse_mla_fp8_workspace_bytes(B, S, Hq, dc, dr, k);
    if (need > 0 && (!workspace || workspace_bytes < need || !dsa::aligned16(workspace)))
        return DSA_ERR_WORKSPACE;
    return dsa::launch_sparse_mla_fp8(q, kv_fp8, t_max, idx, B, S, Hq, dc, dr, k, start_pos,
                                      sm_scale, out, lse, workspace,
                                      reinterpret_cast<cudaStream_t>(stream));
}
