// indexer_prologue.cu -- the indexer's query and key preparation in one pass:
// rotary embedding of the first rope_dim elements (not interleaved),
// rotate_activation, act_quant (fp32 or ue8m0 scale), and the key's cache
// append.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward, query
// and key preparation: the first rope_head_dim elements of each query head
// and of the key get the rotary embedding (not interleaved) and are put back
// in front of the rest; both are then rotated (rotate_activation) and
// quantised (act_quant with the configured scale format), and the key's codes
// and scale are written into the caches at positions start_pos .. end_pos-1.
//
// G = D / 64 adjacent lanes hold one D-vector, 64 contiguous elements each
// (lane part p: elements [64p, 64p + 64)), as in quant.cuh's
// rotate_quant_lanes; a warp holds 32 / G vectors (query head vectors first,
// then the new tokens' keys).  Rotary pairs are element j and element j + R/2
// (j < R/2).  For R <= 64 both live in part 0's registers; for R = 128 (D = 128)
// they are the same register of the two lanes of a vector, one shuffle apart.
// With (c, s) the angle of frequency j at the token's position, the lower
// element becomes x1*c - x2*s and the upper x1*s + x2*c (x1 lower, x2 upper),
// each product and sum rounded to fp32.  Then the butterfly, the scale and the
// codes of rotate_quant_lanes.  HBM-bound: 4*D (fp32) or 2*D (bf16) bytes in
// and D + 4 bytes out per vector, plus the angles (R/2 * 8 bytes per token,
// L2-resident and the same address for every head of a token).
#include "common.cuh"
#include "quant.cuh"

namespace dsa {
namespace {

struct PrologueArgs {
    const void *q;          // [B, S, H, D]
    const void *k;          // [B, S, D]
    const float *cs;        // [S, R/2, 2] (cos, sin)
    uint8_t *q_fp8;         // [B, S, H, D]
    float *q_scale;         // [B, S, H]
    uint8_t *k_cache;       // [B, t_max, D]
    float *k_scale;         // [B, t_max]
    int64_t start_pos, t_max;
    int B, S, H, R;
    int ue8m0;
};

// Loads 64 contiguous elements (fp32 or bf16) as fp32; zeros when !valid.
template <typename Tin>
__device__ __forceinline__ void load64(const Tin *src, bool valid, float (&r)[64]) {
    if constexpr (sizeof(Tin) == 4) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float4 t = valid ? reinterpret_cast<const float4 *>(src)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            r[4 * i] = t.x; r[4 * i + 1] = t.y; r[4 * i + 2] = t.z; r[4 * i + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint4 t = valid ? reinterpret_cast<const uint4 *>(src)[i] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int h = 0; h < 4; h++) {
                r[8 * i + 2 * h] = __uint_as_float(w[h] << 16);
                r[8 * i + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
            }
        }
    }
}

template <int D, int R, typename Tin>
__global__ void __launch_bounds__(256, 2) indexer_prologue_kernel(const PrologueArgs a) {
    constexpr int G = D / 64;                  // lanes per vector
    const int lane = threadIdx.x & 31;
    const int part = lane % G;
    const int64_t nq = (int64_t)a.B * a.S * a.H;
    const int64_t total = nq + (int64_t)a.B * a.S;
    const int64_t per_warp = 32 / G;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * per_warp;
         base < total; base += warps * per_warp) {
        const int64_t v = base + lane / G;   // both lanes of a vector agree on `valid`
        const bool valid = v < total;
        const bool is_q = v < nq;
        const int64_t t = is_q ? v / a.H : v - nq;   // token index b * S + s
        const int s = valid ? (int)(t % a.S) : 0;
        float r[64];
        if (is_q) load64<Tin>(static_cast<const Tin *>(a.q) + v * D + part * 64, valid, r);
        else load64<Tin>(static_cast<const Tin *>(a.k) + t * D + part * 64, valid, r);
        if constexpr (R > 0 && R <= 64) {
            if (part == 0 && valid) {
                const float4 *cs = reinterpret_cast<const float4 *>(a.cs + (int64_t)s * R);
#pragma unroll
                for (int j2 = 0; j2 < R / 4; j2++) {            // two frequencies per float4
                    const float4 c2 = cs[j2];
                    const float cc[2] = {c2.x, c2.z}, ss[2] = {c2.y, c2.w};
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        const int j = 2 * j2 + u;
                        const float x1 = r[j], x2 = r[j + R / 2];
                        r[j] = __fsub_rn(__fmul_rn(x1, cc[u]), __fmul_rn(x2, ss[u]));
                        r[j + R / 2] = __fadd_rn(__fmul_rn(x1, ss[u]), __fmul_rn(x2, cc[u]));
                    }
                }
            }
        } else if constexpr (R == 128) {
            static_assert(D == 128, "rotary part within the vector");
            const float4 *cs = reinterpret_cast<const float4 *>(a.cs + (int64_t)s * R);
            const bool upper = part == 1;
#pragma unroll
            for (int j2 = 0; j2 < 32; j2++) {
                const float4 c2 = valid ? cs[j2] : make_float4(1.f, 0.f, 1.f, 0.f);
                const float cc[2] = {c2.x, c2.z}, ss[2] = {c2.y, c2.w};
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const int j = 2 * j2 + u;
                    const float p = __shfl_xor_sync(0xffffffffu, r[j], 1);
                    r[j] = upper ? __fadd_rn(__fmul_rn(p, ss[u]), __fmul_rn(r[j], cc[u]))
                                 : __fsub_rn(__fmul_rn(r[j], cc[u]), __fmul_rn(p, ss[u]));
                }
            }
        }
        uint32_t codes[16];
        float sc;
        rotate_quant_lanes<D>(r, codes, &sc, a.ue8m0 != 0);
        if (valid) {
            uint8_t *dst;
            float *dscale;
            if (is_q) {
                dst = a.q_fp8 + v * D;
                dscale = a.q_scale + v;
            } else {
                const int64_t row = (t / a.S) * a.t_max + a.start_pos + s;
                dst = a.k_cache + row * D;
                dscale = a.k_scale + row;
            }
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + part * 64);
#pragma unroll
            for (int i = 0; i < 4; i++)
                d4[i] = make_uint4(codes[4 * i], codes[4 * i + 1], codes[4 * i + 2], codes[4 * i + 3]);
            if (part == 0) *dscale = sc;
        }
    }
}

template <int D, int R, typename Tin>
dsa_status launch_r(const PrologueArgs &a, cudaStream_t stream) {
    const int64_t total = (int64_t)a.B * a.S * (a.H + 1);
    const int64_t per_block = 8 * (32 / (D / 64));
    int64_t blocks = (total + per_block - 1) / per_block;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    indexer_prologue_kernel<D, R, Tin><<<(unsigned)blocks, 256, 0, stream>>>(a);
    return launch_status();
}

template <int D, typename Tin>
dsa_status launch(const PrologueArgs &a, cudaStream_t stream) {
    switch (a.R) {
    case 0: return launch_r<D, 0, Tin>(a, stream);
    case 8: return launch_r<D, 8, Tin>(a, stream);
    case 16: return launch_r<D, 16, Tin>(a, stream);
    case 32: return launch_r<D, 32, Tin>(a, stream);
    case 64: return launch_r<D, 64, Tin>(a, stream);
    default:
        if constexpr (D == 128) return launch_r<D, 128, Tin>(a, stream);
        return DSA_ERR_UNSUPPORTED;
    }
}

bool rope_dim_ok(int R, int d) {
    return R == 0 || R == 8 || R == 16 || R == 32 || R == 64 || (R == 128 && d == 128);
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_indexer_prologue(const void *q, const void *k, dsa_dtype x_dtype, int B,
                                           int S, int H, int d, int rope_dim, const float *rope_cs,
                                           dsa_scale_fmt scale_fmt, int64_t start_pos,
                                           int64_t t_max, uint8_t *q_fp8, float *q_scale,
                                           uint8_t *k_cache, float *k_scale,
                                           dsa_stream_t stream) {
    if (B < 0 || S < 0 || H < 0 || start_pos < 0 || t_max < 0) return DSA_ERR_INVALID_ARG;
    if (x_dtype != DSA_F32 && x_dtype != DSA_BF16) return DSA_ERR_INVALID_ARG;
    if (scale_fmt != DSA_SCALE_F32 && scale_fmt != DSA_SCALE_UE8M0) return DSA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return DSA_ERR_UNSUPPORTED;
    if (!dsa::rope_dim_ok(rope_dim, d)) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S == 0) return DSA_OK;
    if (start_pos + S > t_max) return DSA_ERR_INVALID_ARG;
    if (!k || !k_cache || !k_scale || (H > 0 && (!q || !q_fp8 || !q_scale)) ||
        (rope_dim > 0 && !rope_cs))
        return DSA_ERR_INVALID_ARG;
    if ((H > 0 && (!dsa::aligned16(q) || !dsa::aligned16(q_fp8) ||
                   (reinterpret_cast<uintptr_t>(q_scale) & 3))) ||
        !dsa::aligned16(k) || (reinterpret_cast<uintptr_t>(k_cache) & 15) ||
        (reinterpret_cast<uintptr_t>(k_scale) & 3) ||
        (reinterpret_cast<uintptr_t>(rope_cs) & 15))
        return DSA_ERR_INVALID_ARG;
    dsa::PrologueArgs a;
    a.q = q;
    a.k = k;
    a.cs = rope_cs;
    a.q_fp8 = q_fp8;
    a.q_scale = q_scale;
    a.k_cache = k_cache;
    a.k_scale = k_scale;
    a.start_pos = start_pos;
    a.t_max = t_max;
    a.B = B;
    a.S = S;
    a.H = H;
    a.R = rope_dim;
    a.ue8m0 = scale_fmt == DSA_SCALE_UE8M0 ? 1 : 0;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = x_dtype == DSA_BF16;
    if (d == 128)
        return bf ? dsa::launch<128, __nv_bfloat16>(a, st) : dsa::launch<128, float>(a, st);
    return bf ? dsa::launch<64, __nv_bfloat16>(a, st) : dsa::launch<64, float>(a, st);
}
