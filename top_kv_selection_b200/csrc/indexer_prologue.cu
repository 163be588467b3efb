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
// G = D / 64 adjacent lanes hold one D-vector, 64 elements each, as in
// quant.cuh's rotate_quant_lanes; a warp holds 32 / G vectors (query head
// vectors first, then the new tokens' keys).  Rotary pairs are element j and
// element j + R/2 (j < R/2).  For D = 128 the two lanes split the vector on
// the element bit just below the pair's (bit 4 for R = 64, bit 5 for R = 128,
// bit 3 for R = 32 with bf16 input), so that both elements of a pair sit in
// one lane and each lane holds half of the pairs; other rotary widths keep
// contiguous halves, where every pair lies in part 0.  With (c, s) the angle
// of frequency j at the token's position, the lower element becomes
// x1*c - x2*s and the upper x1*s + x2*c (x1 lower, x2 upper), each product and
// sum rounded to fp32.  Then the butterfly, the scale and the codes of
// rotate_quant_lanes.  HBM-bound: 4*D (fp32) or 2*D (bf16) bytes in and D + 4
// bytes out per vector, plus the angles (R/2 * 8 bytes per token, L2-resident
// and staged once per warp pass when the pass covers at most two tokens).
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
    int small;              // every vector index fits in 31 bits
};

// A warp's vectors pass through shared memory: the warp copies them with
// coalesced 16-byte cp.async pieces (consecutive lanes, consecutive pieces), and
// lane o, which owns 64 elements of one vector, then reads its CPL pieces.
// Piece j of owner o sits at slot o * CPL + (j ^ (o % 8)): both the copies
// (8 consecutive lanes hit 8 different 16-byte bank groups) and the owners'
// reads (lanes o .. o + 7 at the same j, likewise) are free of bank conflicts.
// Two buffers per warp: the next vectors are in flight while these are
// rotated.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16u : 0u)
                 : "memory");
}

template <int D, typename Tin, int X> struct Stage {
    static constexpr int G = D / 64;                        // lanes per vector
    static constexpr int kVecs = 32 / G;                    // vectors per warp and pass
    static constexpr int kVecBytes = D * (int)sizeof(Tin);
    static constexpr int kBytes = kVecs * kVecBytes;        // one buffer
    static constexpr int kCPL = 64 * (int)sizeof(Tin) / 16; // pieces a lane owns (8 or 16)
    static constexpr int kPieces = kBytes / 16;

    // copies the vectors [base, base + kVecs) (zeros past `total`) into buf
    __device__ __forceinline__ static void issue(uint32_t buf, const PrologueArgs &a, int64_t base,
                                                 int64_t nq, int64_t total, int lane) {
        constexpr int kPerVec = kVecBytes / 16;
        constexpr int kEPC = 16 / (int)sizeof(Tin);           // elements per piece
        static_assert(G == 1 || kEPC <= (1 << X), "a piece stays within one lane's elements");
#pragma unroll
        for (int i = 0; i < kPieces / 32; i++) {
            const int c = lane + 32 * i;
            const int64_t v = base + c / kPerVec;
            const int cc = c % kPerVec, off = cc * 16;
            const bool valid = v < total;
            const uint8_t *src =
                v < nq ? static_cast<const uint8_t *>(a.q) + v * kVecBytes
                       : static_cast<const uint8_t *>(a.k) + (valid ? v - nq : 0) * kVecBytes;
            // owner lane (vector, part) and the piece's place among its registers
            const int e0 = cc * kEPC;
            const int p = G == 2 ? (e0 >> X) & 1 : 0;
            const int i0 = G == 2 ? ((e0 >> (X + 1)) << X) | (e0 & ((1 << X) - 1)) : e0;
            const int o = (c / kPerVec) * G + p, j = i0 / kEPC;
            cp_async16_zfill(buf + (uint32_t)(o * kCPL + (j ^ (o & 7))) * 16u, src + off, valid);
        }
    }
    // lane o's 64 elements from buf, as fp32
    __device__ __forceinline__ static void read(uint32_t buf, int o, float (&r)[64]) {
#pragma unroll
        for (int j = 0; j < kCPL; j++) {
            uint4 t;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(t.x), "=r"(t.y), "=r"(t.z), "=r"(t.w)
                         : "r"(buf + (uint32_t)(o * kCPL + (j ^ (o & 7))) * 16u));
            if constexpr (sizeof(Tin) == 4) {
                r[4 * j] = __uint_as_float(t.x);
                r[4 * j + 1] = __uint_as_float(t.y);
                r[4 * j + 2] = __uint_as_float(t.z);
                r[4 * j + 3] = __uint_as_float(t.w);
            } else {
                const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    r[8 * j + 2 * h] = __uint_as_float(w[h] << 16);
                    r[8 * j + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
                }
            }
        }
    }
};

// Token (b * S + s) of query vector v, and the position s of vector v's token
// (a query head vector or a key); 32-bit arithmetic when the problem fits.
__device__ __forceinline__ int64_t token_of(const PrologueArgs &a, int64_t v) {
    return a.small ? (int64_t)((uint32_t)v / (uint32_t)a.H) : v / a.H;
}
__device__ __forceinline__ int token_pos(const PrologueArgs &a, int64_t v, int64_t nq,
                                         int64_t total) {
    if (v >= total) return 0;
    const int64_t t = v < nq ? token_of(a, v) : v - nq;
    return a.small ? (int)((uint32_t)t % (uint32_t)a.S) : (int)(t % a.S);
}

// Two fp32 products rounded to nearest, never fused into a following add
// (an explicit rounding mode keeps ptxas from contracting it into an fma).
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 pa, pb, pr;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "mul.rn.f32x2 pr, pa, pb;\n\tmov.b64 {%0, %1}, pr;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// The angles of a pass whose vectors are all query heads of at most two
// tokens (every pass when H >= 16 and H divides by 16) are copied next to its
// vectors: rows t_lo and t_lo + 1 of the table, R floats pairs each; other
// passes (the keys, few heads) read the table directly.
__device__ __forceinline__ bool angles_staged(const PrologueArgs &a, int64_t base, int n,
                                              int64_t nq, int64_t *t_lo) {
    if (base + n > nq) return false;
    const int64_t t0 = token_of(a, base), t1 = token_of(a, base + n - 1);
    *t_lo = t0;
    return t1 - t0 <= 1;
}
template <int R>
__device__ __forceinline__ void issue_angles(uint32_t dst, const PrologueArgs &a, int64_t base,
                                             int n, int64_t nq, int lane) {
    int64_t t_lo;
    if (!angles_staged(a, base, n, nq, &t_lo)) return;
    const bool two = token_of(a, base + n - 1) > t_lo;
    constexpr int kPer = R / 4;                  // 16-byte pieces per row
#pragma unroll
    for (int c = lane; c < 2 * kPer; c += 32) {
        const int row = c / kPer;
        const int64_t t = t_lo + row;
        const int sp = row == 0 || two ? (a.small ? (int)((uint32_t)t % (uint32_t)a.S) : (int)(t % a.S)) : 0;
        cp_async16_zfill(dst + (uint32_t)c * 16u, a.cs + (int64_t)sp * R + (c % kPer) * 4,
                         row == 0 || two);
    }
}

// The lane split of a 128-vector for rotary part R: on the bit just below the
// rotary pair's bit, so that both lanes of a vector hold half of the pairs
// (element j and j + R/2 in the same lane); bit 6 (contiguous halves) when
// the part is too short for a 16-byte piece to stay in one lane.
template <int D, int R, typename Tin> constexpr int lane_split() {
    if (D != 128) return 6;
    if (R == 128) return 5;
    if (R == 64) return 4;
    if (R == 32 && sizeof(Tin) == 2) return 3;
    return 6;
}

template <int D, int R, typename Tin>
__global__ void __launch_bounds__(256, 2) indexer_prologue_kernel(const PrologueArgs a) {
    constexpr int X = lane_split<D, R, Tin>();
    using St = Stage<D, Tin, X>;
    constexpr int G = D / 64;                  // lanes per vector
    extern __shared__ __align__(16) uint8_t stage_smem[];
    const int lane = threadIdx.x & 31;
    const int part = lane % G;
    const int64_t nq = (int64_t)a.B * a.S * a.H;
    const int64_t total = nq + (int64_t)a.B * a.S;
    const int64_t per_warp = St::kVecs;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t stride = warps * per_warp;
    const int warp = threadIdx.x >> 5;
    const uint32_t buf0 = (uint32_t)__cvta_generic_to_shared(stage_smem) +
                          (uint32_t)(warp * 2 * St::kBytes);
    // the staged angles: after the 8 warps' vector buffers, two rows per buffer
    constexpr int kAngBytes = 2 * (R > 0 ? R : 4) * 4;
    const int ang_off = 8 * 2 * St::kBytes + warp * 2 * kAngBytes;
    const uint32_t ang0 = (uint32_t)__cvta_generic_to_shared(stage_smem) + (uint32_t)ang_off;
    int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + warp) * per_warp;
    if (base < total) {
        St::issue(buf0, a, base, nq, total, lane);
        if constexpr (R > 0) issue_angles<R>(ang0, a, base, St::kVecs, nq, lane);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int it = 0; base < total; base += stride, it++) {
        const uint32_t cur = buf0 + (uint32_t)((it & 1) * St::kBytes);
        // the next pass's vectors (and angles) into the other buffer (its reads
        // ended at the __syncwarp of the previous pass), then this pass's pieces
        if (base + stride < total) {
            const int nb = (it + 1) & 1;
            St::issue(buf0 + (uint32_t)(nb * St::kBytes), a, base + stride, nq, total, lane);
            if constexpr (R > 0)
                issue_angles<R>(ang0 + (uint32_t)(nb * kAngBytes), a, base + stride, St::kVecs, nq,
                                lane);
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();
        const int64_t v = base + lane / G;   // both lanes of a vector agree on `valid`
        const bool valid = v < total;
        const bool is_q = v < nq;
        const int64_t t = is_q ? token_of(a, v) : v - nq;   // token index b * S + s
        const int s = valid ? token_pos(a, v, nq, total) : 0;
        float r[64];
        St::read(cur, lane, r);
        // this vector's angles: the staged copy, or the table
        const float4 *cs = nullptr;
        if constexpr (R > 0) {
            int64_t t_lo = 0;
            cs = angles_staged(a, base, St::kVecs, nq, &t_lo)
                     ? reinterpret_cast<const float4 *>(stage_smem + ang_off + (it & 1) * kAngBytes +
                                                        (int)(t - t_lo) * R * 4)
                     : reinterpret_cast<const float4 *>(a.cs + (int64_t)s * R);
        }
        if constexpr (R > 0 && X < 6) {
            // both lanes: pairs (register m, register 2^X + m), m < 2^X, at
            // frequency part * 2^X + m
            if (valid) {
                constexpr int M = 1 << X;
                const float4 *cp = cs + part * (M / 2);
#pragma unroll
                for (int m2 = 0; m2 < M / 2; m2++) {
                    const float4 c2 = cp[m2];
                    const float cc[2] = {c2.x, c2.z}, ss[2] = {c2.y, c2.w};
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        const int m = 2 * m2 + u;
                        const float x1 = r[m], x2 = r[M + m];
                        r[m] = __fsub_rn(__fmul_rn(x1, cc[u]), __fmul_rn(x2, ss[u]));
                        r[M + m] = __fadd_rn(__fmul_rn(x1, ss[u]), __fmul_rn(x2, cc[u]));
                    }
                }
            }
        } else if constexpr (R > 0 && R <= 64) {
            if (part == 0 && valid) {
                // lower x1 c - x2 s, upper x1 s + x2 c, each product and sum
                // rounded once: two packed products and a packed sum
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
        // every lane is done with this pass's buffer (vectors and angles)
        __syncwarp();
        uint32_t codes[16];
        float sc;
        rotate_quant_lanes<D, X>(r, codes, &sc, a.ue8m0 != 0);
        if (valid) {
            uint8_t *dst;
            float *dscale;
            if (is_q) {
                dst = a.q_fp8 + v * D;
                dscale = a.q_scale + v;
            } else {
                const int64_t bb = a.small ? (int64_t)((uint32_t)t / (uint32_t)a.S) : t / a.S;
                const int64_t row = bb * a.t_max + a.start_pos + s;
                dst = a.k_cache + row * D;
                dscale = a.k_scale + row;
            }
            // registers run k .. run k + run - 1 are consecutive elements, run =
            // min(16, 2^X) under the lane split (contiguous halves: 16)
            static_assert(G == 1 || X >= 3, "8-code runs at least");
            if constexpr (G == 2 && X == 3) {
#pragma unroll
                for (int m = 0; m < 8; m++)
                    *reinterpret_cast<uint2 *>(dst + split_element<X>(8 * m, part)) =
                        make_uint2(codes[2 * m], codes[2 * m + 1]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++)
                    *reinterpret_cast<uint4 *>(dst + (G == 2 ? split_element<X>(16 * i, part) : 16 * i)) =
                        make_uint4(codes[4 * i], codes[4 * i + 1], codes[4 * i + 2], codes[4 * i + 3]);
            }
            if (part == 0) *dscale = sc;
        }
    }
}

template <int D, int R, typename Tin>
dsa_status launch_r(const PrologueArgs &a, cudaStream_t stream) {
    using St = Stage<D, Tin, lane_split<D, R, Tin>()>;
    const int64_t total = (int64_t)a.B * a.S * (a.H + 1);
    const int64_t per_block = 8 * St::kVecs;
    int64_t blocks = (total + per_block - 1) / per_block;
    const size_t smem = (size_t)8 * 2 * St::kBytes + (size_t)8 * 2 * (2 * (R > 0 ? R : 4) * 4);
    // every SM holds as many CTAs as its shared memory and registers allow;
    // the warps stride over the vectors
    const int per_sm = smem * 2 <= 227 * 1024 ? 2 : 1;
    const int64_t cap = (int64_t)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (cudaFuncSetAttribute(indexer_prologue_kernel<D, R, Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DSA_ERR_CUDA;
    indexer_prologue_kernel<D, R, Tin><<<(unsigned)blocks, 256, smem, stream>>>(a);
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
    a.small = (int64_t)B * S * ((int64_t)H + 1) + 64 <= INT32_MAX ? 1 : 0;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = x_dtype == DSA_BF16;
    if (d == 128)
        return bf ? dsa::launch<128, __nv_bfloat16>(a, st) : dsa::launch<128, float>(a, st);
    return bf ? dsa::launch<64, __nv_bfloat16>(a, st) : dsa::launch<64, float>(a, st);
}
