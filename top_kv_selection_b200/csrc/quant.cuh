// quant.cuh -- rotate_activation + act_quant of one D-vector by one warp
// (rotate_quant_warp) or by D / 64 lanes (rotate_quant_lanes).
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward
// (rotate_activation, then act_quant with one scale per vector).
//
// Lane L holds elements [E*L, E*L + E), E = D / 32.  Butterfly stage h pairs
// element i with i ^ h: for h < E both live in the lane's registers,
// otherwise in lane L ^ (h / E) at the same register slot.  The lower element
// becomes a + b and the upper a - b, in fp32, stages in the order h = 1, 2, 4,
// ..., D/2 -- the same dataflow as the plain in-place transform, so the result
// is bit-identical to it.  Then one multiply by fp32(D^-1/2), a warp max of
// |x|, scale = max(amax, 1e-4) / 448 and the e4m3 codes of x / scale (round to
// nearest even, saturate to +-448), both divisions correctly rounded (the
// per-element one by div_rn_by from the vector's reciprocal).
#pragma once

#include "common.cuh"

namespace dsa {

template <int D> struct HadamardScale;
template <> struct HadamardScale<64> { static constexpr float value = 0.125f; };
// nearest fp32 to 128^-1/2 = sqrt(2)/16: 0x3DB504F3
template <> struct HadamardScale<128> { static constexpr float value = 0x1.6a09e6p-4f; };

// Two fp32 -> two e4m3 codes packed as (lo | hi << 8); the first PTX source
// operand fills the upper byte.
__device__ __forceinline__ uint32_t e4m3x2_rn_sat(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// x / s correctly rounded, given rs = RN(1/s) (one correctly rounded
// reciprocal per vector): Markstein's FMA correction -- q0 = RN(x * rs),
// e = x - q0 * s exactly (one FMA), q = RN(q0 + e * rs) -- which yields RN(x / s)
// when no intermediate overflows or underflows (here |x / s| <= 448 and
// s >= 1e-4 / 448).
__device__ __forceinline__ float div_rn_by(float x, float s, float rs) {
    const float q0 = __fmul_rn(x, rs);
    const float e = __fmaf_rn(-q0, s, x);
    return __fmaf_rn(e, rs, q0);
}

// The ue8m0 scale format: the smallest power of two not below s (s positive
// and normal): keep the exponent when the significand bits are zero, else
// step it up by one.
__device__ __forceinline__ float pow2_ceil(float s) {
    const uint32_t b = __float_as_uint(s);
    return (b & 0x007FFFFFu) ? __uint_as_float((b & 0x7F800000u) + 0x00800000u) : s;
}

// Rotates and quantises the vector held in r (this lane's E elements).
// Returns this lane's E codes packed little-endian; *scale gets the vector's
// scale (same value in every lane), rounded up to a power of two when ue8m0.
// All 32 lanes must call it.
template <int D>
__device__ __forceinline__ uint32_t rotate_quant_warp(float (&r)[D / 32], float *scale,
                                                      bool ue8m0 = false) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 1; h < E; h <<= 1) {
#pragma unroll
        for (int e = 0; e < E; e++) {
            if (e & h) continue;
            const float a = r[e], b = r[e + h];
            r[e] = a + b;
            r[e + h] = a - b;
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < E; e++) {
            const float p = __shfl_xor_sync(0xffffffffu, r[e], m);
            r[e] = upper ? __fsub_rn(p, r[e]) : __fadd_rn(r[e], p);
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; e++) {
        r[e] = __fmul_rn(r[e], HadamardScale<D>::value);
        amax = fmaxf(amax, fabsf(r[e]));
    }
    amax = warp_max(amax);
    float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
    if (ue8m0) s = pow2_ceil(s);
    const float rs = __frcp_rn(s);
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < E; e += 2)
        packed |= e4m3x2_rn_sat(div_rn_by(r[e], s, rs), div_rn_by(r[e + 1], s, rs)) << (8 * e);
    *scale = s;
    return packed;
}

// The same rotation and quantisation with the vector split over G = D / 64
// adjacent lanes, 64 elements each.  For D = 128 the lane pair splits the
// vector on element bit X: lane part p holds the elements whose bit X is p, in
// register order (register i holds element ((i >> X) << (X + 1)) | (p << X) |
// (i & (2^X - 1)); X = 6, the default, gives part p the elements
// [64p, 64p + 64)).  Butterfly stages run over element bits 0, 1, ..., D-1's
// top bit in that order; the stage on bit X pairs the two lanes (the lane
// holding the lower element takes a + b, the other a - b), every other stage
// pairs two registers of a lane.  Every lane of the warp must call it (lanes
// of a vector that does not exist pass zeros).  codes[j] holds the e4m3 codes
// of registers 4j .. 4j + 3, little-endian.
//
// Stages on register strides >= 2, the scaling and the division run on packed
// fp32 pairs (one instruction for two elements, each rounded as the scalar
// operation would be: a - b as a + (-b), p - a as fma(a, -1, p),
// fma(-q0, s, x) as fma(q0, -s, x)), so the results are bit-identical to the
// scalar form.
template <int D, int X = 6>
__device__ __forceinline__ void rotate_quant_lanes(float (&r)[64], uint32_t (&codes)[16],
                                                   float *scale, bool ue8m0 = false) {
    static_assert(D == 64 || D == 128, "one or two lanes per vector");
    static_assert(D == 64 ? X == 6 : (X >= 1 && X <= 6), "lane split bit");
    constexpr int kBits = D == 128 ? 7 : 6;
#pragma unroll
    for (int b = 0; b < kBits; b++) {
        if (D == 128 && b == X) {
            // lower lane: a + p; upper lane: p - a = fma(a, -1, p)
            const float sg = (threadIdx.x & 1) ? -1.f : 1.f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                const float2 p = make_float2(__shfl_xor_sync(0xffffffffu, r[e], 1),
                                             __shfl_xor_sync(0xffffffffu, r[e + 1], 1));
                const float2 v = __ffma2_rn(make_float2(r[e], r[e + 1]), sg2, p);
                r[e] = v.x;
                r[e + 1] = v.y;
            }
            continue;
        }
        const int h = (D == 128 && b > X) ? 1 << (b - 1) : 1 << b;   // register stride
        if (h == 1) {
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                const float a = r[e], c = r[e + 1];
                r[e] = a + c;
                r[e + 1] = a - c;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                if (e & h) continue;
                const float2 a = make_float2(r[e], r[e + 1]);
                const float2 c = make_float2(r[e + h], r[e + h + 1]);
                const float2 sum = __fadd2_rn(a, c);
                const float2 dif = __fadd2_rn(a, make_float2(-c.x, -c.y));
                r[e] = sum.x;
                r[e + 1] = sum.y;
                r[e + h] = dif.x;
                r[e + h + 1] = dif.y;
            }
        }
    }
    const float2 hs = make_float2(HadamardScale<D>::value, HadamardScale<D>::value);
    float am0 = 0.f, am1 = 0.f;
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float2 v = __fmul2_rn(make_float2(r[e], r[e + 1]), hs);
        r[e] = v.x;
        r[e + 1] = v.y;
        am0 = fmaxf(am0, fabsf(v.x));
        am1 = fmaxf(am1, fabsf(v.y));
    }
    float amax = fmaxf(am0, am1);
    if constexpr (D == 128) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
    if (ue8m0) s = pow2_ceil(s);
    const float rs = __frcp_rn(s);
    // x / s correctly rounded, two at a time (div_rn_by on each element)
    const float2 rs2 = make_float2(rs, rs), ns2 = make_float2(-s, -s);
    auto div2 = [&](float x0, float x1) {
        const float2 x = make_float2(x0, x1);
        const float2 q0 = __fmul2_rn(x, rs2);
        const float2 er = __ffma2_rn(q0, ns2, x);
        return __ffma2_rn(er, rs2, q0);
    };
#pragma unroll
    for (int j = 0; j < 16; j++) {
        const float2 lo = div2(r[4 * j], r[4 * j + 1]);
        const float2 hi = div2(r[4 * j + 2], r[4 * j + 3]);
        codes[j] = e4m3x2_rn_sat(lo.x, lo.y) | e4m3x2_rn_sat(hi.x, hi.y) << 16;
    }
    *scale = s;
}

// Element of register i of lane part p under the lane split on bit X.
template <int X>
__host__ __device__ constexpr int split_element(int i, int p) {
    return ((i >> X) << (X + 1)) | (p << X) | (i & ((1 << X) - 1));
}

// Loads this lane's E elements of a D-vector (fp32 or bf16).
template <int D, typename T>
__device__ __forceinline__ void load_lane_slice(const T *vec, float (&r)[D / 32]) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const T *src = vec + lane * E;
    if constexpr (E == 4 && sizeof(T) == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(src);
        r[0] = t.x; r[1] = t.y; r[2] = t.z; r[3] = t.w;
    } else if constexpr (E == 2 && sizeof(T) == 4) {
        const float2 t = *reinterpret_cast<const float2 *>(src);
        r[0] = t.x; r[1] = t.y;
    } else {
#pragma unroll
        for (int e = 0; e < E; e++) r[e] = to_f32<T>(src[e]);
    }
}

}  // namespace dsa
