// scorer.cuh -- tile shape and shared-memory operand layout common to the
// indexer scorers (decode: index_scores.cu, grouped prefill:
// index_scores_prefill.cu).
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace dsa {

constexpr int kTile = 128;       // tokens per key tile = MMA M
constexpr int kStages = 6;       // key-tile ring depth
constexpr int kAcc = 2;          // TMEM accumulator buffers

// K-major FP8 operand rows of D bytes: 128-byte rows swizzled in 16-byte
// chunks (D = 128) or 64-byte rows (D = 64), matching the key tensor map.
template <int D> struct KSwizzle;
template <> struct KSwizzle<128> {
    static constexpr tc::Swizzle kind = tc::kSwizzle128B;
    static constexpr uint32_t sbo = 1024;    // 8 rows x 128 B
    __device__ static int chunk(int row, int c) { return c ^ (row & 7); }
};
template <> struct KSwizzle<64> {
    static constexpr tc::Swizzle kind = tc::kSwizzle64B;
    static constexpr uint32_t sbo = 512;     // 8 rows x 64 B
    __device__ static int chunk(int row, int c) { return c ^ ((row >> 1) & 3); }
};

// Grouped prefill scorer (index_scores_prefill.cu): rows per group, or 0 when
// the one-row-per-CTA scorer is the plan.
int prefill_group_rows(int B, int S, int H);
dsa_status launch_prefill_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                                 const uint8_t *k_cache, const float *k_scale, int64_t t_max,
                                 int B, int S, int H, int D, int64_t start_pos, int64_t T,
                                 float softmax_scale, float *scores, cudaStream_t stream);

}  // namespace dsa
