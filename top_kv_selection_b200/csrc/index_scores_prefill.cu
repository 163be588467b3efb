// index_scores_prefill.cu -- fp8_index scoring of many causal query rows.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward (the
// weight fold, fp8_index and the causal mask of a prefill chunk), as in
// index_scores.cu; this file holds the grouped kernel used when a call has
// enough query rows to fill the GPU with groups of them.
#include "common.cuh"
#include "quant.cuh"
#include "scorer.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

// ---------------------------------------------------------------------------
// Prefill scorer, persistent: one CTA per SM works through groups of G
// consecutive causal query rows of one sequence (G = 256 / NH rows of NH padded
// heads: 4 rows of 64 heads).  One 128-token key tile (the MMA's A) serves all
// G rows of a group:
//   warp 0      TMA producer of key tiles, one ring across all the CTA's groups;
//   warp 1      TMEM + tcgen05.mma kind::f8f6f4, M = 128 tokens,
//               N = G * NH <= 256, into a double-buffered 2 x 256-column
//               accumulator, the query operand of group k in buffer k & 1;
//   warps 2..17 epilogue: warp w reads TMEM lane quarter w % 4 (its tokens)
//               and the 64-column slice (w - 2) / 4 of the accumulator (64 / NH
//               whole rows), writing each row's causally masked score
//               k_scale * sum_h w'_h ReLU(dot_h) with packed two-lane FMAs.
//               They also fetch the query codes of the group after next with
//               zero-filling cp.async as soon as its buffer's MMAs are done,
//               publish them after the next group's first tile, and write each
//               group's masked tail after its tiles.
// The groups are ordered longest first and dealt to the CTAs in a snake
// (CTA c takes the c-th group of even rounds and the c-th from the end of odd
// rounds), which evens out the total per CTA.
// The epilogue is CUDA-core bound at about the rate the FP8 MMA needs: per
// 128-token tile, 128 x 256 (token, head, row) terms of one max and half a
// packed FMA each.
constexpr int kGEpiWarps = 16;
constexpr int kGEpi = 32 * kGEpiWarps;   // epilogue threads
constexpr int kGThreads = 64 + kGEpi;
constexpr int kGCols = 256;              // accumulator columns per buffer

struct GroupArgs {
    const uint8_t *q_fp8;
    const float *q_scale;
    const float *w;
    const float *k_scale;
    float *scores;
    int64_t t_max, start_pos, T;
    int B, S, H, NH, G, n_groups;
    float head_scale, softmax_scale;
    int *err;
};

template <int D>
__host__ __device__ constexpr size_t group_smem_bytes() {
    return 1024 + (size_t)kStages * kTile * D + 2 * (size_t)kGCols * D + 4 * kGCols * sizeof(float) +
           (2 * kStages + 2 * kAcc + 4) * sizeof(uint64_t) + 16;
}

// One group: sequence b, rows s0 .. s0 + g_rows - 1, key tiles 0 .. n_tiles - 1.
struct Group {
    int64_t b, s0, n_vis;
    int g_rows, n_tiles;
};

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tc::smem_u32(dst)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async4_zfill(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(tc::smem_u32(dst)),
                 "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}

template <int D, int NH>
__global__ void __launch_bounds__(kGThreads, 1)
score_group_kernel(const __grid_constant__ CUtensorMap tmap_k, const GroupArgs a) {
    static_assert(NH == 16 || NH == 32 || NH == 64, "whole rows per 64-column slice");
    constexpr int G = kGCols / NH;       // rows per group
    constexpr int RS = 64 / NH;          // rows per epilogue slice
    constexpr int N = G * NH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sk = smem;
    uint8_t *sq = sk + kStages * kTile * D;                      // [2][256 operand rows][D]
    float *wf = reinterpret_cast<float *>(sq + 2 * kGCols * D);  // [2][256] folded weights
    float *w_in = wf + 2 * kGCols;                               // [256] weights and query
    float *qs_in = w_in + kGCols;                                // [256] scales being fetched
    uint64_t *full = reinterpret_cast<uint64_t *>(qs_in + kGCols);
    uint64_t *empty = full + kStages;
    uint64_t *accf = empty + kStages;
    uint64_t *acce = accf + kAcc;
    uint64_t *q_full = acce + kAcc;      // [2] query buffer published
    uint64_t *q_empty = q_full + 2;      // [2] the MMAs reading it are done
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(q_empty + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = a.B * a.n_groups;
    // the k-th group of this CTA (snake over the longest-first order), or -1
    auto group_index = [&](int k) -> int {
        const int P = (int)gridDim.x, c = (int)blockIdx.x;
        const int64_t gi = (int64_t)k * P + ((k & 1) ? P - 1 - c : c);
        return gi < total ? (int)gi : -1;
    };
    auto describe = [&](int gi) -> Group {
        Group g;
        g.b = gi % a.B;
        g.s0 = (int64_t)(a.n_groups - 1 - gi / a.B) * G;
        g.g_rows = a.S - g.s0 < G ? (int)(a.S - g.s0) : G;
        const int64_t last = a.start_pos + g.s0 + g.g_rows - 1;   // longest row's last key
        g.n_vis = a.T < last + 1 ? a.T : last + 1;
        g.n_tiles = (int)((g.n_vis + kTile - 1) / kTile);
        return g;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < kAcc; i++) {
            tc::mbar_init(&accf[i], 1);
            tc::mbar_init(&acce[i], kGEpi);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&q_full[i], kGEpi);
            tc::mbar_init(&q_empty[i], 1);
        }
        *abort = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap_k);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_holder, kAcc * kGCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            // every group of a sequence reads these keys: keep them in L2
            const uint64_t pol = tc::l2_evict_last_policy();
            int it = 0;
            bool ok = true;
            for (int k = 0; ok; k++) {
                const int gi = group_index(k);
                if (gi < 0) break;
                const Group g = describe(gi);
                for (int i = 0; i < g.n_tiles; i++, it++) {
                    const int st = it % kStages;
                    if (!tc::mbar_wait(&empty[st], ((uint32_t)(it / kStages) & 1u) ^ 1u, a.err, abort)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[st], kTile * D);
                    tc::tma_load_3d(sk + st * kTile * D, &tmap_k, 0, i * kTile, (int)g.b, &full[st], pol);
                }
            }
            // wait (bounded) for the last loads still landing in shared memory
            for (int j = it > kStages ? it - kStages : 0; j < it; j++)
                tc::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, a.err, abort);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::instr_desc(tc::kFmtE4M3, tc::kFmtE4M3, kTile, N);
            const uint32_t sk_addr = tc::smem_u32(sk), sq_addr = tc::smem_u32(sq);
            int it = 0;
            bool ok = true;
            for (int k = 0; ok; k++) {
                const int gi = group_index(k);
                if (gi < 0) break;
                const Group g = describe(gi);
                const int qb = k & 1;
                if (!tc::mbar_wait(&q_full[qb], (uint32_t)(k >> 1) & 1u, a.err, abort)) break;
                for (int i = 0; i < g.n_tiles; i++, it++) {
                    const int st = it % kStages, ac = it % kAcc;
                    if (!tc::mbar_wait(&full[st], (uint32_t)(it / kStages) & 1u, a.err, abort) ||
                        !tc::mbar_wait(&acce[ac], ((uint32_t)(it / kAcc) & 1u) ^ 1u, a.err, abort)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(ac * kGCols);
#pragma unroll
                    for (int kk = 0; kk < D / 32; kk++) {
                        const uint64_t ad = tc::smem_desc(sk_addr + st * kTile * D + kk * 32,
                                                          KSwizzle<D>::sbo, KSwizzle<D>::kind);
                        const uint64_t bd = tc::smem_desc(sq_addr + qb * kGCols * D + kk * 32,
                                                          KSwizzle<D>::sbo, KSwizzle<D>::kind);
                        tc::mma_f8f6f4(d_tmem, ad, bd, idesc, kk > 0);
                    }
                    tc::tc_commit(&empty[st]);
                    tc::tc_commit(&accf[ac]);
                }
                tc::tc_commit(&q_empty[qb]);   // this group's operand buffer may be refilled
            }
        }
    } else {
        const int t = threadIdx.x - 64;                      // 0 .. kGEpi - 1
        constexpr int kChunks = D / 16;
        // query codes of group k into operand buffer k & 1 (operand row r * NH + h
        // = row s0 + r, head h; zeros for padded heads and rows past S), once the
        // MMAs of group k - 2 no longer read it; its weights and query scales into
        // w_in / qs_in (thread t fetches entry t and later folds it)
        auto prepare = [&](int k) {
            const int gi = group_index(k);
            if (gi < 0) return;
            const Group g = describe(gi);
            const int qb = k & 1;
            if (k >= 2) tc::mbar_wait(&q_empty[qb], (uint32_t)((k - 2) >> 1) & 1u, a.err, abort);
            uint8_t *dstq = sq + qb * kGCols * D;
            for (int i = t; i < kGCols * kChunks; i += kGEpi) {
                const int orow = i / kChunks, c = i - orow * kChunks;
                const int r = orow / NH, h = orow - r * NH;
                const bool valid = r < g.g_rows && h < a.H;
                const uint8_t *src =
                    valid ? a.q_fp8 + ((g.b * a.S + g.s0 + r) * a.H + h) * D + c * 16 : a.q_fp8;
                cp_async16_zfill(dstq + orow * D + KSwizzle<D>::chunk(orow, c) * 16, src, valid);
            }
            if (t < kGCols) {
                const int r = t / NH, h = t - r * NH;
                const bool valid = r < g.g_rows && h < a.H;
                const int64_t qi = valid ? (g.b * a.S + g.s0 + r) * a.H + h : 0;
                cp_async4_zfill(w_in + t, a.w + qi, valid);
                cp_async4_zfill(qs_in + t, a.q_scale + qi, valid);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        // completes group k's operand copy (the only one in flight), writes its
        // folded weights w' = ((w * H^-1/2) * q_scale) * softmax_scale and
        // publishes the buffer to the MMA warp
        auto finish = [&](int k) {
            if (group_index(k) < 0) return;
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            if (t < kGCols) {                        // zero-filled entries fold to 0
                float x = __fmul_rn(w_in[t], a.head_scale);
                x = __fmul_rn(x, qs_in[t]);
                wf[(k & 1) * kGCols + t] = __fmul_rn(x, a.softmax_scale);
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&q_full[k & 1]);
        };

        prepare(0);
        finish(0);
        prepare(1);
        asm volatile("bar.sync 1, %0;" ::"n"(kGEpi) : "memory");   // group 0's weights

        const int quarter = warp & 3, slice = (warp - 2) >> 2;      // tokens, 64 columns
        const int tok = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int it = 0;
        bool ok = true;
        for (int k = 0;; k++) {
            const int gi = group_index(k);
            if (gi < 0) break;
            const Group g = describe(gi);
            // per-tile bookkeeping in 32-bit offsets from this thread's token:
            // tile i covers this thread's position i * kTile + tok
            const float *ks_tok = a.k_scale + g.b * a.t_max + tok;
            const int nv_rel = (int)(g.n_vis - tok);        // positions with keys: off < nv_rel
            const int t_rel = (int)(a.T - tok);             // positions that exist: off < t_rel
            float *orow[RS];                                // this thread's rows (null: padding)
            int vis_rel[RS];                                // causal: off < vis_rel
#pragma unroll
            for (int rl = 0; rl < RS; rl++) {
                const int r = slice * RS + rl;
                orow[rl] = r < g.g_rows ? a.scores + (g.b * a.S + g.s0 + r) * a.T + tok : nullptr;
                vis_rel[rl] = (int)(a.start_pos + g.s0 + r + 1 - tok);
            }
            auto load_ks = [&](int ii) -> float {
                return ii * kTile < nv_rel ? __ldg(ks_tok + ii * kTile) : 0.f;
            };
            float ks0 = load_ks(0), ks1 = load_ks(1), ks2 = load_ks(2);
            const float4 *w4 = reinterpret_cast<const float4 *>(wf + (k & 1) * kGCols + slice * 64);
            for (int i = 0; i < g.n_tiles; i++, it++) {
                const int ac = it % kAcc;
                const int off = i * kTile;
                const float ks = ks0;
                ks0 = ks1;
                ks1 = ks2;
                ks2 = load_ks(i + 3);
                if (ok && !tc::mbar_wait(&accf[ac], (uint32_t)(it / kAcc) & 1u, a.err, abort)) ok = false;
                if (ok) {
                    tc::tc_fence_after();
                    const uint32_t taddr =
                        tmem_base + lane_addr + (uint32_t)(ac * kGCols + slice * 64);
                    // the slice's 64 columns in two halves of 32 (registers); the
                    // accumulator is released once the second half is loaded
                    float2 acc01[RS], acc23[RS];
#pragma unroll
                    for (int rl = 0; rl < RS; rl++) {
                        acc01[rl] = make_float2(0.f, 0.f);
                        acc23[rl] = make_float2(0.f, 0.f);
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; hh++) {
                        uint32_t v[32];
                        tc::tmem_ld16(taddr + 32 * hh, *reinterpret_cast<uint32_t(*)[16]>(v));
                        tc::tmem_ld16(taddr + 32 * hh + 16, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
                        tc::tmem_wait_ld();
                        if (hh == 1) {
                            tc::tc_fence_before();
                            tc::mbar_arrive(&acce[ac]);
                        }
#pragma unroll
                        for (int q4 = 0; q4 < 8; q4++) {
                            const int e = 32 * hh + 4 * q4;       // column within the slice
                            const int rl = e / NH;                // row within the slice
                            const float4 wv = w4[e / 4];
                            acc01[rl] = __ffma2_rn(make_float2(wv.x, wv.y),
                                                   make_float2(fmaxf(__uint_as_float(v[4 * q4]), 0.f),
                                                               fmaxf(__uint_as_float(v[4 * q4 + 1]), 0.f)),
                                                   acc01[rl]);
                            acc23[rl] = __ffma2_rn(make_float2(wv.z, wv.w),
                                                   make_float2(fmaxf(__uint_as_float(v[4 * q4 + 2]), 0.f),
                                                               fmaxf(__uint_as_float(v[4 * q4 + 3]), 0.f)),
                                                   acc23[rl]);
                        }
                    }
#pragma unroll
                    for (int rl = 0; rl < RS; rl++) {
                        if (orow[rl] != nullptr && off < t_rel) {
                            const float acc = (acc01[rl].x + acc01[rl].y) + (acc23[rl].x + acc23[rl].y);
                            orow[rl][off] = off < vis_rel[rl] ? ks * acc : -INFINITY;
                        }
                    }
                }
                if (i == 0) finish(k + 1);           // before this group's MMAs run out
            }
            // the rows' positions beyond the group's last key tile are masked
            for (int r = 0; r < g.g_rows; r++) {
                float *orow = a.scores + (g.b * a.S + g.s0 + r) * a.T;
                for (int64_t tt = (int64_t)g.n_tiles * kTile + t; tt < a.T; tt += kGEpi)
                    orow[tt] = -INFINITY;
            }
            // every epilogue thread is done with group k's weights and TMEM reads
            asm volatile("bar.sync 1, %0;" ::"n"(kGEpi) : "memory");
            prepare(k + 2);
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kAcc * kGCols);
    }
}

template <int D, int NH>
dsa_status launch_group(GroupArgs g, const uint8_t *k_cache, cudaStream_t stream) {
    CUtensorMap tmap;
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)g.t_max, (uint64_t)g.B};
    const uint64_t strides[2] = {(uint64_t)D, (uint64_t)g.t_max * D};
    const uint32_t box[3] = {(uint32_t)D, (uint32_t)kTile, 1};
    const CUtensorMapSwizzle swz =
        D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    if (!encode_tmap(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k_cache, dims, strides, box, swz))
        return DSA_ERR_CUDA;
    const size_t smem = group_smem_bytes<D>();
    if (cudaFuncSetAttribute(score_group_kernel<D, NH>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DSA_ERR_CUDA;
    // persistent: one CTA per SM (or per group, if fewer)
    const int64_t total = (int64_t)g.B * g.n_groups;
    const int grid = total < num_sms() ? (int)total : num_sms();
    score_group_kernel<D, NH><<<(unsigned)grid, kGThreads, smem, stream>>>(tmap, g);
    return launch_status();
}

}  // namespace

// Rows per group of the prefill scorer for H heads, or 0 when one query row
// per CTA with the key range split across CTAs is the plan (too few groups to
// fill the SMs, or padded heads other than 16, 32 or 64).
int prefill_group_rows(int B, int S, int H) {
    const int NH = (H + 15) / 16 * 16;
    if (NH != 16 && NH != 32 && NH != 64) return 0;
    const int G = kGCols / NH;
    const int64_t groups = (int64_t)B * ((S + G - 1) / G);
    return groups >= num_sms() ? G : 0;
}


dsa_status launch_prefill_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                                 const uint8_t *k_cache, const float *k_scale, int64_t t_max,
                                 int B, int S, int H, int D, int64_t start_pos, int64_t T,
                                 float softmax_scale, float *scores, cudaStream_t stream) {
    GroupArgs g = {};
    g.q_fp8 = q_fp8;
    g.q_scale = q_scale;
    g.w = w;
    g.k_scale = k_scale;
    g.scores = scores;
    g.t_max = t_max;
    g.start_pos = start_pos;
    g.T = T;
    g.B = B;
    g.S = S;
    g.H = H;
    g.NH = (H + 15) / 16 * 16;
    g.G = prefill_group_rows(B, S, H);
    g.n_groups = (S + g.G - 1) / g.G;
    g.head_scale = (float)(1.0 / sqrt((double)H));
    g.softmax_scale = softmax_scale;
    g.err = device_error_word();
    switch (g.NH * 1000 + D) {
        case 16128: return launch_group<128, 16>(g, k_cache, stream);
        case 32128: return launch_group<128, 32>(g, k_cache, stream);
        case 64128: return launch_group<128, 64>(g, k_cache, stream);
        case 16064: return launch_group<64, 16>(g, k_cache, stream);
        case 32064: return launch_group<64, 32>(g, k_cache, stream);
        default: return launch_group<64, 64>(g, k_cache, stream);
    }
}

}  // namespace dsa
