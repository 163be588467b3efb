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
// Prefill scorer: a CTA owns G consecutive causal query rows of one sequence
// (G = 256 / NH rows of NH padded heads: 4 rows of 64 heads) and streams their
// key tiles once.  One key tile (the MMA's A) serves all G rows:
//   warp 0      TMA producer of 128-token key tiles (as the decode scorer);
//   warp 1      TMEM + tcgen05.mma kind::f8f6f4, M = 128 tokens,
//               N = G * NH <= 256, into a double-buffered 2 x 256-column
//               accumulator;
//   warps 2..17 epilogue: warp w reads TMEM lane quarter w % 4 (its tokens)
//               and the 64-column slice (w - 2) / 4 of the accumulator (64 / NH
//               whole rows), writing each row's causally masked score
//               k_scale * sum_h w'_h ReLU(dot_h); the weighted sum uses packed
//               two-lane FMAs.
// Groups are taken longest first (the last group of every sequence first).
// The epilogue is CUDA-core bound at about the rate the FP8 MMA needs: per
// 128-token tile, 128 x 256 (token, head, row) terms of one max and half a
// packed FMA each.
constexpr int kGEpiWarps = 16;
constexpr int kGThreads = 64 + 32 * kGEpiWarps;
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
    return 1024 + (size_t)kStages * kTile * D + (size_t)kGCols * D + kGCols * sizeof(float) +
           (2 * kStages + 2 * kAcc + 1) * sizeof(uint64_t) + 16;
}

template <int D, int NH>
__global__ void __launch_bounds__(kGThreads, 1)
score_group_kernel(const __grid_constant__ CUtensorMap tmap_k, const GroupArgs a) {
    static_assert(NH == 16 || NH == 32 || NH == 64, "whole rows per 64-column slice");
    constexpr int G = kGCols / NH;       // rows per group
    constexpr int RS = 64 / NH;          // rows per epilogue slice
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sk = smem;
    uint8_t *sq = sk + kStages * kTile * D;                  // [256 operand rows][D]
    float *wf = reinterpret_cast<float *>(sq + kGCols * D);  // folded weights per operand row
    uint64_t *full = reinterpret_cast<uint64_t *>(wf + kGCols);
    uint64_t *empty = full + kStages;
    uint64_t *accf = empty + kStages;
    uint64_t *acce = accf + kAcc;
    uint64_t *q_ready = acce + kAcc;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(q_ready + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x % a.B;
    const int64_t s0 = (int64_t)(a.n_groups - 1 - blockIdx.x / a.B) * G;
    const int g_rows = a.S - s0 < G ? (int)(a.S - s0) : G;       // rows of this group
    const int64_t last = a.start_pos + s0 + g_rows - 1;          // its longest row's last key
    const int64_t n_vis = a.T < last + 1 ? a.T : last + 1;
    const int n_tiles = (int)((n_vis + kTile - 1) / kTile);
    constexpr int N = G * NH;

    // every row's scores beyond the group's last key tile are masked
    for (int r = 0; r < g_rows; r++) {
        float *orow = a.scores + (b * a.S + s0 + r) * a.T;
        for (int64_t t = (int64_t)n_tiles * kTile + threadIdx.x; t < a.T; t += kGThreads)
            orow[t] = -INFINITY;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < kAcc; i++) {
            tc::mbar_init(&accf[i], 1);
            tc::mbar_init(&acce[i], kGEpiWarps * 32);
        }
        tc::mbar_init(q_ready, kGEpiWarps * 32);
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
            // every group of the sequence reads these keys: keep them in L2
            const uint64_t pol = tc::l2_evict_last_policy();
            int issued = 0;
            for (int i = 0; i < n_tiles; i++) {
                const int st = i % kStages;
                if (!tc::mbar_wait(&empty[st], ((uint32_t)(i / kStages) & 1u) ^ 1u, a.err, abort)) break;
                tc::mbar_arrive_expect_tx(&full[st], kTile * D);
                tc::tma_load_3d(sk + st * kTile * D, &tmap_k, 0, i * kTile, (int)b, &full[st], pol);
                issued = i + 1;
            }
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; j++)
                tc::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, a.err, abort);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::instr_desc(tc::kFmtE4M3, tc::kFmtE4M3, kTile, N);
            const uint32_t sk_addr = tc::smem_u32(sk), sq_addr = tc::smem_u32(sq);
            const bool q_ok = tc::mbar_wait(q_ready, 0, a.err, abort);
            for (int i = 0; q_ok && i < n_tiles; i++) {
                const int st = i % kStages, ac = i % kAcc;
                if (!tc::mbar_wait(&full[st], (uint32_t)(i / kStages) & 1u, a.err, abort)) break;
                if (!tc::mbar_wait(&acce[ac], ((uint32_t)(i / kAcc) & 1u) ^ 1u, a.err, abort))
                    break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(ac * kGCols);
#pragma unroll
                for (int k = 0; k < D / 32; k++) {
                    const uint64_t ad = tc::smem_desc(sk_addr + st * kTile * D + k * 32,
                                                      KSwizzle<D>::sbo, KSwizzle<D>::kind);
                    const uint64_t bd =
                        tc::smem_desc(sq_addr + k * 32, KSwizzle<D>::sbo, KSwizzle<D>::kind);
                    tc::mma_f8f6f4(d_tmem, ad, bd, idesc, k > 0);
                }
                tc::tc_commit(&empty[st]);
                tc::tc_commit(&accf[ac]);
            }
        }
    } else {
        // query operand: operand row r * NH + h holds row s0 + r, head h (zeros
        // for padded heads and rows past S), K-major and swizzled
        const int t = threadIdx.x - 64;                      // 0 .. 32 * kGEpiWarps - 1
        constexpr int kChunks = D / 16;
        for (int i = t; i < kGCols * kChunks; i += 32 * kGEpiWarps) {
            const int orow = i / kChunks, c = i - orow * kChunks;
            const int r = orow / NH, h = orow - r * NH;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < g_rows && h < a.H)
                v = *reinterpret_cast<const uint4 *>(a.q_fp8 + ((b * a.S + s0 + r) * a.H + h) * D +
                                                     c * 16);
            *reinterpret_cast<uint4 *>(sq + orow * D + KSwizzle<D>::chunk(orow, c) * 16) = v;
        }
        if (t < kGCols) {
            float x = 0.f;
            const int r = t / NH, h = t - r * NH;
            if (r < g_rows && h < a.H) {
                const int64_t qi = (b * a.S + s0 + r) * a.H + h;
                x = __fmul_rn(a.w[qi], a.head_scale);
                x = __fmul_rn(x, a.q_scale[qi]);
                x = __fmul_rn(x, a.softmax_scale);
            }
            wf[t] = x;
        }
        tc::fence_proxy_async_smem();
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kGEpiWarps) : "memory");
        tc::mbar_arrive(q_ready);

        const int quarter = warp & 3, slice = (warp - 2) >> 2;   // tokens, 64 columns
        const int tok = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const float *ks_row = a.k_scale + b * a.t_max;
        auto load_ks = [&](int ii) -> float {
            const int64_t tt = (int64_t)ii * kTile + tok;
            return ii < n_tiles && tt < n_vis ? __ldg(ks_row + tt) : 0.f;
        };
        float ks0 = load_ks(0), ks1 = load_ks(1), ks2 = load_ks(2);
        const float4 *w4 = reinterpret_cast<const float4 *>(wf + slice * 64);
        for (int i = 0; i < n_tiles; i++) {
            const int ac = i % kAcc;
            const int64_t tp = (int64_t)i * kTile + tok;
            const float ks = ks0;
            ks0 = ks1;
            ks1 = ks2;
            ks2 = load_ks(i + 3);
            if (!tc::mbar_wait(&accf[ac], (uint32_t)(i / kAcc) & 1u, a.err, abort)) break;
            tc::tc_fence_after();
            uint32_t v[64];
            const uint32_t taddr = tmem_base + lane_addr + (uint32_t)(ac * kGCols + slice * 64);
#pragma unroll
            for (int j = 0; j < 4; j++)
                tc::tmem_ld16(taddr + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * j));
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(&acce[ac]);          // the values are in registers
#pragma unroll
            for (int rl = 0; rl < RS; rl++) {
                float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
#pragma unroll
                for (int h = 0; h < NH; h += 4) {
                    const float4 wv = w4[(rl * NH + h) / 4];
                    const int e = rl * NH + h;
                    acc01 = __ffma2_rn(make_float2(wv.x, wv.y),
                                       make_float2(fmaxf(__uint_as_float(v[e]), 0.f),
                                                   fmaxf(__uint_as_float(v[e + 1]), 0.f)),
                                       acc01);
                    acc23 = __ffma2_rn(make_float2(wv.z, wv.w),
                                       make_float2(fmaxf(__uint_as_float(v[e + 2]), 0.f),
                                                   fmaxf(__uint_as_float(v[e + 3]), 0.f)),
                                       acc23);
                }
                const int r = slice * RS + rl;
                if (r < g_rows && tp < a.T) {
                    const int64_t srow = s0 + r;
                    const float acc = (acc01.x + acc01.y) + (acc23.x + acc23.y);
                    a.scores[(b * a.S + srow) * a.T + tp] =
                        tp < a.start_pos + srow + 1 ? ks * acc : -INFINITY;
                }
            }
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
    score_group_kernel<D, NH><<<(unsigned)((int64_t)g.B * g.n_groups), kGThreads, smem, stream>>>(
        tmap, g);
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
