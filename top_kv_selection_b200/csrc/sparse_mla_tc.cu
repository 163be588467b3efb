// sparse_mla_tc.cu -- tensor-core sparse latent attention (bf16, V3.2 shapes).
//
// Pages: the diagram "DeepSeek Sparse Attention, one decode step in one layer
// (V3.2 sizes)" (core attention in MQA mode: 128 heads over the gathered
// 576-wide latent rows, each row key and value) and the MLA prefill excerpt
// of "DeepSeek-V3.2-Exp - Causal mask" (index mask + causal mask, softmax,
// value mix).
//
// Shapes: Hq = 128 heads (the MMA M), rows [c (512) | k_pe (64)] bf16.
// One CTA computes, for one query row, one 256-wide half of the output over
// one share ("split") of the selected rows:
//   warps 5..8  gather 32 selected rows per tile into a 2-stage ring with
//               16-byte cp.async, straight into the 128B-swizzled K-major
//               layout (nine 64-column blocks of 32 rows x 128 B); each warp
//               copies 8 rows, consecutive lanes consecutive 16-byte pieces;
//               a tile is published (wait, proxy fence, arrive) two tiles
//               later, or at once before the producer would block;
//   warp 0      S = Q C^T: 36 tcgen05.mma kind::f16 (M=128, N=32, K=16) per
//               tile with both operands in shared memory (the whole query,
//               144 KB, is loaded once by TMA); O += P C[:, half]: 2 MMAs
//               (N=256, K=16) with A = P from TMEM and B = the same shared
//               tile read as an MN-major operand (no transpose copy).  The
//               previous tile's PV is slotted between this tile's QK column
//               blocks as soon as its P is ready, so its stage is freed early;
//   warps 1..4  one thread per head: online softmax in the exp2 domain with
//               lazy rescaling (the fp32 accumulator in TMEM is rescaled only
//               when a head's running max grows by more than 8), P written to
//               TMEM as bf16, then the epilogue.
// TMEM: O 256 | S 2 x 32 | P 2 x 16 columns.  The logits are computed by both
// halves of a row (the output accumulator alone fills half of TMEM and the
// query fills most of shared memory), so each gathered row is read twice from
// L2 but once from HBM.
// With several splits per row, unnormalised partial outputs and (max, sum)
// pairs go to the workspace and a combine kernel merges them.
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

constexpr int kHq = 128, kDc = 512, kDr = 64, kDqk = kDc + kDr;
constexpr int kNB = kDqk / 64;                  // 64-column blocks per row: 9
constexpr int kDh = 256;                        // output columns per CTA
constexpr int kRows = 32;                       // gathered rows per tile
constexpr int kStages = 2;
constexpr int kThreads = 288;               // warp 0 MMA, 1..4 softmax, 5..8 gather
constexpr int kMaxSel = 2048;                   // selection slots held in shared memory
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kTmemCols = 512;
constexpr int kBlk = kRows * 128;               // bytes of one column block of a tile
constexpr int kTileBytes = kNB * kBlk;          // 36864
constexpr int kQBlk = kHq * 128;                // 16384
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kTileBytes + (size_t)kNB * kQBlk +
                              kMaxSel * sizeof(int32_t) + 32 * sizeof(uint64_t) + 64;
constexpr int kLag = 2;                          // gather tiles in flight per thread beyond the one issued

struct MlaArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *kv;
    const int32_t *idx;
    __nv_bfloat16 *out;
    float *lse;
    float *part_o;      // [units][128][256]  (splits > 1)
    float2 *part_ml;    // [units][128]
    int64_t t_max;
    int64_t start_pos;
    int S, k, splits;
    float scale_log2;   // sm_scale * log2(e)
    int *err;
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ int block_scan_flag_all(bool flag, int *warp_tot, int *total) {
    constexpr int kW = kThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned ballot = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int w = 0; w < kW; w++) {
            const int v = warp_tot[w];
            warp_tot[w] = acc;
            acc += v;
        }
        warp_tot[kW] = acc;
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    *total = warp_tot[kW];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sc = smem;                                      // C tiles
    uint8_t *sq = sc + kStages * kTileBytes;                 // Q, nine 64-column blocks
    int32_t *list = reinterpret_cast<int32_t *>(sq + kNB * kQBlk);
    uint64_t *bars = reinterpret_cast<uint64_t *>(list + kMaxSel);
    uint64_t *c_full = bars, *c_empty = bars + kStages;
    uint64_t *s_full = bars + 2 * kStages, *s_empty = s_full + 2;
    uint64_t *p_full = s_empty + 2, *pv_done = p_full + 2;
    uint64_t *q_full = pv_done + 2, *q_ready = q_full + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(q_ready + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *scan_tmp = const_cast<int *>(abort) + 1;            // 10 ints

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;                             // (row * 2 + half) * splits + sp
    const int sp = unit % a.splits;
    const int half = (unit / a.splits) & 1;
    const int64_t row = unit / (a.splits * 2);
    const int64_t b = row / a.S, s = row - b * a.S;
    const int64_t limit = a.start_pos + s;
    const bool is_softmax = warp >= 1 && warp <= 4;
    const int quarter = warp & 3;                            // softmax warps: TMEM lane quarter
    const int h = quarter * 32 + lane;                       // softmax warps: head
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            tc::mbar_init(&c_full[i], 128);
            tc::mbar_init(&c_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&s_empty[i], 128);
            tc::mbar_init(&p_full[i], 128);
            tc::mbar_init(&pv_done[i], 1);
        }
        tc::mbar_init(q_full, 1);
        *abort = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tm_q);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_holder, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // the query does not depend on the preceding kernel: load it first
    if (threadIdx.x == 160) {
        tc::mbar_arrive_expect_tx(q_full, kNB * kQBlk);
        for (int j = 0; j < kNB; j++)
            tc::tma_load_2d(sq + j * kQBlk, &tm_q, j * 64, (int)(row * kHq), q_full);
    }

    // valid selections of this row, in slot order
    constexpr int kPer = (kMaxSel + kThreads - 1) / kThreads;
    int32_t slot[kPer];
#pragma unroll
    for (int r = 0; r < kPer; r++) {
        const int j = r * kThreads + threadIdx.x;
        slot[r] = j < a.k ? __ldg(a.idx + row * a.k + j) : -1;
    }
    int n = 0;
#pragma unroll
    for (int r = 0; r < kPer; r++) {
        if (r * kThreads >= a.k) break;
        const int32_t t = slot[r];
        const bool v = t >= 0 && (int64_t)t <= limit && (int64_t)t < a.t_max;
        if (t >= 0 && (int64_t)t <= limit && (int64_t)t >= a.t_max) record_error(a.err, DSA_ERR_DEVICE);
        int tot;
        const int pos = block_scan_flag_all(v, scan_tmp, &tot);
        if (v) list[n + pos] = t;
        n += tot;
    }
    const int lo = (int)((int64_t)sp * n / a.splits);
    const int n_my = (int)((int64_t)(sp + 1) * n / a.splits) - lo;
    const int n_tiles = (n_my + kRows - 1) / kRows;

    if (n_tiles == 0) {                                      // nothing selected here
        if (threadIdx.x == 160) tc::mbar_wait(q_full, 0, a.err, abort);   // Q copy landed
        if (is_softmax) {
            if (a.splits > 1) {
                float4 *po = reinterpret_cast<float4 *>(a.part_o + ((int64_t)unit * kHq + h) * kDh);
                for (int c = 0; c < kDh / 4; c++) po[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                a.part_ml[(int64_t)unit * kHq + h] = make_float2(-INFINITY, 0.f);
            } else {
                __nv_bfloat16 *o = a.out + (row * kHq + h) * kDc + half * kDh;
                for (int c = 0; c < kDh; c++) o[c] = __float2bfloat16_rn(0.f);
                if (half == 0 && a.lse) a.lse[row * kHq + h] = -INFINITY;
            }
        }
    } else if (warp >= 5) {
        // ---- gather: warp w copies rows 8w..8w+7 of each tile; lane l copies
        // the 16-byte pieces l, l+32, l+64 (< 72) of each row
        const int pw = warp - 5;
        const int64_t rbase = b * a.t_max;
        int issued = 0, signalled = 0;
        for (int i = 0; i < n_tiles; i++) {
            const int st = i % kStages;
            const uint32_t ph = ((uint32_t)(i / kStages) & 1u) ^ 1u;
            if (!tc::mbar_test_wait(&c_empty[st], ph)) {
                // about to block: first publish every tile issued so far, since
                // the stage we wait for is freed only after they are consumed
                cp_async_wait<0>();
                tc::fence_proxy_async_smem();
                for (; signalled < issued; signalled++) tc::mbar_arrive(&c_full[signalled % kStages]);
                if (!tc::mbar_wait(&c_empty[st], ph, a.err, abort)) break;
            }
            uint8_t *tile = sc + st * kTileBytes;
#pragma unroll 1
            for (int jj = 0; jj < 8; jj++) {
                const int j = pw * 8 + jj;
                int r = i * kRows + j;
                if (r >= n_my) r = n_my - 1;                 // padding: a valid row
                const __nv_bfloat16 *src = a.kv + (rbase + list[lo + r]) * kDqk;
#pragma unroll
                for (int u = 0; u < 3; u++) {
                    const int c = lane + 32 * u;
                    if (c < 72)
                        cp_async16(tile + (c >> 3) * kBlk + j * 128 + (((c & 7) ^ (j & 7)) << 4),
                                   src + c * 8);
                }
            }
            cp_async_commit();
            issued = i + 1;
            if (issued - signalled > kLag) {
                cp_async_wait<kLag>();
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&c_full[signalled % kStages]);
                signalled++;
            }
        }
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        for (; signalled < issued; signalled++) tc::mbar_arrive(&c_full[signalled % kStages]);
    } else if (warp == 0) {
        if (lane == 0) {
            const uint32_t id_qk = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, kRows);
            const uint32_t id_pv = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, kDh, true);
            const uint32_t sc_addr = tc::smem_u32(sc), sq_addr = tc::smem_u32(sq);
            bool ok = tc::mbar_wait(q_full, 0, a.err, abort);
            // O += P C[:, half] for tile j (P(j) must be published)
            auto pv_issue = [&](int j) {
                const int st = j % kStages, pb = j & 1;
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kRows / 16; ks++) {
                    const uint64_t bd = tc::smem_desc(
                        sc_addr + st * kTileBytes + half * (kDh / 64) * kBlk + ks * 2048, 1024,
                        tc::kSwizzle128B, kBlk);
                    tc::mma_f16_ts(tmem + kColO, tmem + kColP + pb * 16 + ks * 8, bd, id_pv,
                                   j > 0 || ks > 0);
                }
                tc::tc_commit(&c_empty[st]);
                tc::tc_commit(&pv_done[pb]);
            };
            // S = Q C^T for tile i, one 64-column block at a time; the PV of the
            // previous tile (pend >= 0) is slotted in as soon as its P is
            // published, so its stage is released without waiting for all of
            // this tile's MMAs
            auto qk = [&](int i, int pend) -> bool {
                const int st = i % kStages, sb = i & 1;
                if (!tc::mbar_wait(&c_full[st], (uint32_t)(i / kStages) & 1u, a.err, abort)) return false;
                if (!tc::mbar_wait(&s_empty[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u, a.err, abort)) return false;
                tc::tc_fence_after();
                const uint32_t d = tmem + kColS + sb * kRows;
#pragma unroll 1
                for (int cb = 0; cb < kNB; cb++) {
                    if (pend >= 0 && tc::mbar_test_wait(&p_full[pend & 1], (uint32_t)(pend >> 1) & 1u)) {
                        pv_issue(pend);
                        pend = -1;
                    }
#pragma unroll
                    for (int ks = 0; ks < 4; ks++) {
                        const uint64_t ad = tc::smem_desc(sq_addr + cb * kQBlk + ks * 32, 1024, tc::kSwizzle128B);
                        const uint64_t bd = tc::smem_desc(sc_addr + st * kTileBytes + cb * kBlk + ks * 32,
                                                          1024, tc::kSwizzle128B);
                        tc::mma_f16(d, ad, bd, id_qk, (cb | ks) != 0);
                    }
                }
                tc::tc_commit(&s_full[sb]);
                if (pend >= 0) {
                    if (!tc::mbar_wait(&p_full[pend & 1], (uint32_t)(pend >> 1) & 1u, a.err, abort)) return false;
                    pv_issue(pend);
                }
                return true;
            };
            if (ok) ok = qk(0, -1);
            for (int i = 1; ok && i < n_tiles; i++) ok = qk(i, i - 1);
            if (ok && tc::mbar_wait(&p_full[(n_tiles - 1) & 1], (uint32_t)((n_tiles - 1) >> 1) & 1u, a.err, abort))
                pv_issue(n_tiles - 1);
        }
    } else {
        // ---- softmax warps
        float m_run = -INFINITY, l = 0.f;
        bool ok = true;
        for (int i = 0; i < n_tiles && ok; i++) {
            const int sb = i & 1;
            if (!tc::mbar_wait(&s_full[sb], (uint32_t)(i >> 1) & 1u, a.err, abort)) { ok = false; break; }
            tc::tc_fence_after();
            uint32_t r0[16], r1[16];
            tc::tmem_ld16(tmem + lane_addr + kColS + sb * kRows, r0);
            tc::tmem_ld16(tmem + lane_addr + kColS + sb * kRows + 16, r1);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(&s_empty[sb]);
            const int nv = n_my - i * kRows;
            float sv[kRows];
            float m_tile = -INFINITY;
#pragma unroll
            for (int j = 0; j < kRows; j++) {
                const uint32_t bits = j < 16 ? r0[j] : r1[j - 16];
                sv[j] = j < nv ? __uint_as_float(bits) * a.scale_log2 : -INFINITY;
                m_tile = fmaxf(m_tile, sv[j]);
            }
            if (__any_sync(0xffffffffu, m_tile > m_run + 8.f)) {
                const float m_new = fmaxf(m_run, m_tile);
                const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
                if (i > 0) {
                    if (!tc::mbar_wait(&pv_done[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, a.err, abort)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < kDh; c0 += 16) {
                        uint32_t o[16];
                        tc::tmem_ld16(tmem + lane_addr + kColO + c0, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; e++) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tc::tmem_st16(tmem + lane_addr + kColO + c0, o);
                    }
                    tc::tmem_wait_st();
                }
                l *= alpha;
                m_run = m_new;
            }
            if (i >= 2 && !tc::mbar_wait(&pv_done[i & 1], (uint32_t)((i - 2) >> 1) & 1u, a.err, abort)) {
                ok = false;
                break;
            }
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; c++) {
                const float p0 = exp2f(sv[2 * c] - m_run), p1 = exp2f(sv[2 * c + 1] - m_run);
                l += p0 + p1;
                const __nv_bfloat162 v = __floats2bfloat162_rn(p0, p1);
                pk[c] = *reinterpret_cast<const uint32_t *>(&v);
            }
            tc::tmem_st16(tmem + lane_addr + kColP + (i & 1) * 16, pk);
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&p_full[i & 1]);
        }
        if (ok && tc::mbar_wait(&pv_done[(n_tiles - 1) & 1], (uint32_t)((n_tiles - 1) >> 1) & 1u,
                                a.err, abort)) {
            tc::tc_fence_after();
            if (a.splits > 1) {
                float4 *po = reinterpret_cast<float4 *>(a.part_o + ((int64_t)unit * kHq + h) * kDh);
#pragma unroll 1
                for (int c0 = 0; c0 < kDh; c0 += 16) {
                    uint32_t o[16];
                    tc::tmem_ld16(tmem + lane_addr + kColO + c0, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; v++)
                        po[c0 / 4 + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                     __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                }
                a.part_ml[(int64_t)unit * kHq + h] = make_float2(m_run, l);
            } else {
                const float inv = l > 0.f ? 1.f / l : 0.f;
                uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + half * kDh);
#pragma unroll 1
                for (int c0 = 0; c0 < kDh; c0 += 16) {
                    uint32_t o[16], w[8];
                    tc::tmem_ld16(tmem + lane_addr + kColO + c0, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                                       __uint_as_float(o[2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    o16[c0 / 8] = make_uint4(w[0], w[1], w[2], w[3]);
                    o16[c0 / 8 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
                if (half == 0 && a.lse) a.lse[row * kHq + h] = l > 0.f ? (m_run + log2f(l)) * kLn2 : -INFINITY;
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// Merges the splits of each (row, half): out = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s.
// One warp per head; lane l covers output columns 8l..8l+7 (coalesced rows).
constexpr int kCombineHeads = 8;
__global__ void __launch_bounds__(32 * kCombineHeads)
sparse_mla_combine_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml,
                          int splits, __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    const int groups = kHq / kCombineHeads;
    const int64_t rh = blockIdx.x / groups;                 // row * 2 + half
    const int64_t row = rh >> 1;
    const int half = (int)(rh & 1);
    const int h = (int)(blockIdx.x % groups) * kCombineHeads + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t u0 = rh * splits;
    // all (max, sum) pairs first, then the partial rows four splits at a time,
    // so that the loads of a batch are in flight together
    float m = -INFINITY;
    for (int sp = 0; sp < splits; sp++) m = fmaxf(m, part_ml[(u0 + sp) * kHq + h].x);
    float L = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int sp0 = 0; sp0 < splits; sp0 += 4) {
        float2 ml[4];
        float4 x[4], y[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int sp = sp0 + u;
            ml[u] = sp < splits ? part_ml[(u0 + sp) * kHq + h] : make_float2(-INFINITY, 0.f);
            if (sp < splits) {
                const float4 *po =
                    reinterpret_cast<const float4 *>(part_o + ((u0 + sp) * kHq + h) * kDh) + 2 * lane;
                x[u] = po[0];
                y[u] = po[1];
            }
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
            if (ml[u].x == -INFINITY) continue;
            const float w = exp2f(ml[u].x - m);
            L += w * ml[u].y;
            acc[0] += w * x[u].x; acc[1] += w * x[u].y; acc[2] += w * x[u].z; acc[3] += w * x[u].w;
            acc[4] += w * y[u].x; acc[5] += w * y[u].y; acc[6] += w * y[u].z; acc[7] += w * y[u].w;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint32_t wv[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        wv[e] = *reinterpret_cast<const uint32_t *>(&v);
    }
    reinterpret_cast<uint4 *>(out + (row * kHq + h) * kDc + half * kDh)[lane] =
        make_uint4(wv[0], wv[1], wv[2], wv[3]);
    if (half == 0 && lse && lane == 0) lse[row * kHq + h] = L > 0.f ? (m + log2f(L)) * kLn2 : -INFINITY;
}

int mla_splits(int64_t rows, int k) {
    const int64_t units = rows * 2;
    int64_t sp = num_sms() / units;
    const int64_t max_sp = (k + kRows - 1) / kRows;
    if (sp > max_sp) sp = max_sp;
    if (sp < 1) sp = 1;
    return (int)sp;
}

}  // namespace

bool sparse_mla_tc_supported(int Hq, int dc, int dr, int k, dsa_dtype dt) {
    return dt == DSA_BF16 && Hq == kHq && dc == kDc && dr == kDr && k <= kMaxSel;
}

size_t sparse_mla_tc_workspace_bytes(int B, int S, int k) {
    const int64_t rows = (int64_t)B * S;
    const int sp = mla_splits(rows, k);
    if (sp <= 1) return 0;
    const int64_t units = rows * 2 * sp;
    return align_up((size_t)units * kHq * kDh * sizeof(float), 256) +
           (size_t)units * kHq * sizeof(float2);
}

dsa_status launch_sparse_mla_tc(const void *q, const void *kv, int64_t t_max, const int32_t *idx,
                                int B, int S, int k, int64_t start_pos, float sm_scale, void *out,
                                float *lse, void *ws, cudaStream_t stream) {
    const int64_t rows = (int64_t)B * S;
    CUtensorMap tm_q;
    {
        const uint64_t dims[2] = {(uint64_t)kDqk, (uint64_t)(rows * kHq)};
        const uint64_t strides[1] = {(uint64_t)kDqk * 2};
        const uint32_t box[2] = {64, 128};
        if (!encode_tmap(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
            return DSA_ERR_CUDA;
    }
    MlaArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.kv = static_cast<const __nv_bfloat16 *>(kv);
    a.idx = idx;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.t_max = t_max;
    a.start_pos = start_pos;
    a.S = S;
    a.k = k;
    a.splits = mla_splits(rows, k);
    a.scale_log2 = sm_scale * kLog2e;
    a.err = device_error_word();
    a.part_o = nullptr;
    a.part_ml = nullptr;
    if (a.splits > 1) {
        const int64_t units = rows * 2 * a.splits;
        a.part_o = static_cast<float *>(ws);
        a.part_ml = reinterpret_cast<float2 *>(static_cast<char *>(ws) +
                                               align_up((size_t)units * kHq * kDh * sizeof(float), 256));
    }
    if (cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return DSA_ERR_CUDA;
    sparse_mla_tc_kernel<<<(unsigned)(rows * 2 * a.splits), kThreads, kSmemBytes, stream>>>(tm_q, a);
    dsa_status st = launch_status();
    if (st != DSA_OK || a.splits == 1) return st;
    sparse_mla_combine_kernel<<<(unsigned)(rows * 2 * (kHq / kCombineHeads)), 32 * kCombineHeads,
                                0, stream>>>(a.part_o, a.part_ml, a.splits, a.out, lse);
    return launch_status();
}

}  // namespace dsa
