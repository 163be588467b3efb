// sparse_mla_tc.cu -- tensor-core sparse latent attention (V3.2 shapes).
//
// Pages: the diagram "DeepSeek Sparse Attention, one decode step in one layer
// (V3.2 sizes)" (core attention in MQA mode: 128 heads over the gathered
// 576-wide latent rows, each row key and value; latents cached as "FP8 + bf16
// RoPE" in 656-byte rows) and the MLA prefill excerpt of "DeepSeek-V3.2-Exp -
// Causal mask" (index mask + causal mask, softmax, value mix).
//
// Shapes: Hq = 128 heads (the MMA M), rows [c (512) | k_pe (64)].
// Work unit: one query row and U = 128 consecutive slots of its selection
// (slots holding -1 or a future position count as empty rows), computed by one
// CTA, which
//   1. gathers the unit's rows in nine 64-column chunks (eight latent blocks
//      and the rotary block), each into its own 16 KB 128B-swizzled K-major
//      tile -- all nine stay resident, so every gather is issued up front --
//      and accumulates the logits S = Q C^T (M = 128 heads, N = 128, K = 576)
//      in TMEM with 36 tcgen05.mma kind::f16, A = the query's latent part
//      from TMEM and its rotary block from shared memory;
//   2. runs an exact softmax over the unit's 128 logits of each head (the
//      thread's logits stay in registers between the max and the exp2 pass)
//      and writes P as bf16 into shared memory, the A operand of the value mix;
//   3. accumulates O = P C[:, 0:512] (M = 128, K = 128), whose B operands are
//      the latent chunks already resident (read MN-major), into all 512 TMEM
//      columns as four N = 128 quarters, each committed on its own;
//   4. writes bf16 out (+ lse) when the row has one unit, else a normalised
//      fp16 partial with its (max, sum, power-of-two ranges per column half),
//      quarter by quarter as the MMAs complete, so that the stores overlap the
//      following quarters' MMAs.  The once-per-CTA loops here are rolled:
//      straight-line code that runs once stalls on instruction fetch.  The partials of
//      a row's units ("splits") are merged by a combine kernel launched right
//      behind (programmatic launch: its CTAs are resident, waiting, while the
//      attention finishes).  The attention itself is a plain programmatic
//      launch too, so its CTAs start their set-up (barriers, TMEM, the query's
//      TMA) on the SMs the top-k leaves free.
//
// Shared memory: nine chunk regions R0..R8 (R k holds chunk k), the query's
// rotary block, and P (two 16 KB K-major blocks).  The query's latent blocks
// are staged by TMA in P's space (blocks 0, 1) and in R2..R7 (blocks 2..7)
// before the work threads move them to TMEM, so chunks 0, 1 and 8 are gathered
// at once and chunks 2..7 once the staging is free.
// TMEM: S in columns [0, 128) and the query's latent part in [256, 512) while
// the logits accumulate; then O in [0, 512).
//
// The FP8 variant reads 656-byte rows [512 e4m3 | 4 fp32 block scales | 64
// bf16].  The codes of a latent chunk are copied into the upper half of its
// region and decoded in place (code * block scale, rounded to bf16 -- the same
// decoded operand as the oracle's), so the rows cross HBM once at 656 bytes
// and no decoded copy is ever written to memory.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

constexpr int kHq = 128, kDc = 512, kDr = 64, kDqk = kDc + kDr;
constexpr int kU = 128;                         // selected rows per unit (the MMA N of the logits)
constexpr int kChunks = 9;                      // 8 latent blocks + the rotary block
constexpr int kRegion = kU * 128;               // one chunk of 128 rows: 16 KB
constexpr int kQBlk = kHq * 128;                // one 64-column block of the query: 16 KB
constexpr int kQRope = kChunks * kRegion;       // the query's rotary block
constexpr int kP = kQRope + kQBlk;              // P: two K-major blocks of 64 slots
constexpr int kScales = kP + 2 * kQBlk;         // FP8: the unit's block scales, 16 B per row
constexpr int kList = kScales + kU * 16;        // the unit's rows (int32)
constexpr int kBars = kList + kU * 4;
constexpr int kWork = 256;                      // gather / softmax / epilogue threads
constexpr int kThreads = kWork + 32;            // + one TMA / MMA warp
constexpr int kMaxSel = 2048;                   // selection slots per query row
constexpr int kOct = kDc / 8;                   // output octets per head: 64
constexpr uint32_t kColS = 0, kColQ = 256, kColO = 0, kTmemCols = 512;
constexpr int kRowFp8 = kDc + 4 * (kDc / 128) + 2 * kDr;   // 656
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t kSmemBytes = 1024 + (size_t)kBars + 32 * sizeof(uint64_t) + 64;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// where the query's latent block cb is staged by TMA
__device__ __forceinline__ int q_stage(int cb) { return cb < 2 ? kP + cb * kQBlk : cb * kRegion; }

struct MlaArgs {
    const __nv_bfloat16 *q;    // [rows, 128, 576]
    const __nv_bfloat16 *kv;   // bf16 rows [B, t_max, 576]
    const uint8_t *kv8;        // FP8 rows [B, t_max, 656]
    const int32_t *idx;
    __nv_bfloat16 *out;
    float *lse;
    __half *part_o;            // [blocks][64 octets][128][8] (split partials)
    float4 *part_ml;           // [blocks][128] (max, sum, fp16 range of columns 0..255, of 256..511)
    int64_t t_max;
    int64_t start_pos;
    int64_t row0;              // first query row of this launch
    int S, k, splits;
    float scale_log2;          // sm_scale * log2(e)
    int *err;
};

// 16-byte cp.async; src_bytes = 0 fills the 16 bytes with zeros (nothing is read)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Arrives on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts against the barrier's initial count); the thread does
// not wait.
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar))
                 : "memory");
}
// waits until at most n of this thread's cp.async groups are pending (0 <= n <= 5)
__device__ __forceinline__ void cp_async_wait_n(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    }
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// 2^x by the SFU (relative error about 2^-22, far below the bf16 rounding of
// P; 2^-inf = +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Eight e4m3 codes (two words) times the block scale, rounded to bf16 pairs.
__device__ __forceinline__ uint4 decode8(uint32_t w0, uint32_t w1, float sc) {
    uint32_t o[4];
    const uint32_t w[2] = {w0, w1};
#pragma unroll
    for (int q = 0; q < 2; q++) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>((w[q] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
            const __nv_bfloat162 v2 = __floats2bfloat162_rn(f.x * sc, f.y * sc);
            o[2 * q + h] = *reinterpret_cast<const uint32_t *>(&v2);
        }
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Merges output columns [8 c8, 8 c8 + 8) of head h of one query row from its
// splits' fp16 partials (blocks blk0 .. blk0 + splits - 1), for NC octets
// c8[0..NC) at once: with w_s = 2^(m_s - M) l_s and Y_s = O_s / (l_s sc_s),
// out = sum_s w_s sc_s Y_s / sum_s w_s and lse = (M + log2 sum_s w_s) ln 2.
// The loads of kMergeBatch splits are in flight together (eight of the
// sixteen of a 2048-slot row, for two octets at once); further batches
// rescale the running sums.
constexpr int kMergeBatch = 8;
template <int NC>
__device__ __forceinline__ void merge_octets(const __half *part_o, const float4 *part_ml, int splits,
                                             int64_t blk0, int64_t row, const int (&c8)[NC], int h,
                                             __nv_bfloat16 *out, float *lse) {
    float M = -INFINITY, L = 0.f;
    float acc[NC][8];
#pragma unroll
    for (int n = 0; n < NC; n++)
#pragma unroll
        for (int e = 0; e < 8; e++) acc[n][e] = 0.f;
    for (int s0 = 0; s0 < splits; s0 += kMergeBatch) {
        float4 ml[kMergeBatch];
        uint4 x[kMergeBatch][NC];
#pragma unroll
        for (int u = 0; u < kMergeBatch; u++) {
            const int sp = s0 + u;
            ml[u] = sp < splits ? part_ml[(blk0 + sp) * kHq + h] : make_float4(-INFINITY, 0.f, 1.f, 1.f);
#pragma unroll
            for (int n = 0; n < NC; n++)
                if (sp < splits)
                    x[u][n] = reinterpret_cast<const uint4 *>(part_o + (blk0 + sp) * kHq * kDc)[c8[n] * kHq + h];
        }
        float mb = M;
#pragma unroll
        for (int u = 0; u < kMergeBatch; u++) mb = fmaxf(mb, ml[u].x);
        if (mb == -INFINITY) continue;
        if (mb > M) {                                  // rescale the running sums
            const float r = M == -INFINITY ? 0.f : ex2(M - mb);
            L *= r;
#pragma unroll
            for (int n = 0; n < NC; n++)
#pragma unroll
                for (int e = 0; e < 8; e++) acc[n][e] *= r;
            M = mb;
        }
#pragma unroll
        for (int u = 0; u < kMergeBatch; u++) {
            if (ml[u].x == -INFINITY) continue;
            const float w = ex2(ml[u].x - M) * ml[u].y;
            L += w;
#pragma unroll
            for (int n = 0; n < NC; n++) {
                const float ws = w * (c8[n] < kOct / 2 ? ml[u].z : ml[u].w);
                const uint32_t xs[4] = {x[u][n].x, x[u][n].y, x[u][n].z, x[u][n].w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&xs[e]));
                    acc[n][2 * e] = fmaf(ws, f.x, acc[n][2 * e]);
                    acc[n][2 * e + 1] = fmaf(ws, f.y, acc[n][2 * e + 1]);
                }
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int n = 0; n < NC; n++) {
        uint32_t w8[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(acc[n][2 * e] * inv, acc[n][2 * e + 1] * inv);
            w8[e] = *reinterpret_cast<const uint32_t *>(&v);
        }
        reinterpret_cast<uint4 *>(out + (row * kHq + h) * kDc)[c8[n]] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        if (c8[n] == 0 && lse) lse[row * kHq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int32_t *list = reinterpret_cast<int32_t *>(sm + kList);             // the unit's rows
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBars);
    uint64_t *chunk_full = bars;                 // [9] chunk k gathered (256 arrivals)
    uint64_t *q_full = bars + kChunks;           // the query landed (TMA)
    uint64_t *q_ready = q_full + 1;              // the query's latent part is in TMEM (256 arrivals)
    uint64_t *s_done = q_ready + 1;              // every logit MMA is complete
    uint64_t *p_full = s_done + 1;               // P is in shared memory (256 arrivals)
    uint64_t *o_full = p_full + 1;               // [4] column quarter q of O is complete
    uint64_t *mma_fin = o_full + 4;              // every issued MMA is complete
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 20);   // after the 18 barriers
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    uint32_t *vmask = reinterpret_cast<uint32_t *>(const_cast<int *>(abort) + 1);   // [4]
    // softmax exchange (max and sum of the two slot halves): the query's
    // rotary block, free once the logits are complete
    float *red = reinterpret_cast<float *>(sm + kQRope);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x = (row - row0) * splits + sp
    const int sp = (int)(blockIdx.x % (unsigned)a.splits);
    const int64_t row = a.row0 + blockIdx.x / (unsigned)a.splits;
    const int64_t b = row / a.S, s = row - b * a.S;
    const int64_t limit = a.start_pos + s;
    const uint32_t sbase = tc::smem_u32(sm);

    if (warp == kWork / 32) {
        if (lane == 0) {
            for (int i = 0; i < kChunks; i++) tc::mbar_init(&chunk_full[i], kWork);
            tc::mbar_init(q_full, 1);
            tc::mbar_init(q_ready, kWork);
            tc::mbar_init(s_done, 1);
            tc::mbar_init(p_full, kWork);
            for (int i = 0; i < 4; i++) tc::mbar_init(&o_full[i], 1);
            tc::mbar_init(mma_fin, 1);
            *abort = 0;
            tc::fence_mbar_init();
            tc::tma_prefetch_desc(&tm_q);
        }
        __syncwarp();
        tc::tmem_alloc(tmem_holder, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    if (warp == kWork / 32 && lane == 0) {
        // the query: its rotary block stays in shared memory (the MMA's A
        // operand there); its eight latent blocks are staged in P's space and
        // R2..R7 and moved to TMEM by the work threads
        tc::mbar_arrive_expect_tx(q_full, kChunks * kQBlk);
        tc::tma_load_2d(sm + kQRope, &tm_q, kDc, (int)(row * kHq), q_full);
        for (int cb = 0; cb < 8; cb++)
            tc::tma_load_2d(sm + q_stage(cb), &tm_q, cb * 64, (int)(row * kHq), q_full);
    }
    // a kernel launched after this one (the split combine) may start its set-up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // The selections come from the preceding kernel (the top-k): wait for it
    // (a no-op without a programmatic launch), then read them with plain loads.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // This unit is the slots [lo, lo + 128) of the row's selection, slot lo + j
    // as row j.  A slot counts when it holds a causal position (>= 0 and <=
    // start_pos + s); vmask has one bit per row.  (A top-k selection lists
    // its positions first and pads with -1, so its units are dense.)
    const int lo = sp * kU;
    if (threadIdx.x < kU) {
        const int j = threadIdx.x;
        int32_t t = -1;
        if (lo + j < a.k) {
            t = a.idx[row * a.k + lo + j];
            if (t >= 0 && (int64_t)t <= limit) {
                if ((int64_t)t >= a.t_max) {
                    record_error(a.err, DSA_ERR_DEVICE);
                    t = -1;
                }
            } else {
                t = -1;
            }
        }
        list[j] = t;
        const uint32_t bal = __ballot_sync(0xffffffffu, t >= 0);
        if (lane == 0) vmask[warp] = bal;
    }
    __syncthreads();
    const uint32_t any = vmask[0] | vmask[1] | vmask[2] | vmask[3];
    const int64_t rbase = b * a.t_max;

    if (!any) {
        // nothing selected in this unit: an empty partial (or a zero output)
        if (threadIdx.x < kWork) {
            const int h = threadIdx.x & (kHq - 1), c = threadIdx.x >> 7;
            if (a.splits > 1) {
                uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)blockIdx.x * kHq * kDc) + h;
                for (int o8 = 32 * c; o8 < 32 * c + 32; o8++) po[o8 * kHq] = make_uint4(0u, 0u, 0u, 0u);
                if (c == 0) a.part_ml[(int64_t)blockIdx.x * kHq + h] = make_float4(-INFINITY, 0.f, 1.f, 1.f);
            } else {
                uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + c * 256);
                for (int j = 0; j < 32; j++) o16[j] = make_uint4(0u, 0u, 0u, 0u);
                if (c == 0 && a.lse) a.lse[row * kHq + h] = -INFINITY;
            }
        }
        if (warp == kWork / 32 && lane == 0) tc::mbar_wait(q_full, 0, a.err, abort);
    } else if (warp < kWork / 32) {
        const int gt = threadIdx.x;
        const int q4 = warp & 3, c = warp >> 2;          // TMEM lane quarter; slot half / column half
        const int h = q4 * 32 + lane;                    // head
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        bool ok = true;
        // ------------------------------------------------------------ gather
        // Issue chunk k into region k: 16-byte cp.async pieces (empty rows are
        // zero-filled: finite values that meet P = 0).  bf16 rows and the FP8
        // rotary block land in their swizzled tile; FP8 codes land in the
        // upper half of the region, to be decoded in place.
        auto issue = [&](int k) {
            const uint32_t rg = sbase + k * kRegion;
            if (!kFp8 || k == 8) {
#pragma unroll
                for (int u = 0; u < kU * 8 / kWork; u++) {
                    const int f = gt + u * kWork, j = f >> 3, p = f & 7;
                    const int32_t tl = list[j];
                    const bool v = tl >= 0;
                    const int64_t t = v ? (int64_t)tl : 0;
                    const void *src;
                    if constexpr (kFp8)
                        src = a.kv8 + (rbase + t) * kRowFp8 + kDc + 4 * (kDc / 128) + p * 16;
                    else
                        src = a.kv + (rbase + t) * kDqk + k * 64 + p * 8;
                    cp_async16(rg + j * 128 + ((p ^ (j & 7)) << 4), src, v ? 16u : 0u);
                }
            } else {
#pragma unroll
                for (int u = 0; u < kU * 4 / kWork; u++) {
                    const int f = gt + u * kWork, j = f >> 2, p = f & 3;
                    const int32_t tl = list[j];
                    const bool v = tl >= 0;
                    const int64_t t = v ? (int64_t)tl : 0;
                    cp_async16(rg + kRegion / 2 + j * 64 + p * 16,
                               a.kv8 + (rbase + t) * kRowFp8 + k * 64 + p * 16, v ? 16u : 0u);
                }
                if (k == 0 && gt < kU) {                  // the row's four block scales
                    const int32_t tl = list[gt];
                    const bool v = tl >= 0;
                    const int64_t t = v ? (int64_t)tl : 0;
                    cp_async16(sbase + kScales + gt * 16, a.kv8 + (rbase + t) * kRowFp8 + kDc,
                               v ? 16u : 0u);
                }
            }
            cp_async_commit();
            // bf16 chunks are published by the copies themselves (an arrival
            // when this thread's copies so far have landed)
            if constexpr (!kFp8) cp_async_arrive(&chunk_full[k]);
        };
        // FP8: chunk k has landed for this thread (`pending` later groups may
        // still be in flight); its latent codes are decoded in place (every
        // thread's codes must have landed before any are read, and every read
        // must be done before the first write), then the chunk is published.
        auto publish = [&](int k, int pending) {
            cp_async_wait_n(pending);
            if (k != 8) {
                const uint32_t rg = sbase + k * kRegion;
                constexpr int kPer = kU * 4 / kWork;         // 16-code pieces per thread
                uint4 cw[kPer];
                float sc[kPer];
                tc::named_barrier(1, kWork);
#pragma unroll
                for (int u = 0; u < kPer; u++) {
                    const int f = gt + u * kWork, j = f >> 2, p = f & 3;
                    cw[u] = ld_shared_v4(rg + kRegion / 2 + j * 64 + p * 16);
                    sc[u] = reinterpret_cast<const float *>(sm + kScales + j * 16)[k >> 1];
                }
                tc::named_barrier(1, kWork);
#pragma unroll
                for (int u = 0; u < kPer; u++) {
                    const int f = gt + u * kWork, j = f >> 2, p = f & 3;
                    st_shared_v4(rg + j * 128 + (((2 * p) ^ (j & 7)) << 4), decode8(cw[u].x, cw[u].y, sc[u]));
                    st_shared_v4(rg + j * 128 + (((2 * p + 1) ^ (j & 7)) << 4), decode8(cw[u].z, cw[u].w, sc[u]));
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&chunk_full[k]);
        };
        // chunks 0, 1 and 8 go to free regions at once; 2..7 once the query's
        // latent part has left its staging
        issue(0);
        issue(1);
        issue(8);
        // the query's latent part (head h, blocks 4c..4c+3) from its swizzled
        // staging to TMEM columns kColQ + 32 cb, two bf16 per column
        if (ok && !tc::mbar_wait(q_full, 0, a.err, abort)) ok = false;
#pragma unroll 1
        for (int blk = 0; blk < 4; blk++) {
            const int cb = 4 * c + blk;
            const uint32_t src = sbase + q_stage(cb) + h * 128;
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                uint32_t r[16];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const uint4 v = ld_shared_v4(src + (((4 * hf + i) ^ (h & 7)) << 4));
                    r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
                }
                tc::tmem_st16(tmem + lane_addr + kColQ + cb * 32 + hf * 16, r);
            }
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(q_ready);
        tc::named_barrier(1, kWork);            // the staging is no longer read
        for (int k = 2; k < 8; k++) issue(k);
        if constexpr (kFp8) {
            // in issue order: 0, 1, 8, 2, ..., 7
            publish(0, 8);
            publish(1, 7);
            publish(8, 6);
            for (int k = 2; k < 8; k++) publish(k, 7 - k);
        }

        // ----------------------------------------------------------- softmax
        // thread (head h, slot half c): the logits of rows [64c, 64c + 64),
        // kept in registers between the max and the exp2 pass; rows of no
        // selection count as -inf; eight independent chains for the max and
        // the sum
        if (ok && !tc::mbar_wait(s_done, 0, a.err, abort)) ok = false;
        tc::tc_fence_after();
        // (rolled over four groups of 16 logits, re-read from TMEM in the
        // second pass: this code runs once per CTA, and straight-line code
        // of that length stalls on instruction fetch)
        const uint32_t w0 = vmask[2 * c], w1 = vmask[2 * c + 1];
        const bool part = (w0 & w1) != 0xffffffffu;
        const uint32_t scol = tmem + lane_addr + kColS + 64 * c;
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; e++) mx8[e] = -INFINITY;
#pragma unroll 1
        for (int i = 0; i < 4; i++) {
            uint32_t sv[16];
            tc::tmem_ld16(scol + 16 * i, sv);
            tc::tmem_wait_ld();
            const uint32_t wb = (i < 2 ? w0 : w1) >> (16 * (i & 1));
#pragma unroll
            for (int e = 0; e < 16; e++) {
                float x = __uint_as_float(sv[e]) * a.scale_log2;
                if (part && !((wb >> e) & 1u)) x = -INFINITY;
                mx8[e & 7] = fmaxf(mx8[e & 7], x);
            }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        red[c * kHq + h] = mx;
        tc::named_barrier(1, kWork);
        const float m = fmaxf(red[h], red[kHq + h]);       // finite: the unit has a row
        float l8[8];
#pragma unroll
        for (int e = 0; e < 8; e++) l8[e] = 0.f;
        // P of rows [64c, 64c + 64) is the K-major block c of the A operand:
        // head h's 128-byte row, 16-byte piece i = rows 8i .. 8i + 7
        const uint32_t prow = sbase + kP + c * kQBlk + h * 128;
#pragma unroll 1
        for (int i = 0; i < 4; i++) {
            uint32_t sv[16];
            tc::tmem_ld16(scol + 16 * i, sv);
            tc::tmem_wait_ld();
            const uint32_t wb = (i < 2 ? w0 : w1) >> (16 * (i & 1));
#pragma unroll
            for (int hp = 0; hp < 2; hp++) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int x = 8 * hp + 2 * e;
                    float t0 = fmaf(__uint_as_float(sv[x]), a.scale_log2, -m);
                    float t1 = fmaf(__uint_as_float(sv[x + 1]), a.scale_log2, -m);
                    if (part && !((wb >> x) & 1u)) t0 = -INFINITY;
                    if (part && !((wb >> (x + 1)) & 1u)) t1 = -INFINITY;
                    const float p0 = ex2(t0), p1 = ex2(t1);
                    l8[(2 * e) & 7] += p0;
                    l8[(2 * e + 1) & 7] += p1;
                    const __nv_bfloat162 v01 = __floats2bfloat162_rn(p0, p1);
                    pk[e] = *reinterpret_cast<const uint32_t *>(&v01);
                }
                st_shared_v4(prow + (((2 * i + hp) ^ (h & 7)) << 4),
                             make_uint4(pk[0], pk[1], pk[2], pk[3]));
            }
        }
        // P is read by the tensor core (async proxy)
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(p_full);
        red[2 * kHq + c * kHq + h] = ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        tc::named_barrier(1, kWork);
        const float lt = red[2 * kHq + h] + red[3 * kHq + h];

        // ---------------------------------------------------------- epilogue
        if (a.splits == 1) {
            // thread (h, c) owns output columns [256c, 256c + 256)
            if (ok && !tc::mbar_wait(&o_full[2 * c], 0, a.err, abort)) ok = false;
            if (ok && !tc::mbar_wait(&o_full[2 * c + 1], 0, a.err, abort)) ok = false;
            tc::tc_fence_after();
            const uint32_t ocol = tmem + lane_addr + kColO + c * 256;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + c * 256);
#pragma unroll 1
            for (int g = 0; g < 16; g++) {
                uint32_t ov[16];
                tc::tmem_ld16(ocol + 16 * g, ov);
                tc::tmem_wait_ld();
#pragma unroll
                for (int o8 = 0; o8 < 2; o8++) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(ov[8 * o8 + 2 * e]) * inv,
                                                                       __uint_as_float(ov[8 * o8 + 2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    if (ok) o16[2 * g + o8] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (ok && c == 0 && a.lse) a.lse[row * kHq + h] = lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
        } else {
            // O / (l * sc) in fp16 for the split merge, as [column / 8][head]
            // groups of eight halves, sc per column half: the power of two
            // that keeps the half's |O / l| / sc <= 2^14.  The quarters are
            // written in MMA completion order, both threads of a head taking
            // 64 columns of each; a half's two quarters are written with
            // sc = 1 and written again only when the head's max |O| over the
            // half's 256 columns (the two threads' maxima) asks for a larger
            // range.
            const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
            uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)blockIdx.x * kHq * kDc) + h;
            float *ml = reinterpret_cast<float *>(a.part_ml + (int64_t)blockIdx.x * kHq + h);
            float *xmax = red + 4 * kHq;          // [half][c][head]
            auto write_cols = [&](uint32_t ocol, int oct0, float inv, bool track) -> float {
                float amax = 0.f;
#pragma unroll 1
                for (int g = 0; g < 4; g++) {
                    uint32_t ov[16];
                    tc::tmem_ld16(ocol + 16 * g, ov);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int o8 = 0; o8 < 2; o8++) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const float x0 = __uint_as_float(ov[8 * o8 + 2 * e]);
                            const float x1 = __uint_as_float(ov[8 * o8 + 2 * e + 1]);
                            if (track) amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
                            const __half2 v = __floats2half2_rn(x0 * inv, x1 * inv);
                            w[e] = *reinterpret_cast<const uint32_t *>(&v);
                        }
                        if (ok) po[(oct0 + 2 * g + o8) * kHq] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                return amax;
            };
            // quarter q: thread (h, c) writes columns [128q + 64c, 128q + 64c + 64)
            float hmax = 0.f;
#pragma unroll 1
            for (int q = 0; q < 4; q++) {
                if (ok && !tc::mbar_wait(&o_full[q], 0, a.err, abort)) ok = false;
                tc::tc_fence_after();
                hmax = fmaxf(hmax, write_cols(tmem + lane_addr + kColO + 128 * q + 64 * c,
                                              16 * q + 8 * c, inv_l, true));
                if (!(q & 1)) continue;
                // column half hv = q / 2 complete: its range, from both threads of the head
                const int hv = q >> 1;
                xmax[(2 * hv + c) * kHq + h] = hmax;
                hmax = 0.f;
                tc::named_barrier(1, kWork);
                const float amax = fmaxf(xmax[2 * hv * kHq + h], xmax[(2 * hv + 1) * kHq + h]);
                float scl = 1.f;
                while (amax * inv_l > 16384.f * scl) scl *= 2.f;
                if (scl != 1.f) {
                    for (int q2 = q - 1; q2 <= q; q2++)
                        write_cols(tmem + lane_addr + kColO + 128 * q2 + 64 * c, 16 * q2 + 8 * c,
                                   inv_l / scl, false);
                }
                if (ok && c == 0) ml[2 + hv] = scl;
            }
            // (max, sum, range of columns [0, 256), range of columns [256, 512))
            if (ok && c == 0) {
                ml[0] = m;
                ml[1] = lt;
            }
        }
    } else if (lane > 0) {
        // lanes 1..31 of the MMA warp: the unit's rows into L2, whole rows at
        // a time, ahead of the chunk gathers
        for (int j = lane - 1; j < kU; j += 31) {
            if (list[j] < 0) continue;
            if constexpr (kFp8)
                tc::prefetch_l2_bulk(a.kv8 + (rbase + list[j]) * kRowFp8, kRowFp8);
            else
                tc::prefetch_l2_bulk(a.kv + (rbase + list[j]) * kDqk, kDqk * 2);
        }
    } else {
        // ------------------------------------------------------ TMA / MMA
        const uint32_t id_qk = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, kU);
        bool ok = tc::mbar_wait(q_full, 0, a.err, abort) && tc::mbar_wait(q_ready, 0, a.err, abort);
        // chunks in issue order: 0, 1, 8, 2, ..., 7
        for (int i = 0; ok && i < kChunks; i++) {
            const int k = i < 2 ? i : (i == 2 ? 8 : i - 1);
            if (!tc::mbar_wait(&chunk_full[k], 0, a.err, abort)) {
                ok = false;
                break;
            }
            // the chunk's bytes were written through the generic proxy (cp.async
            // or stores): order them before the tensor core's reads
            tc::fence_proxy_async_smem();
            tc::tc_fence_after();
            const uint32_t ca = sbase + k * kRegion;
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                const uint64_t bd = tc::smem_desc(ca + ks * 32, 1024, tc::kSwizzle128B);
                if (k < 8)         // A = the query's latent block k in TMEM
                    tc::mma_f16_ts(tmem + kColS, tmem + kColQ + k * 32 + ks * 8, bd, id_qk,
                                   i > 0 || ks > 0);
                else               // A = the query's rotary block in shared memory
                    tc::mma_f16(tmem + kColS,
                                tc::smem_desc(sbase + kQRope + ks * 32, 1024, tc::kSwizzle128B), bd,
                                id_qk, i > 0 || ks > 0);
            }
        }
        if (ok) tc::tc_commit(s_done);
        if (ok && tc::mbar_wait(p_full, 0, a.err, abort)) {
            tc::tc_fence_after();
            // O[:, 128 q + n] += P C[:, 128 q + n]: K-step ks covers rows
            // [16 ks, 16 ks + 16); A = P (K-major, block ks / 4), B = the latent
            // chunks 2q, 2q + 1 (MN-major, 16 KB between 64-column blocks).
            // Each quarter is committed before the next is issued, so that its
            // epilogue overlaps the following quarters' MMAs.
            const uint32_t id_pv = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, 128, true);
            for (int q = 0; q < 4; q++) {
                for (int ks = 0; ks < kU / 16; ks++) {
                    const uint64_t pa = tc::smem_desc(sbase + kP + (ks >> 2) * kQBlk + (ks & 3) * 32,
                                                      1024, tc::kSwizzle128B);
                    const uint64_t bd = tc::smem_desc(sbase + 2 * q * kRegion + ks * 2048, 1024,
                                                      tc::kSwizzle128B, kRegion);
                    tc::mma_f16(tmem + kColO + 128 * q, pa, bd, id_pv, ks > 0);
                }
                tc::tc_commit(&o_full[q]);
            }
        }
        // every issued MMA completes before TMEM is released
        tc::tc_commit(mma_fin);
        tc::mbar_wait(mma_fin, 0, a.err, abort);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == kWork / 32) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// Merges the splits of each query row: thread (head, octet pair) merges
// sixteen output columns of one head, consecutive threads consecutive heads
// (coalesced reads of the partials): 256 CTAs at B = 8, all resident beside
// the attention's CTAs, waiting.  The next kernel (the next step's scorer) is
// released only once the attention has completed, so that its CTAs do not
// take the SMs that the attention's last CTAs are waiting for.
__global__ void __launch_bounds__(kHq)
sparse_mla_combine_kernel(const __half *part_o, const float4 *part_ml, int splits, int64_t row0,
                          __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    // the partials come from the preceding kernel: wait for it (plain loads below)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the next kernel may start its set-up while the splits are merged
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t r = blockIdx.x / (kOct / 2);           // row - row0
    const int pair = (int)(blockIdx.x % (kOct / 2));
    const int c8[2] = {2 * pair, 2 * pair + 1};
    merge_octets<2>(part_o, part_ml, splits, r * splits, row0 + r, c8, threadIdx.x, out, lse);
}

// Split partials of one query row.
size_t partial_bytes_per_row(int splits) {
    return (size_t)splits * kHq * (kDc * sizeof(__half) + sizeof(float4));
}

// Query rows per launch: all of them, unless their split partials would pass
// kWsBudget; then the rows run in launches of this many (each reusing the
// workspace after its merge).
constexpr size_t kWsBudget = size_t(256) << 20;
int64_t rows_per_launch(int64_t rows, int splits) {
    if (splits <= 1) return rows;
    int64_t r = (int64_t)(kWsBudget / partial_bytes_per_row(splits));
    if (r < 1) r = 1;
    return r < rows ? r : rows;
}

size_t workspace_bytes(int64_t rows, int k) {
    const int sp = (k + kU - 1) / kU;
    if (sp <= 1) return 0;
    const int64_t units = rows_per_launch(rows, sp) * sp;
    return align_up((size_t)units * kHq * kDc * sizeof(__half), 256) +
           (size_t)units * kHq * sizeof(float4);
}

template <bool kFp8>
dsa_status launch(const void *q, const void *kv, int64_t t_max, const int32_t *idx, int B, int S,
                  int k, int64_t start_pos, float sm_scale, void *out, float *lse, void *ws,
                  cudaStream_t stream) {
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
    MlaArgs a = {};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.kv = kFp8 ? nullptr : static_cast<const __nv_bfloat16 *>(kv);
    a.kv8 = kFp8 ? static_cast<const uint8_t *>(kv) : nullptr;
    a.idx = idx;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.t_max = t_max;
    a.start_pos = start_pos;
    a.S = S;
    a.k = k;
    a.splits = (k + kU - 1) / kU;
    a.scale_log2 = sm_scale * kLog2e;
    a.err = device_error_word();
    const int64_t chunk = rows_per_launch(rows, a.splits);
    if (a.splits > 1) {
        const int64_t units = chunk * a.splits;
        a.part_o = static_cast<__half *>(ws);
        a.part_ml = reinterpret_cast<float4 *>(static_cast<char *>(ws) +
                                               align_up((size_t)units * kHq * kDc * sizeof(__half), 256));
    }
    if (cudaFuncSetAttribute(sparse_mla_tc_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return DSA_ERR_CUDA;
    for (int64_t r0 = 0; r0 < rows; r0 += chunk) {
        const int64_t n = rows - r0 < chunk ? rows - r0 : chunk;
        a.row0 = r0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(n * a.splits));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.stream = stream;
        // programmatic launch: the kernel's set-up overlaps the preceding
        // kernel's tail; it waits for that kernel before reading the selections
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, sparse_mla_tc_kernel<kFp8>, tm_q, a) != cudaSuccess)
            return DSA_ERR_CUDA;
        dsa_status st = launch_status();
        if (st != DSA_OK) return st;
        if (a.splits == 1) continue;
        cudaLaunchConfig_t ccfg = {};
        ccfg.gridDim = dim3((unsigned)(n * (kOct / 2)));
        ccfg.blockDim = dim3(kHq);
        ccfg.stream = stream;
        cudaLaunchAttribute cattr[1];
        cattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        cattr[0].val.programmaticStreamSerializationAllowed = 1;
        ccfg.attrs = cattr;
        ccfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&ccfg, sparse_mla_combine_kernel, (const __half *)a.part_o,
                               (const float4 *)a.part_ml, a.splits, r0, a.out, lse) != cudaSuccess)
            return DSA_ERR_CUDA;
        if ((st = launch_status()) != DSA_OK) return st;
    }
    return DSA_OK;
}

}  // namespace

bool sparse_mla_tc_supported(int Hq, int dc, int dr, int k, dsa_dtype dt) {
    return dt == DSA_BF16 && Hq == kHq && dc == kDc && dr == kDr && k <= kMaxSel;
}

bool sparse_mla_fp8_tc_supported(int Hq, int dc, int dr, int k) {
    return Hq == kHq && dc == kDc && dr == kDr && k <= kMaxSel;
}

size_t sparse_mla_tc_workspace_bytes(int B, int S, int k) {
    return workspace_bytes((int64_t)B * S, k);
}

dsa_status launch_sparse_mla_tc(const void *q, const void *kv, int64_t t_max, const int32_t *idx,
                                int B, int S, int k, int64_t start_pos, float sm_scale, void *out,
                                float *lse, void *ws, cudaStream_t stream) {
    return launch<false>(q, kv, t_max, idx, B, S, k, start_pos, sm_scale, out, lse, ws, stream);
}

dsa_status launch_sparse_mla_fp8_tc(const void *q, const uint8_t *kv8, int64_t t_max,
                                    const int32_t *idx, int B, int S, int k, int64_t start_pos,
                                    float sm_scale, void *out, float *lse, void *ws,
                                    cudaStream_t stream) {
    return launch<true>(q, kv8, t_max, idx, B, S, k, start_pos, sm_scale, out, lse, ws, stream);
}

}  // namespace dsa
