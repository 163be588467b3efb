// sparse_mla_tc.cu -- tensor-core sparse latent attention (V3.2 shapes).
//
// Pages: the diagram "DeepSeek Sparse Attention, one decode step in one layer
// (V3.2 sizes)" (core attention in MQA mode: 128 heads over the gathered
// 576-wide latent rows, each row key and value; latents cached as "FP8 + bf16
// RoPE" in 656-byte rows) and the MLA prefill excerpt of "DeepSeek-V3.2-Exp -
// Causal mask" (index mask + causal mask, softmax, value mix).
//
// Shapes: Hq = 128 heads (the MMA M), rows [c (512) | k_pe (64)].
// Work unit: one query row and a contiguous share of U <= 256 of its selected
// rows (in slot order), computed by TWO independent CTAs that differ only in
// which half of the 512 output columns they produce.  Each CTA
//   1. gathers the U rows in nine 64-column chunks (eight latent blocks and
//      the rotary block) into 128B-swizzled K-major tiles, and accumulates the
//      full logits S = Q C^T (M = 128 heads, N = U, K = 576) in TMEM with 36
//      tcgen05.mma kind::f16 -- the logits are complete in every CTA, so no
//      partial logits ever move between CTAs;
//   2. runs an exact softmax over the U logits of each head (two passes over
//      TMEM: the max, then exp2, the sum and P as bf16 written in place over
//      the logits it came from);
//   3. accumulates O = P C[:, own 256 columns] (M = 128, N = 256, K = U) with
//      A = P read from TMEM and B = the CTA's four own latent chunks, which
//      were gathered last and stay in shared memory (read MN-major), so the
//      value mix needs no second gather;
//   4. writes its 256 output columns: bf16 out (+ lse) when the row has one
//      unit, else a normalised fp16 partial with its (max, sum, power-of-two
//      range) for the split combine.
// The two CTAs of a unit read the same rows; the second read is served from
// L2 (each CTA also prefetches half of the unit's rows into L2 at its start).
//
// Shared memory: five 32 KB chunk regions G0..G4 and the CTA's four own query
// blocks (64 KB).  The query's five other blocks are staged by TMA in G2..G4
// and consumed first, so the own latent chunks (chunks 5..8) can land in
// G1..G4 -- consecutive regions, one MN-major operand with a 32 KB stride
// between its 64-column blocks.  Chunk order and regions:
//   chunk   0    1    2    3    4      5..8
//   block   4 other latent blocks, rope, 4 own latent blocks
//   region  G0   G1   G0   G1   G0     G1 G2 G3 G4
// TMEM: S / P in columns [0, U), O in [256, 512).
//
// The FP8 variant reads 656-byte rows [512 e4m3 | 4 fp32 block scales | 64
// bf16] and decodes each latent chunk while gathering it (code * block scale,
// rounded to bf16 -- the same decoded operand as the oracle's), so the rows
// cross HBM once at 656 bytes and no decoded copy is ever written to memory.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

constexpr int kHq = 128, kDc = 512, kDr = 64, kDqk = kDc + kDr;
constexpr int kUnitMax = 256;                   // selected rows per unit (max MMA N)
constexpr int kChunks = 9;                      // 8 latent blocks + the rotary block
constexpr int kRegion = kUnitMax * 128;         // one chunk of 256 rows: 32 KB
constexpr int kQBlk = kHq * 128;                // one 64-column block of the query: 16 KB
constexpr int kOwnQ = 5 * kRegion;              // the own query blocks follow G0..G4
constexpr int kBig = kOwnQ + 4 * kQBlk;         // 224 KB of operands
constexpr int kWork = 256;                      // gather / softmax / epilogue threads
constexpr int kThreads = kWork + 32;            // + one TMA / MMA warp
constexpr int kMaxSel = 2048;                   // selection slots per query row
constexpr int kLag = 1;                         // gather chunks in flight beyond the newest
constexpr uint32_t kColS = 0, kColO = 256, kTmemCols = 512;
constexpr int kRowFp8 = kDc + 4 * (kDc / 128) + 2 * kDr;   // 656
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t kSmemBytes = 1024 + (size_t)kBig + kUnitMax * sizeof(int32_t) +
                              32 * sizeof(uint64_t) + 64;

// chunk schedule of the CTA with output half `half`
__device__ __forceinline__ int chunk_block(int k, int half) {
    return k < 4 ? (1 - half) * 4 + k : (k == 4 ? 8 : half * 4 + (k - 5));
}
__device__ __forceinline__ int chunk_region(int k) { return k < 5 ? (k & 1) : k - 4; }
__device__ __forceinline__ int q_offset(int k) {
    return k < 5 ? 2 * kRegion + k * kQBlk : kOwnQ + (k - 5) * kQBlk;
}
// the MMA whose completion frees the region chunk k is written into
//   chunk k    0   1   2   3   4   5   6   7   8
//   waits on   -   -   0   1   2   3   1   3   4
__device__ __forceinline__ int chunk_dep(int k) {
    return k < 2 ? -1 : (k < 6 ? k - 2 : (k == 6 ? 1 : (k == 7 ? 3 : 4)));
}

struct MlaArgs {
    const __nv_bfloat16 *kv;   // bf16 rows [B, t_max, 576]
    const uint8_t *kv8;        // FP8 rows [B, t_max, 656]
    const int32_t *idx;
    __nv_bfloat16 *out;
    float *lse;
    __half *part_o;            // [units][256 / 8][128][8]  (splits > 1), unit = (row * splits + sp) * 2 + half
    float4 *part_ml;           // [units][128] (max, sum, scale of the fp16 partial, 0)
    int64_t t_max;
    int64_t start_pos;
    int S, k, splits, unit_rows;
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
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
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

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int32_t *list = reinterpret_cast<int32_t *>(sm + kBig);              // the unit's rows
    uint64_t *bars = reinterpret_cast<uint64_t *>(list + kUnitMax);
    uint64_t *chunk_full = bars;                 // [9] chunk k gathered (256 arrivals)
    uint64_t *mma_done = bars + kChunks;         // [9] chunk k's logit MMAs complete
    uint64_t *q_full = bars + 2 * kChunks;       // the query's TMA copy landed
    uint64_t *p_full = q_full + 1;               // P is in TMEM (256 arrivals)
    uint64_t *o_full = p_full + 1;               // the value mix is complete
    uint64_t *mma_fin = o_full + 1;              // every issued MMA is complete
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 24);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *scan_tmp = const_cast<int *>(abort) + 1;                         // 9 ints
    // softmax exchange (max, sum, output range of the two column halves):
    // region G0, free once the logits are complete
    float *red = reinterpret_cast<float *>(sm);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;                 // (row * splits + sp) * 2 + half
    const int half = unit & 1;
    const int sp = (unit >> 1) % a.splits;
    const int64_t row = (unit >> 1) / a.splits;
    const int64_t b = row / a.S, s = row - b * a.S;
    const int64_t limit = a.start_pos + s;
    const int U = a.unit_rows;
    const uint32_t sbase = tc::smem_u32(sm);

    if (warp == kWork / 32) {
        if (lane == 0) {
            for (int i = 0; i < kChunks; i++) {
                tc::mbar_init(&chunk_full[i], kWork);
                tc::mbar_init(&mma_done[i], 1);
            }
            tc::mbar_init(q_full, 1);
            tc::mbar_init(p_full, kWork);
            tc::mbar_init(o_full, 1);
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
        // the query's nine 64-column blocks (the own four to their own region)
        tc::mbar_arrive_expect_tx(q_full, kChunks * kQBlk);
        for (int k = 0; k < kChunks; k++)
            tc::tma_load_2d(sm + q_offset(k), &tm_q, chunk_block(k, half) * 64, (int)(row * kHq),
                            q_full);
    }
    // a kernel launched after this one (the split combine) may start its set-up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // The selections come from the preceding kernel (the top-k): wait for it
    // (a no-op without a programmatic launch), then read them with plain loads.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // valid selections of this row in slot order; this unit takes positions
    // [lo, lo + U) of that list.  Threads 0..255 hold 8 consecutive slots each.
    const int lo = sp * U;
    int n_total = 0;
    {
        constexpr int kPer = kMaxSel / kWork;
        int32_t v8[kPer];
        int cnt = 0;
#pragma unroll
        for (int e = 0; e < kPer; e++) {
            const int j = threadIdx.x * kPer + e;
            int32_t t = threadIdx.x < kWork && j < a.k ? a.idx[row * a.k + j] : -1;
            if (t >= 0 && (int64_t)t <= limit) {
                if ((int64_t)t >= a.t_max) {
                    record_error(a.err, DSA_ERR_DEVICE);
                    t = -1;
                }
            } else {
                t = -1;
            }
            v8[e] = t;
            cnt += t >= 0 ? 1 : 0;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) scan_tmp[warp] = incl;
        __syncthreads();
        int pos = incl - cnt;
#pragma unroll
        for (int w = 0; w < kThreads / 32; w++) {
            const int c = scan_tmp[w];
            if (w < warp) pos += c;
            n_total += c;
        }
#pragma unroll
        for (int e = 0; e < kPer; e++) {
            if (v8[e] < 0) continue;
            if (pos >= lo && pos < lo + U) list[pos - lo] = v8[e];
            pos++;
        }
    }
    __syncthreads();
    int n_my = n_total - lo;
    n_my = n_my < 0 ? 0 : (n_my > U ? U : n_my);
    const int64_t rbase = b * a.t_max;
    // each CTA of the unit prefetches every other row into L2 (its partner the rest)
    {
        const int j = 2 * (int)threadIdx.x + half;
        if (j < n_my) {
            if constexpr (kFp8)
                tc::prefetch_l2_bulk(a.kv8 + (rbase + list[j]) * kRowFp8, kRowFp8);
            else
                tc::prefetch_l2_bulk(a.kv + (rbase + list[j]) * kDqk, kDqk * 2);
        }
    }

    if (n_my == 0) {
        // nothing selected in this unit: an empty partial (or a zero output)
        if (threadIdx.x < kWork) {
            const int h = threadIdx.x & (kHq - 1), c = threadIdx.x >> 7;
            if (a.splits > 1) {
                uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)unit * kHq * 256) + h;
                for (int o8 = 16 * c; o8 < 16 * c + 16; o8++) po[o8 * kHq] = make_uint4(0u, 0u, 0u, 0u);
                if (c == 0) a.part_ml[(int64_t)unit * kHq + h] = make_float4(-INFINITY, 0.f, 1.f, 0.f);
            } else {
                uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + half * 256 + c * 128);
                for (int j = 0; j < 16; j++) o16[j] = make_uint4(0u, 0u, 0u, 0u);
                if (half == 0 && c == 0 && a.lse) a.lse[row * kHq + h] = -INFINITY;
            }
        }
        if (warp == kWork / 32 && lane == 0) tc::mbar_wait(q_full, 0, a.err, abort);
    } else if (warp < kWork / 32) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x;
        bool ok = true;
        int issued = 0, signalled = 0;
        // publish every chunk issued so far (before blocking on a region)
        auto publish_all = [&]() {
            cp_async_wait<0>();
            tc::fence_proxy_async_smem();
            for (; signalled < issued; signalled++) tc::mbar_arrive(&chunk_full[signalled]);
        };
        for (int k = 0; k < kChunks; k++) {
            const int dep = chunk_dep(k);
            if (dep >= 0 && !tc::mbar_test_wait(&mma_done[dep], 0)) {
                publish_all();
                if (!tc::mbar_wait(&mma_done[dep], 0, a.err, abort)) {
                    ok = false;
                    break;
                }
            }
            const int cb = chunk_block(k, half);
            const uint32_t rg = sbase + chunk_region(k) * kRegion;
            if (!kFp8 || cb == 8) {
                // 16-byte pieces straight into the swizzled tile; rows past the
                // unit's end are zero-filled (finite values times P = 0)
                for (int f = gt; f < U * 8; f += kWork) {
                    const int j = f >> 3, p = f & 7;
                    const bool v = j < n_my;
                    const int64_t t = v ? (int64_t)list[j] : 0;
                    const void *src;
                    if constexpr (kFp8)
                        src = a.kv8 + (rbase + t) * kRowFp8 + kDc + 4 * (kDc / 128) + p * 16;
                    else
                        src = a.kv + (rbase + t) * kDqk + cb * 64 + p * 8;
                    cp_async16(rg + j * 128 + ((p ^ (j & 7)) << 4), src, v ? 16u : 0u);
                }
            } else {
                // FP8 latent block cb: 16 codes per piece, decoded with the
                // block's scale into two 16-byte bf16 pieces of the tile row
                constexpr int kPer = kUnitMax * 4 / kWork;   // pieces per thread (4)
                uint4 cw[kPer];
                float sc[kPer];
#pragma unroll
                for (int u = 0; u < kPer; u++) {
                    const int f = gt + u * kWork, j = f >> 2, p = f & 3;
                    cw[u] = make_uint4(0u, 0u, 0u, 0u);
                    sc[u] = 0.f;
                    if (j < n_my) {
                        const uint8_t *r8 = a.kv8 + (rbase + list[j]) * kRowFp8;
                        cw[u] = *reinterpret_cast<const uint4 *>(r8 + cb * 64 + p * 16);
                        sc[u] = *reinterpret_cast<const float *>(r8 + kDc + 4 * (cb >> 1));
                    }
                }
#pragma unroll
                for (int u = 0; u < kPer; u++) {
                    const int f = gt + u * kWork, j = f >> 2, p = f & 3;
                    if (j >= U) continue;
                    const uint4 lo8 = decode8(cw[u].x, cw[u].y, sc[u]);
                    const uint4 hi8 = decode8(cw[u].z, cw[u].w, sc[u]);
                    st_shared_v4(rg + j * 128 + (((2 * p) ^ (j & 7)) << 4), lo8);
                    st_shared_v4(rg + j * 128 + (((2 * p + 1) ^ (j & 7)) << 4), hi8);
                }
            }
            cp_async_commit();
            issued = k + 1;
            if (issued - signalled > kLag) {
                cp_async_wait<kLag>();
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&chunk_full[signalled]);
                signalled++;
            }
        }
        publish_all();

        // ----------------------------------------------------------- softmax
        // thread (head h, column half c): logits of rows [c U/2, (c+1) U/2)
        const int q4 = warp & 3, c = warp >> 2;
        const int h = q4 * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int hc = U / 2, base = c * hc;
        if (ok && !tc::mbar_wait(&mma_done[kChunks - 1], 0, a.err, abort)) ok = false;
        tc::tc_fence_after();
        float mx = -INFINITY;
        for (int i = 0; i < hc; i += 32) {
            uint32_t r0[16], r1[16];
            tc::tmem_ld16(tmem + lane_addr + kColS + base + i, r0);
            tc::tmem_ld16(tmem + lane_addr + kColS + base + i + 16, r1);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e++) {
                if (base + i + e < n_my) mx = fmaxf(mx, __uint_as_float(r0[e]) * a.scale_log2);
                if (base + i + 16 + e < n_my) mx = fmaxf(mx, __uint_as_float(r1[e]) * a.scale_log2);
            }
        }
        red[c * kHq + h] = mx;
        tc::named_barrier(1, kWork);
        const float m = fmaxf(red[h], red[kHq + h]);       // finite: row 0 is valid
        float l = 0.f;
        for (int i = 0; i < hc; i += 32) {
            uint32_t r0[16], r1[16], pk[16];
            tc::tmem_ld16(tmem + lane_addr + kColS + base + i, r0);
            tc::tmem_ld16(tmem + lane_addr + kColS + base + i + 16, r1);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const int j0 = base + i + 2 * e;
                const float p0 = j0 < n_my ? exp2f(fmaf(__uint_as_float(r0[2 * e]), a.scale_log2, -m)) : 0.f;
                const float p1 = j0 + 1 < n_my ? exp2f(fmaf(__uint_as_float(r0[2 * e + 1]), a.scale_log2, -m)) : 0.f;
                const float p2 = j0 + 16 < n_my ? exp2f(fmaf(__uint_as_float(r1[2 * e]), a.scale_log2, -m)) : 0.f;
                const float p3 = j0 + 17 < n_my ? exp2f(fmaf(__uint_as_float(r1[2 * e + 1]), a.scale_log2, -m)) : 0.f;
                l += (p0 + p1) + (p2 + p3);
                const __nv_bfloat162 v01 = __floats2bfloat162_rn(p0, p1);
                const __nv_bfloat162 v23 = __floats2bfloat162_rn(p2, p3);
                pk[e] = *reinterpret_cast<const uint32_t *>(&v01);
                pk[8 + e] = *reinterpret_cast<const uint32_t *>(&v23);
            }
            // P of rows [base + i, base + i + 32) over the logits already read
            tc::tmem_st16(tmem + lane_addr + kColS + base + i / 2, pk);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(p_full);
        red[2 * kHq + c * kHq + h] = l;
        tc::named_barrier(1, kWork);
        const float lt = red[2 * kHq + h] + red[3 * kHq + h];

        // ---------------------------------------------------------- epilogue
        // thread (h, c) writes output columns [128c, 128c + 128) of this CTA's 256
        if (ok && !tc::mbar_wait(o_full, 0, a.err, abort)) ok = false;
        tc::tc_fence_after();
        const uint32_t ocol = tmem + lane_addr + kColO + c * 128;
        if (a.splits > 1) {
            // O / (l * sc) in fp16, sc the power of two that keeps |O / l| / sc
            // <= 2^14, as [column / 8][head] groups of eight halves
            float amax = 0.f;
            for (int j = 0; j < 128; j += 16) {
                uint32_t o[16];
                tc::tmem_ld16(ocol + j, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e++) amax = fmaxf(amax, fabsf(__uint_as_float(o[e])));
            }
            red[4 * kHq + c * kHq + h] = amax;
            tc::named_barrier(1, kWork);
            amax = fmaxf(red[4 * kHq + h], red[5 * kHq + h]);
            const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
            float scl = 1.f;
            while (amax * inv_l > 16384.f * scl) scl *= 2.f;
            const float inv = inv_l / scl;
            uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)unit * kHq * 256) + h;
            for (int j = 0; j < 128; j += 16) {
                uint32_t o[16], w[8];
                tc::tmem_ld16(ocol + j, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const __half2 v = __floats2half2_rn(__uint_as_float(o[2 * e]) * inv,
                                                        __uint_as_float(o[2 * e + 1]) * inv);
                    w[e] = *reinterpret_cast<const uint32_t *>(&v);
                }
                if (ok) {
                    const int o8 = (c * 128 + j) / 8;
                    po[o8 * kHq] = make_uint4(w[0], w[1], w[2], w[3]);
                    po[(o8 + 1) * kHq] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (ok && c == 0) a.part_ml[(int64_t)unit * kHq + h] = make_float4(m, lt, scl, 0.f);
        } else {
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + half * 256 + c * 128);
            for (int j = 0; j < 128; j += 16) {
                uint32_t o[16], w[8];
                tc::tmem_ld16(ocol + j, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                                   __uint_as_float(o[2 * e + 1]) * inv);
                    w[e] = *reinterpret_cast<const uint32_t *>(&v);
                }
                if (ok) {
                    o16[j / 8] = make_uint4(w[0], w[1], w[2], w[3]);
                    o16[j / 8 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (ok && half == 0 && c == 0 && a.lse)
                a.lse[row * kHq + h] = lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
        }
    } else if (lane == 0) {
        // ------------------------------------------------------ TMA / MMA
        const uint32_t id_qk = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, U);
        const uint32_t id_pv = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, 256, true);
        bool ok = tc::mbar_wait(q_full, 0, a.err, abort);
        for (int k = 0; ok && k < kChunks; k++) {
            if (!tc::mbar_wait(&chunk_full[k], 0, a.err, abort)) {
                ok = false;
                break;
            }
            tc::tc_fence_after();
            const uint32_t qa = sbase + q_offset(k), ca = sbase + chunk_region(k) * kRegion;
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                const uint64_t ad = tc::smem_desc(qa + ks * 32, 1024, tc::kSwizzle128B);
                const uint64_t bd = tc::smem_desc(ca + ks * 32, 1024, tc::kSwizzle128B);
                tc::mma_f16(tmem + kColS, ad, bd, id_qk, k > 0 || ks > 0);
            }
            tc::tc_commit(&mma_done[k]);
        }
        if (ok && tc::mbar_wait(p_full, 0, a.err, abort)) {
            tc::tc_fence_after();
            // O += P C[:, own 256]: K-step ks covers rows [16 ks, 16 ks + 16),
            // whose P sits in the first quarter of its column half
            const int hc = U / 2;
            for (int ks = 0; ks < U / 16; ks++) {
                const int r0 = 16 * ks, c = r0 / hc;
                const uint32_t pa = tmem + kColS + c * hc + (r0 - c * hc) / 2;
                const uint64_t bd = tc::smem_desc(sbase + kRegion + ks * 2048, 1024,
                                                  tc::kSwizzle128B, kRegion);
                tc::mma_f16_ts(tmem + kColO, pa, bd, id_pv, ks > 0);
            }
            tc::tc_commit(o_full);
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

// Merges the splits of each (row, half): with w_s = 2^(m_s - m) l_s and the
// stored partials Y_s = O_s / (l_s sc_s), out = sum_s w_s sc_s Y_s / sum_s w_s.
// The partials are [column / 8][head] groups of eight halves; thread (head,
// octet) merges eight output columns of one head, consecutive threads
// consecutive heads (coalesced).
__global__ void __launch_bounds__(kHq)
sparse_mla_combine_kernel(const __half *part_o, const float4 *part_ml, int splits,
                          __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    // the partials come from the preceding kernel: wait for it (plain loads below)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int groups = 256 / 8;
    const int64_t rh = blockIdx.x / groups;                 // row * 2 + half
    const int64_t row = rh >> 1;
    const int half = (int)(rh & 1);
    const int h = threadIdx.x;
    const int c8 = (int)(blockIdx.x % groups);
    // partial of split sp: unit (row * splits + sp) * 2 + half
    const int64_t u0 = row * splits * 2 + half;
    float m = -INFINITY;
    for (int sp = 0; sp < splits; sp++) m = fmaxf(m, part_ml[(u0 + 2 * sp) * kHq + h].x);
    float L = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // four splits at a time, so that their loads are in flight together
    for (int sp0 = 0; sp0 < splits; sp0 += 4) {
        float4 ml[4];
        uint4 x[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int sp = sp0 + u;
            ml[u] = sp < splits ? part_ml[(u0 + 2 * sp) * kHq + h] : make_float4(-INFINITY, 0.f, 1.f, 0.f);
            if (sp < splits)
                x[u] = reinterpret_cast<const uint4 *>(part_o + (u0 + 2 * sp) * kHq * 256)[c8 * kHq + h];
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
            if (ml[u].x == -INFINITY) continue;
            const float w = exp2f(ml[u].x - m) * ml[u].y;
            L += w;
            const float ws = w * ml[u].z;
            const uint32_t xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&xs[e]));
                acc[2 * e] += ws * f.x;
                acc[2 * e + 1] += ws * f.y;
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint32_t w8[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        w8[e] = *reinterpret_cast<const uint32_t *>(&v);
    }
    reinterpret_cast<uint4 *>(out + (row * kHq + h) * kDc + half * 256)[c8] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
    if (half == 0 && c8 == 0 && lse) lse[row * kHq + h] = L > 0.f ? (m + log2f(L)) * kLn2 : -INFINITY;
}

// Rows per unit: the smallest of 64, 128, 192, 256 whose units (two CTAs
// each) fit on the SMs at once; 256 when none does.
int mla_unit_rows(int64_t rows, int k) {
    for (int u = 64; u <= kUnitMax; u += 64)
        if (rows * 2 * ((k + u - 1) / u) <= num_sms()) return u;
    return kUnitMax;
}

size_t workspace_bytes(int64_t rows, int k) {
    const int u = mla_unit_rows(rows, k);
    const int sp = (k + u - 1) / u;
    if (sp <= 1) return 0;
    const int64_t units = rows * 2 * sp;
    return align_up((size_t)units * kHq * 256 * sizeof(__half), 256) +
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
    a.kv = kFp8 ? nullptr : static_cast<const __nv_bfloat16 *>(kv);
    a.kv8 = kFp8 ? static_cast<const uint8_t *>(kv) : nullptr;
    a.idx = idx;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.t_max = t_max;
    a.start_pos = start_pos;
    a.S = S;
    a.k = k;
    a.unit_rows = mla_unit_rows(rows, k);
    a.splits = (k + a.unit_rows - 1) / a.unit_rows;
    a.scale_log2 = sm_scale * kLog2e;
    a.err = device_error_word();
    if (a.splits > 1) {
        const int64_t units = rows * 2 * a.splits;
        a.part_o = static_cast<__half *>(ws);
        a.part_ml = reinterpret_cast<float4 *>(static_cast<char *>(ws) +
                                               align_up((size_t)units * kHq * 256 * sizeof(__half), 256));
    }
    if (cudaFuncSetAttribute(sparse_mla_tc_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * a.splits * 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    // programmatic launch: the kernel's set-up overlaps the preceding kernel's
    // tail; it waits for that kernel before reading the selections
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, sparse_mla_tc_kernel<kFp8>, tm_q, a) != cudaSuccess)
        return DSA_ERR_CUDA;
    dsa_status st = launch_status();
    if (st != DSA_OK || a.splits == 1) return st;
    cudaLaunchConfig_t ccfg = {};
    ccfg.gridDim = dim3((unsigned)(rows * 2 * (256 / 8)));
    ccfg.blockDim = dim3(kHq);
    ccfg.stream = stream;
    cudaLaunchAttribute cattr[1];
    cattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    cattr[0].val.programmaticStreamSerializationAllowed = 1;
    ccfg.attrs = cattr;
    ccfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&ccfg, sparse_mla_combine_kernel, (const __half *)a.part_o,
                           (const float4 *)a.part_ml, a.splits, a.out, lse) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
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
