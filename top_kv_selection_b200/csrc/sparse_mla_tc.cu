// sparse_mla_tc.cu -- tensor-core sparse latent attention (bf16, V3.2 shapes).
//
// Pages: the diagram "DeepSeek Sparse Attention, one decode step in one layer
// (V3.2 sizes)" (core attention in MQA mode: 128 heads over the gathered
// 576-wide latent rows, each row key and value) and the MLA prefill excerpt
// of "DeepSeek-V3.2-Exp - Causal mask" (index mask + causal mask, softmax,
// value mix).
//
// Shapes: Hq = 128 heads (the MMA M), rows [c (512) | k_pe (64)] bf16.
// A cluster of two CTAs computes one query row over one share ("split") of
// its selected rows.  CTA r of the pair owns
//   - columns [256r, 256r + 320) of the query and of every gathered row
//     (five 64-column blocks; block 4 of CTA 0 and block 0 of CTA 1 are the
//     same columns 256..319),
//   - the logit contraction over columns [288r, 288r + 288), i.e. half of
//     q . [c | k_pe], and
//   - output columns [256r, 256r + 256).
// Per tile of 64 gathered rows:
//   warps 5..8  gather the CTA's 640 bytes of each row with 16-byte cp.async
//               straight into the 128B-swizzled K-major layout (a 2-stage
//               ring; a tile is published two tiles later, or at once before
//               the producer would block);
//   warp 0      S_r = Q_r C_r^T: 18 tcgen05.mma kind::f16 (M=128, N=64, K=16)
//               with both operands in shared memory; O += P C[:, own 256]:
//               4 MMAs (N=256, K=16) with A = P from TMEM and B = the same
//               shared tile read as an MN-major operand.  The previous tile's
//               PV is slotted between this tile's QK blocks once its P is
//               ready;
//   warps 1..4  one thread per head: read the partial logits S_r from TMEM,
//               send them to the partner CTA's shared memory (DSMEM), add
//               the partner's (S_0 + S_1 in both CTAs: the same bits, since
//               fp32 addition commutes), then the online softmax in the exp2
//               domain with lazy rescaling (the TMEM accumulator is rescaled
//               only when a head's running max grows by more than 8), P to
//               TMEM as bf16, and the epilogue.
// Both CTAs run the same softmax on the same logits, so their P, running max
// and sum agree exactly; each accumulates its own half of the output.
// TMEM: O 256 | S 2 x 64 | P 2 x 32 columns.
// With several splits per row, each split's output normalised by its own sum
// and divided by a power of two that keeps it below 2^14 (fp16: an 11-bit
// significand, finer than the bf16 result), with its (max, sum, power of two),
// goes to the workspace, and a combine kernel merges them.
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

constexpr int kHq = 128, kDc = 512, kDr = 64, kDqk = kDc + kDr;
constexpr int kLB = 5;                          // 64-column blocks held per CTA
constexpr int kDh = 256;                        // output columns per CTA
constexpr int kRows = 64;                       // gathered rows per tile (QK N)
constexpr int kStages = 3;
constexpr int kThreads = 288;               // warp 0 MMA, 1..4 softmax, 5..8 gather
constexpr int kMaxSel = 2048;                   // selection slots held in shared memory
// TMEM columns: O (fp32) | S (fp32) | P (bf16 pairs) | Q (bf16 pairs, this CTA's 320)
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352, kTmemCols = 512;
static_assert(kColQ + kLB * 64 / 2 == kTmemCols, "the query fills the last TMEM columns");
constexpr int kBlk = kRows * 128;               // bytes of one column block of a tile
constexpr int kTileBytes = kLB * kBlk;          // 40960
constexpr int kChunks = kLB * 8;                // 16-byte pieces of a row per CTA: 40
constexpr int kRxBytes = kHq * kRows * 4;       // partner's partial logits
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kTileBytes + 2 * kRxBytes +
                              kMaxSel * sizeof(int32_t) + 32 * sizeof(uint64_t) + 64;
constexpr int kQStage = 1;                       // the query is staged in ring stages 1..2
static_assert(kQStage + 2 <= kStages, "query staging");
constexpr int kLag = 1;                          // gather tiles in flight per thread beyond the one issued
constexpr int kQBlk = kHq * 128;                 // one 64-column block of the query (TMA box)

struct MlaArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *kv;
    const int32_t *idx;
    __nv_bfloat16 *out;
    float *lse;
    __half *part_o;     // [units][256 / 8][128][8]  (splits > 1), unit = (row * splits + sp) * 2 + r
    float4 *part_ml;    // [units][128] (max, sum, scale of the fp16 partial, 0)
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

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sc = smem;                                      // C tiles
    // this CTA's partial logits to send, and the partner's received: [16][128] float4
    float4 *tx = reinterpret_cast<float4 *>(sc + kStages * kTileBytes);
    float4 *rx = tx + kRxBytes / 16;
    int32_t *list = reinterpret_cast<int32_t *>(sc + kStages * kTileBytes + 2 * kRxBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(list + kMaxSel);
    uint64_t *c_full = bars, *c_empty = bars + kStages;
    uint64_t *s_full = bars + 2 * kStages, *s_empty = s_full + 1;
    uint64_t *p_full = s_empty + 1, *pv_done = p_full + 1;
    uint64_t *q_ready = pv_done + 1;    // the query is in TMEM
    uint64_t *q_full = q_ready + 1;     // the query's TMA copy (ring stages 2..3) landed
    uint64_t *q_free = q_full + 1;      // ... and has been moved to TMEM
    uint64_t *rx_full = q_free + 1;     // partner's logits of the current tile landed (bytes)
    uint64_t *tx_ok = rx_full + 1;      // partner has read what this CTA sent last
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tx_ok + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *scan_tmp = const_cast<int *>(abort) + 1;            // 10 ints

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;                             // (row * splits + sp) * 2 + r
    const int cr = unit & 1;                                 // rank in the pair
    const int sp = (unit >> 1) % a.splits;
    const int64_t row = (unit >> 1) / a.splits;
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
        tc::mbar_init(s_full, 1);
        tc::mbar_init(s_empty, 128);
        tc::mbar_init(p_full, 128);
        tc::mbar_init(pv_done, 1);
        tc::mbar_init(q_ready, 128);
        tc::mbar_init(q_full, 1);
        tc::mbar_init(q_free, 128);
        tc::mbar_init(rx_full, 1);
        tc::mbar_init(tx_ok, 1);
        *abort = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tm_q);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_holder, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    tc::cluster_sync_all();          // both CTAs' barriers exist before any remote arrive
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // a kernel launched after this one (the split combine) may start its set-up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        // this CTA's five 64-column blocks of the query, staged in ring
        // stages 1..2 until the softmax warps have moved them to TMEM
        tc::mbar_arrive_expect_tx(q_full, kLB * kQBlk);
        for (int j = 0; j < kLB; j++)
            tc::tma_load_2d(sc + kQStage * kTileBytes + j * kQBlk, &tm_q, (cr * 4 + j) * 64,
                            (int)(row * kHq), q_full);
    }

    // The selections come from the preceding kernel (the top-k): wait for it
    // to complete (a no-op without a programmatic launch), then read them with
    // plain loads, which stay after the wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // valid selections of this row, in slot order (the same list in both CTAs):
    // threads 0..255 take 8 consecutive slots each, one block-wide scan
    constexpr int kPer = kMaxSel / 256;
    int32_t v8[kPer];
    int cnt = 0;
#pragma unroll
    for (int e = 0; e < kPer; e++) {
        const int j = threadIdx.x * kPer + e;
        int32_t t = threadIdx.x < 256 && j < a.k ? a.idx[row * a.k + j] : -1;
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
    int n = 0, pos = incl - cnt;
#pragma unroll
    for (int w = 0; w < 8; w++) {
        const int c = scan_tmp[w];
        if (w < warp) pos += c;
        n += c;
    }
#pragma unroll
    for (int e = 0; e < kPer; e++)
        if (v8[e] >= 0) list[pos++] = v8[e];
    __syncthreads();
    // this split's tiles of 64 rows
    const int nt_all = (n + kRows - 1) / kRows;
    const int t_lo = (int)((int64_t)sp * nt_all / a.splits);
    const int t_hi = (int)((int64_t)(sp + 1) * nt_all / a.splits);
    const int lo = t_lo * kRows;
    const int n_my = (t_hi * kRows < n ? t_hi * kRows : n) - lo;
    const int n_tiles = t_hi - t_lo;

    // the query (this CTA's 320 columns, two bf16 per TMEM column) moves from
    // its staging copy to TMEM, one head per lane, by the softmax warps
    if (is_softmax) {
        if (tc::mbar_wait(q_full, 0, a.err, abort)) {
            const uint8_t *qs = sc + kQStage * kTileBytes;
#pragma unroll 1
            for (int c = 0; c < kLB * 8 / 4; c++) {          // 10 x 4 pieces of 16 bytes
                uint32_t r[16];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int piece = 4 * c + u, blk = piece >> 3, ch = piece & 7;
                    const uint4 v = *reinterpret_cast<const uint4 *>(
                        qs + blk * kQBlk + h * 128 + ((ch ^ (h & 7)) << 4));
                    r[4 * u] = v.x; r[4 * u + 1] = v.y; r[4 * u + 2] = v.z; r[4 * u + 3] = v.w;
                }
                tc::tmem_st16(tmem + lane_addr + kColQ + c * 16, r);
            }
            tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::mbar_arrive(q_ready);
        tc::mbar_arrive(q_free);
    }

    if (n_tiles == 0) {                                      // nothing selected here
        if (is_softmax) {
            if (a.splits > 1) {
                uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)unit * kHq * kDh) + h;
                for (int c = 0; c < kDh / 8; c++) po[c * kHq] = make_uint4(0u, 0u, 0u, 0u);
                a.part_ml[(int64_t)unit * kHq + h] = make_float4(-INFINITY, 0.f, 1.f, 0.f);
            } else {
                __nv_bfloat16 *o = a.out + (row * kHq + h) * kDc + cr * kDh;
                for (int c = 0; c < kDh; c++) o[c] = __float2bfloat16_rn(0.f);
                if (cr == 0 && a.lse) a.lse[row * kHq + h] = -INFINITY;
            }
        }
    } else if (warp >= 5) {
        // ---- gather: the 128 threads copy the tile's 64 x 40 pieces of 16
        // bytes, consecutive threads consecutive pieces of a row
        const int gt = threadIdx.x - 160;
        const int64_t rbase = b * a.t_max;
        const __nv_bfloat16 *kv_cols = a.kv + cr * kDh;     // this CTA's first column
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
            if (i == kQStage && !tc::mbar_wait(q_free, 0, a.err, abort)) break;   // the query's staging
            uint8_t *tile = sc + st * kTileBytes;
#pragma unroll 4
            for (int f = gt; f < kRows * kChunks; f += 128) {
                const int j = f / kChunks, c = f - j * kChunks;
                int r = i * kRows + j;
                if (r >= n_my) r = n_my - 1;                 // padding: a valid row
                const __nv_bfloat16 *src = kv_cols + (rbase + list[lo + r]) * kDqk;
                cp_async16(tile + (c >> 3) * kBlk + j * 128 + (((c & 7) ^ (j & 7)) << 4), src + c * 8);
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
        // publish the remaining tiles in order, each as soon as it has landed
        for (; signalled < issued; signalled++) {
            if (issued - signalled - 1 >= 1) cp_async_wait<1>();
            else cp_async_wait<0>();
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&c_full[signalled % kStages]);
        }
    } else if (warp == 0) {
        if (lane == 0) {
            const uint32_t id_qk = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, kRows);
            const uint32_t id_pv = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 128, kDh, true);
            const uint32_t sc_addr = tc::smem_u32(sc);
            // this CTA's K steps (16 columns each) of the logit contraction:
            // 18 of the 20 in its five blocks
            const int ks_first = cr == 0 ? 0 : 2, ks_last = cr == 0 ? 4 * kLB - 2 : 4 * kLB;
            bool ok = tc::mbar_wait(q_ready, 0, a.err, abort);
            // O += P C[:, own 256] for tile j (P(j) must be published)
            auto pv_issue = [&](int j) {
                const int st = j % kStages;
                tc::tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kRows / 16; ks++) {
                    const uint64_t bd = tc::smem_desc(sc_addr + st * kTileBytes + ks * 2048, 1024,
                                                      tc::kSwizzle128B, kBlk);
                    tc::mma_f16_ts(tmem + kColO, tmem + kColP + ks * 8, bd, id_pv, j > 0 || ks > 0);
                }
                tc::tc_commit(&c_empty[st]);
                tc::tc_commit(pv_done);
            };
            // S_r = Q_r C_r^T for tile i, A = Q from TMEM; the PV of the previous
            // tile (pend >= 0) is slotted in as soon as its P is published
            auto qk = [&](int i, int pend) -> bool {
                const int st = i % kStages;
                if (!tc::mbar_wait(&c_full[st], (uint32_t)(i / kStages) & 1u, a.err, abort)) return false;
                if (!tc::mbar_wait(s_empty, ((uint32_t)i & 1u) ^ 1u, a.err, abort)) return false;
                tc::tc_fence_after();
#pragma unroll 1
                for (int kk = ks_first; kk < ks_last; kk++) {
                    if ((kk & 3) == 0 && pend >= 0 &&
                        tc::mbar_test_wait(p_full, (uint32_t)pend & 1u)) {
                        pv_issue(pend);
                        pend = -1;
                    }
                    const int cb = kk >> 2, ks = kk & 3;
                    const uint64_t bd = tc::smem_desc(sc_addr + st * kTileBytes + cb * kBlk + ks * 32,
                                                      1024, tc::kSwizzle128B);
                    tc::mma_f16_ts(tmem + kColS, tmem + kColQ + kk * 8, bd, id_qk, kk != ks_first);
                }
                tc::tc_commit(s_full);
                if (pend >= 0) {
                    if (!tc::mbar_wait(p_full, (uint32_t)pend & 1u, a.err, abort)) return false;
                    pv_issue(pend);
                }
                return true;
            };
            if (ok) ok = qk(0, -1);
            for (int i = 1; ok && i < n_tiles; i++) ok = qk(i, i - 1);
            if (ok && tc::mbar_wait(p_full, (uint32_t)(n_tiles - 1) & 1u, a.err, abort))
                pv_issue(n_tiles - 1);
        }
    } else {
        // ---- softmax warps
        // Per tile the 128 threads write this CTA's partial logits to `tx`, and
        // one thread (the elected) pushes the 32 KB into the partner's `rx` with
        // a bulk copy counted on the partner's rx_full; after reading `rx` the
        // elected thread tells the partner (tx_ok) that it may send again,
        // which also means this CTA's previous copy has landed.
        const uint32_t peer = (uint32_t)(cr ^ 1);
        const uint32_t peer_rx = tc::map_shared_rank(rx, peer);
        const uint32_t peer_rx_full = tc::map_shared_rank(rx_full, peer);
        const uint32_t peer_tx_ok = tc::map_shared_rank(tx_ok, peer);
        const bool elected = threadIdx.x == 32;
        float m_run = -INFINITY, l = 0.f;
        // A failed (timed-out) wait only clears `ok`: the thread carries on to the
        // next named barrier, where all 128 threads leave the loop together.
        bool ok = true;
        for (int i = 0; i < n_tiles; i++) {
            if (elected) tc::mbar_arrive_expect_tx(rx_full, kRxBytes);   // tile i's bytes
            if (ok && !tc::mbar_wait(s_full, (uint32_t)i & 1u, a.err, abort)) ok = false;
            tc::tc_fence_after();
            uint32_t own[kRows];
#pragma unroll
            for (int q = 0; q < kRows / 16; q++)
                tc::tmem_ld16(tmem + lane_addr + kColS + q * 16,
                              *reinterpret_cast<uint32_t(*)[16]>(own + q * 16));
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(s_empty);
            // `tx` may be rewritten once the partner has read tile i-1
            if (ok && i > 0 && !tc::mbar_wait_cluster(tx_ok, (uint32_t)(i - 1) & 1u, a.err, abort))
                ok = false;
#pragma unroll
            for (int q = 0; q < kRows / 4; q++)
                tx[q * kHq + h] = make_float4(__uint_as_float(own[4 * q]), __uint_as_float(own[4 * q + 1]),
                                              __uint_as_float(own[4 * q + 2]), __uint_as_float(own[4 * q + 3]));
            tc::fence_proxy_async_smem();
            if (tc::named_barrier_any(1, 128, !ok)) break;
            if (elected) tc::bulk_copy_to_peer(peer_rx, tx, kRxBytes, peer_rx_full);
            if (ok && !tc::mbar_wait(rx_full, (uint32_t)i & 1u, a.err, abort)) ok = false;
            const int nv = n_my - i * kRows;
            float sv[kRows];
            float m_tile = -INFINITY;
#pragma unroll
            for (int q = 0; q < kRows / 4; q++) {
                const float4 o = rx[q * kHq + h];
                const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int j = 4 * q + e;
                    const float lg = __uint_as_float(own[j]) + ov[e];   // S_0 + S_1 in either CTA
                    sv[j] = j < nv ? lg * a.scale_log2 : -INFINITY;
                    m_tile = fmaxf(m_tile, sv[j]);
                }
            }
            if (tc::named_barrier_any(1, 128, !ok)) break;      // every thread has read `rx`
            if (elected) tc::mbar_arrive_cluster(peer_tx_ok);
            // PV(i-1) must be done: it reads P, and O may be rescaled below
            if (i > 0) {
                if (ok && !tc::mbar_wait(pv_done, (uint32_t)(i - 1) & 1u, a.err, abort)) ok = false;
                tc::tc_fence_after();
            }
            if (__any_sync(0xffffffffu, m_tile > m_run + 8.f)) {
                const float m_new = fmaxf(m_run, m_tile);
                const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
                if (i > 0) {
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
            uint32_t pk[kRows / 2];
#pragma unroll
            for (int c = 0; c < kRows / 2; c++) {
                const float p0 = exp2f(sv[2 * c] - m_run), p1 = exp2f(sv[2 * c + 1] - m_run);
                l += p0 + p1;
                const __nv_bfloat162 v = __floats2bfloat162_rn(p0, p1);
                pk[c] = *reinterpret_cast<const uint32_t *>(&v);
            }
            tc::tmem_st16(tmem + lane_addr + kColP, *reinterpret_cast<uint32_t(*)[16]>(pk));
            tc::tmem_st16(tmem + lane_addr + kColP + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(p_full);
        }
        if (ok && tc::mbar_wait(pv_done, (uint32_t)(n_tiles - 1) & 1u, a.err, abort)) {
            tc::tc_fence_after();
            if (a.splits > 1) {
                // O / (l * sc) as [column / 8][head] groups of eight halves (a
                // warp stores 512 contiguous bytes), sc the power of two that
                // keeps |O / l| / sc <= 2^14 (a first pass finds max |O|)
                float amax = 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < kDh; c0 += 16) {
                    uint32_t o[16];
                    tc::tmem_ld16(tmem + lane_addr + kColO + c0, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) amax = fmaxf(amax, fabsf(__uint_as_float(o[e])));
                }
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                float sc = 1.f;
                while (amax * inv_l > 16384.f * sc) sc *= 2.f;
                const float inv = inv_l / sc;
                uint4 *po = reinterpret_cast<uint4 *>(a.part_o + (int64_t)unit * kHq * kDh) + h;
#pragma unroll 1
                for (int c0 = 0; c0 < kDh; c0 += 16) {
                    uint32_t o[16], w[8];
                    tc::tmem_ld16(tmem + lane_addr + kColO + c0, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        const __half2 v = __floats2half2_rn(__uint_as_float(o[2 * e]) * inv,
                                                            __uint_as_float(o[2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    po[(c0 / 8) * kHq] = make_uint4(w[0], w[1], w[2], w[3]);
                    po[(c0 / 8 + 1) * kHq] = make_uint4(w[4], w[5], w[6], w[7]);
                }
                a.part_ml[(int64_t)unit * kHq + h] = make_float4(m_run, l, sc, 0.f);
            } else {
                const float inv = l > 0.f ? 1.f / l : 0.f;
                uint4 *o16 = reinterpret_cast<uint4 *>(a.out + (row * kHq + h) * kDc + cr * kDh);
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
                if (cr == 0 && a.lse) a.lse[row * kHq + h] = l > 0.f ? (m_run + log2f(l)) * kLn2 : -INFINITY;
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
    tc::cluster_sync_all();          // the partner no longer touches this CTA's shared memory
}

// Merges the splits of each (row, half): with w_s = 2^(m_s - m) l_s and the
// stored partials Y_s = O_s / (l_s sc_s), out = sum_s w_s sc_s Y_s / sum_s w_s.
// The partials are [column / 8][head] groups of eight halves; thread (head,
// octet) merges eight output columns of one head, consecutive threads
// consecutive heads (coalesced).
constexpr int kCombineOcts = 1;                          // column octets per block
__global__ void __launch_bounds__(kHq * kCombineOcts)
sparse_mla_combine_kernel(const __half *part_o, const float4 *part_ml, int splits,
                          __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    // the partials come from the preceding kernel: wait for it (plain loads below)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int groups = (kDh / 8) / kCombineOcts;
    const int64_t rh = blockIdx.x / groups;                 // row * 2 + half
    const int64_t row = rh >> 1;
    const int half = (int)(rh & 1);
    const int h = threadIdx.x % kHq;
    const int c8 = (int)(blockIdx.x % groups) * kCombineOcts + threadIdx.x / kHq;
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
                x[u] = reinterpret_cast<const uint4 *>(part_o + (u0 + 2 * sp) * kHq * kDh)[c8 * kHq + h];
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
    reinterpret_cast<uint4 *>(out + (row * kHq + h) * kDc + half * kDh)[c8] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
    if (half == 0 && c8 == 0 && lse) lse[row * kHq + h] = L > 0.f ? (m + log2f(L)) * kLn2 : -INFINITY;
}

// Splits per row: as many pairs as fill the SMs once, then as few as give the
// same number of tiles to the busiest split (fewer partials to combine).
int mla_splits(int64_t rows, int k) {
    const int64_t tiles = (k + kRows - 1) / kRows;
    int64_t sp = num_sms() / (rows * 2);
    if (sp > tiles) sp = tiles;
    if (sp < 1) return 1;
    const int64_t per = (tiles + sp - 1) / sp;
    return (int)((tiles + per - 1) / per);
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
    return align_up((size_t)units * kHq * kDh * sizeof(__half), 256) +
           (size_t)units * kHq * sizeof(float4);
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
        a.part_o = static_cast<__half *>(ws);
        a.part_ml = reinterpret_cast<float4 *>(static_cast<char *>(ws) +
                                               align_up((size_t)units * kHq * kDh * sizeof(__half), 256));
    }
    if (cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * a.splits * 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    // programmatic launch: the kernel's set-up overlaps the preceding kernel's
    // tail; it waits for that kernel before reading the selections
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, sparse_mla_tc_kernel, tm_q, a) != cudaSuccess) return DSA_ERR_CUDA;
    dsa_status st = launch_status();
    if (st != DSA_OK || a.splits == 1) return st;
    cudaLaunchConfig_t ccfg = {};
    ccfg.gridDim = dim3((unsigned)(rows * 2 * ((kDh / 8) / kCombineOcts)));
    ccfg.blockDim = dim3(kHq * kCombineOcts);
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

}  // namespace dsa
