// topk.cu -- per-query top-k selection over the causal positions.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward, top-k
// step: each query keeps the positions of its min(index_topk, end_pos)
// largest index scores, after the causal mask of "DeepSeek-V3.2-Exp - Causal
// mask" (Transformer.forward) has set the future positions to -inf.
// Rows with fewer causal positions than K are padded with -1 (the warm-up
// sentinel of the DeepSeek-V4 mask visualiser) instead of masked positions.
//
// Contract: row (b, s) selects the m = min(K, n_valid) largest scores among
// positions t < n_valid = min(T, start_pos + s + 1), ties going to the lower
// position, and writes them in ascending position order.  This is the same as
// finding tau = the m-th largest value and q = m - #(x > tau), then taking
// every x > tau plus the first q positions with x == tau.
//
// Cluster kernel (rows up to ~300K positions): a thread-block cluster of CN
// CTAs owns one row; CTA p keeps the scores of positions [p*L, (p+1)*L) in
// shared memory.  tau is found in rounds whose histograms are merged through
// distributed shared memory by CTA 0, which broadcasts the decision:
//   round 0: 2048 bins linear in value between the row's finite min and max
//            (well spread for smooth score distributions, so shared-memory
//            atomics rarely collide and the threshold bin is small), merged
//            into CTA 0 with distributed shared-memory atomics;
//   then the threshold-bin candidates' keys are gathered into CTA 0, which
//   finds the exact k-th key alone (by ranking every key directly when there
//   are at most 1024 of them, else 11 + 11 + 10-bit radix passes); if there
//   are too many candidates, the radix passes run cluster-wide instead.
// Then every CTA counts its x > tau and x == tau, the counts are exchanged,
// and each CTA writes its selected positions at its offset in position order.
// Cluster barriers are hardware barriers between co-scheduled CTAs.
//
// Fallback kernel (longer rows): one CTA per row, four 8-bit radix passes
// over the row in global memory, then the same ordered compaction.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxSlice = 28672;     // scores per CTA kept in shared memory

// Block-wide exclusive scan of a 0/1 flag; *total receives the block total.
// All threads must call it.
__device__ __forceinline__ int block_scan_flag(bool flag, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned ballot = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
        int v = lane < kWarps ? warp_tot[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane < kWarps) warp_tot[lane] = incl - v;
        if (lane == 31) warp_tot[32] = incl;
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    *total = warp_tot[32];
    __syncthreads();
    return r;
}

// Block-wide exclusive scan of an int; *total receives the block total.
__device__ __forceinline__ int block_scan_int(int v, int *tmp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = lane < kWarps ? tmp[lane] : 0;
        int wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kWarps) tmp[lane] = wi - wv;
        if (lane == 31) tmp[32] = wi;
    }
    __syncthreads();
    const int r = tmp[warp] + incl - v;
    *total = tmp[32];
    __syncthreads();
    return r;
}

// Block-wide sum of an int (result in every thread).
__device__ __forceinline__ int block_sum(int v, int *tmp) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) tmp[threadIdx.x >> 5] = v;
    __syncthreads();
    int r = 0;
    for (int w = 0; w < kWarps; w++) r += tmp[w];
    __syncthreads();
    return r;
}

// Finds, in a histogram of `nb` bins counted from the top, the bin where the
// running count reaches `rank` (1-based); returns the bin and the rank left
// inside it.  Executed by the whole block; `hist` is in shared memory.
__device__ __forceinline__ void find_rank_bin(const unsigned *hist, int nb, unsigned rank,
                                              unsigned *out_bin, unsigned *out_rank,
                                              unsigned *scan_tmp) {
    // inclusive suffix sums over bins, in chunks of kThreads bins from the top
    unsigned above = 0;
    for (int base = nb - 1; base >= 0; base -= kThreads) {
        const int bin = base - (int)threadIdx.x;
        unsigned v = bin >= 0 ? hist[bin] : 0u;
        // inclusive scan in thread order (= descending bins)
        unsigned incl = v;
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane == 31) scan_tmp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            unsigned wv = scan_tmp[lane];
            unsigned wi = wv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned n = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += n;
            }
            scan_tmp[lane] = wi - wv;       // exclusive prefix of warp totals
            if (lane == 31) scan_tmp[32] = wi;
        }
        __syncthreads();
        const unsigned before = above + scan_tmp[warp] + incl - v;   // count strictly above bin
        if (bin >= 0 && before < rank && before + v >= rank) {
            *out_bin = (unsigned)bin;
            *out_rank = rank - before;
        }
        above += scan_tmp[32];
        __syncthreads();
        if (above >= rank) break;
    }
    __syncthreads();
}

__device__ __forceinline__ int linear_bin(float x, float lo, float scale) {
    if (!(x >= lo)) return 0;                       // NaN, -inf
    const float t = __fmul_rn(__fsub_rn(x, lo), scale);
    return t >= (float)(kBins - 1) ? kBins - 1 : (int)t;
}

struct ClusterCtl {
    float lo, hi;           // this CTA's finite min / max
    unsigned bin, rank;     // broadcast by CTA 0
    int n_cand;             // this CTA's threshold-bin candidates
    int n_gt, n_eq;         // this CTA's counts of x > tau, x == tau
};

// Slice element i lives at sv[pad(i)]: one spare word every 32 keeps the
// per-thread contiguous segments (stride seg words) off a single bank.
__device__ __forceinline__ int pad(int i) { return i + (i >> 5); }

// Exact rank search among n keys held in shared memory by one CTA: the
// rank-th largest key (11 + 11 + 10-bit radix passes) and the rank left
// among the keys equal to it.
__device__ void cta_select_keys(const uint32_t *keys, int n, unsigned rank, unsigned *hist,
                                unsigned *scan_tmp, unsigned *s_bin, unsigned *s_rank,
                                uint32_t *tau_out, unsigned *rank_out) {
    uint32_t prefix = 0, mask = 0;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int rd = 0; rd < 3; rd++) {
        const uint32_t dm = (1u << widths[rd]) - 1u;
        for (int i = threadIdx.x; i <= (int)dm; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += kThreads) {
            const uint32_t key = keys[j];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shifts[rd]) & dm], 1u);
        }
        __syncthreads();
        find_rank_bin(hist, (int)dm + 1, rank, s_bin, s_rank, scan_tmp);
        prefix |= *s_bin << shifts[rd];
        mask |= dm << shifts[rd];
        rank = *s_rank;
        __syncthreads();
    }
    *tau_out = prefix;
    *rank_out = rank;
}

constexpr int kGather = 8192;      // candidates CTA 0 can select alone

// Rows of a cache the next kernel gathers at the selected positions: the
// top-k asks L2 for each selected row as it writes the position (a no-op
// when base is null), so that the gather finds them there.
struct RowPrefetch {
    const uint8_t *base;    // row (b, t) at base + (b * t_max + t) * bytes
    int64_t t_max;
    int bytes;              // a multiple of 16
    __device__ __forceinline__ void operator()(int64_t b, int64_t t) const {
        if (base)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + (b * t_max + t) * bytes),
                         "r"(bytes)
                         : "memory");
    }
};

__global__ void __launch_bounds__(kThreads, 1)
topk_cluster_kernel(const float *scores, int S, int64_t T, int64_t start_pos, int K,
                    int L, int store_bins, int32_t *__restrict__ idx, const RowPrefetch pf) {
    // a kernel launched after this one (the sparse attention) may start its
    // set-up now; it reads the selections only after waiting for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cg::cluster_group cl = cg::this_cluster();
    const int CN = (int)cl.num_blocks();
    const int p = (int)cl.block_rank();
    const int64_t row = blockIdx.x / CN;
    const int64_t s = row % S, bseq = row / S;
    int64_t n_valid = start_pos + s + 1;
    if (n_valid > T) n_valid = T;
    const int m = (int64_t)K < n_valid ? K : (int)n_valid;
    int32_t *dst = idx + row * K;
    // The scores come from the preceding kernel (the scorer), and a kernel
    // before that may still read this row's old selections (an attention
    // launched ahead of this top-k): wait for the preceding grid (a no-op
    // without a programmatic launch) before reading or writing anything.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (m == n_valid) {                   // every causal position is selected
        for (int i = p * kThreads + threadIdx.x; i < K; i += CN * kThreads) {
            dst[i] = i < m ? i : -1;
            if (i < m) pf(bseq, i);
        }
        return;                           // uniform across the cluster
    }

    extern __shared__ float sv[];                                   // [pad(L)] scores
    uint32_t *gath = reinterpret_cast<uint32_t *>(sv + pad(L) + 1);  // [kGather] keys (CTA 0)
    uint16_t *cand = reinterpret_cast<uint16_t *>(gath + kGather);  // [L] candidate slots
    // each value's linear bin, [slot within the thread's segment][thread], when
    // shared memory holds it (else recomputed from the score)
    uint16_t *bins = store_bins ? cand + L : nullptr;
    __shared__ unsigned hist[kBins];          // local histogram
    __shared__ unsigned hmerged[kBins];       // cluster histogram (CTA 0)
    __shared__ unsigned scan_tmp[33];
    __shared__ int itmp[33];
    __shared__ ClusterCtl ctl;
    __shared__ unsigned s_bin, s_rank;
    __shared__ uint32_t s_tau;
    __shared__ int s_ncand;
    __shared__ float s_lo, s_hi;

    const int64_t t0 = (int64_t)p * L;
    int64_t t1 = t0 + L;
    if (t1 > n_valid) t1 = n_valid;
    const int len = t1 > t0 ? (int)(t1 - t0) : 0;
    const float *src = scores + row * T + t0;

    // load the slice, finite min / max; clear the histograms
    // (loads are issued in batches of eight per thread so their latencies overlap)
    float lo = INFINITY, hi = -INFINITY;
    const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
    if (vec) {
        const int n4 = len >> 2;
        for (int base = 0; base < n4; base += 8 * kThreads) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = base + u * kThreads + threadIdx.x;
                v[u] = j < n4 ? reinterpret_cast<const float4 *>(src)[j]
                              : make_float4(NAN, NAN, NAN, NAN);
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = base + u * kThreads + threadIdx.x;
                if (j >= n4) continue;
                const float xs[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    sv[pad(4 * j + e)] = xs[e];
                    if (isfinite(xs[e])) {
                        lo = fminf(lo, xs[e]);
                        hi = fmaxf(hi, xs[e]);
                    }
                }
            }
        }
    }
    for (int base = vec ? (len & ~3) : 0; base < len; base += 8 * kThreads) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = base + u * kThreads + threadIdx.x;
            v[u] = i < len ? src[i] : NAN;
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = base + u * kThreads + threadIdx.x;
            if (i >= len) continue;
            sv[pad(i)] = v[u];
            if (isfinite(v[u])) {
                lo = fminf(lo, v[u]);
                hi = fmaxf(hi, v[u]);
            }
        }
    }
    for (int i = threadIdx.x; i < kBins; i += kThreads) {
        hist[i] = 0;
        hmerged[i] = 0;
    }
    lo = -warp_max(-lo);
    hi = warp_max(hi);
    if ((threadIdx.x & 31) == 0) {
        reinterpret_cast<float *>(itmp)[threadIdx.x >> 5] = lo;
        scan_tmp[threadIdx.x >> 5] = __float_as_uint(hi);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float l = INFINITY, h = -INFINITY;
        for (int w = 0; w < kWarps; w++) {
            l = fminf(l, reinterpret_cast<float *>(itmp)[w]);
            h = fmaxf(h, __uint_as_float(scan_tmp[w]));
        }
        ctl.lo = l;
        ctl.hi = h;
    }
    cl.sync();                                                            // (1)
    if (threadIdx.x == 0) {
        float l = INFINITY, h = -INFINITY;
        for (int r = 0; r < CN; r++) {
            const ClusterCtl *rc = cl.map_shared_rank(&ctl, r);
            l = fminf(l, rc->lo);
            h = fmaxf(h, rc->hi);
        }
        s_lo = l;
        s_hi = h;
    }
    __syncthreads();
    const float g_lo = s_lo, g_hi = s_hi;
    const float scale = (g_hi > g_lo && isfinite(g_hi - g_lo)) ? __fdiv_rn((float)kBins, g_hi - g_lo)
                                                                  : 0.f;

    // round 0: linear bins, merged into CTA 0 with distributed shared-memory atomics
    // thread i owns the contiguous segment [i*seg, (i+1)*seg) of the slice
    const int seg = (len + kThreads - 1) / kThreads;
    const int s0 = threadIdx.x * seg < len ? threadIdx.x * seg : len;
    const int s1 = s0 + seg < len ? s0 + seg : len;
    for (int i = s0; i < s1; i++) {
        const int bin = linear_bin(sv[pad(i)], g_lo, scale);
        if (bins) bins[(i - s0) * kThreads + threadIdx.x] = (uint16_t)bin;
        atomicAdd(&hist[bin], 1u);
    }
    auto bin_of = [&](int i) -> int {
        return bins ? (int)bins[(i - s0) * kThreads + threadIdx.x] : linear_bin(sv[pad(i)], g_lo, scale);
    };
    __syncthreads();
    {
        unsigned *h0 = cl.map_shared_rank(hmerged, 0);
        for (int b = threadIdx.x; b < kBins; b += kThreads)
            if (hist[b]) atomicAdd(h0 + b, hist[b]);
    }
    cl.sync();                                                            // (2)
    if (p == 0) {
        find_rank_bin(hmerged, kBins, (unsigned)m, &s_bin, &s_rank, scan_tmp);
        if (threadIdx.x < CN) {
            ClusterCtl *rc = cl.map_shared_rank(&ctl, (int)threadIdx.x);
            rc->bin = s_bin;
            rc->rank = s_rank;
        }
    }
    cl.sync();                                                            // (3)
    const int tb = (int)ctl.bin;
    unsigned rank = ctl.rank;

    // threshold-bin candidates (slot indices, in any order: only their keys
    // matter), appended in one pass
    if (threadIdx.x == 0) s_ncand = 0;
    __syncthreads();
    int above = 0;                        // this thread's values in bins above the threshold bin
    for (int i = s0; i < s1; i++) {
        const int bin = bin_of(i);
        above += bin > tb;
        if (bin == tb) cand[atomicAdd(&s_ncand, 1)] = (uint16_t)i;
    }
    __syncthreads();
    const int n_cand = s_ncand;
    if (threadIdx.x == 0) ctl.n_cand = n_cand;
    cl.sync();                                                            // (4)
    int cand_off = 0, E = 0;
    for (int r = 0; r < CN; r++) {
        const int c = cl.map_shared_rank(&ctl, r)->n_cand;
        if (r < p) cand_off += c;
        E += c;
    }

    uint32_t tau;
    int q;
    if (E <= kGather) {
        // few candidates: CTA 0 selects among all of them alone
        uint32_t *g0 = cl.map_shared_rank(gath, 0);
        for (int j = threadIdx.x; j < n_cand; j += kThreads) g0[cand_off + j] = score_key(sv[pad(cand[j])]);
        cl.sync();                                                        // (5)
        if (p == 0) {
            unsigned rk;
            if (E <= kThreads) {
                // few candidates: rank each key directly (keys larger, keys equal);
                // the key whose range covers `rank` is tau, and rank - #larger of
                // the keys equal to it are taken (every tau-equal thread agrees)
                if ((int)threadIdx.x < E) {
                    const uint32_t kj = gath[threadIdx.x];
                    unsigned gt = 0, eq = 0;
                    for (int i = 0; i < E; i++) {
                        const uint32_t ki = gath[i];
                        gt += ki > kj;
                        eq += ki == kj;
                    }
                    if (gt < rank && gt + eq >= rank) {
                        s_tau = kj;
                        s_rank = rank - gt;
                    }
                }
                __syncthreads();
                rk = s_rank;
            } else {
                cta_select_keys(gath, E, rank, hist, scan_tmp, &s_bin, &s_rank, &s_tau, &rk);
            }
            if (threadIdx.x < CN) {
                ClusterCtl *rc = cl.map_shared_rank(&ctl, (int)threadIdx.x);
                rc->bin = s_tau;
                rc->rank = rk;
            }
        }
        cl.sync();                                                        // (6)
        tau = ctl.bin;
        q = (int)ctl.rank;
    } else {
        // many candidates: radix rounds over each CTA's own candidates,
        // histograms merged into CTA 0 with distributed atomics
        uint32_t prefix = 0, mask = 0;
        const int shifts[3] = {21, 10, 0};
        const int widths[3] = {11, 11, 10};
        for (int rd = 0; rd < 3; rd++) {
            const int sh = shifts[rd];
            const uint32_t dm = (1u << widths[rd]) - 1u;
            for (int i = threadIdx.x; i < kBins; i += kThreads) {
                hist[i] = 0;
                hmerged[i] = 0;
            }
            cl.sync();
            for (int j = threadIdx.x; j < n_cand; j += kThreads) {
                const uint32_t key = score_key(sv[pad(cand[j])]);
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & dm], 1u);
            }
            __syncthreads();
            {
                unsigned *h0 = cl.map_shared_rank(hmerged, 0);
                for (int b = threadIdx.x; b <= (int)dm; b += kThreads)
                    if (hist[b]) atomicAdd(h0 + b, hist[b]);
            }
            cl.sync();
            if (p == 0) {
                find_rank_bin(hmerged, (int)dm + 1, rank, &s_bin, &s_rank, scan_tmp);
                if (threadIdx.x < CN) {
                    ClusterCtl *rc = cl.map_shared_rank(&ctl, (int)threadIdx.x);
                    rc->bin = s_bin;
                    rc->rank = s_rank;
                }
            }
            cl.sync();
            prefix |= ctl.bin << sh;
            mask |= dm << sh;
            rank = ctl.rank;
        }
        tau = prefix;
        q = (int)rank;
    }

    // counts, exchanged through the cluster, give each CTA its output offset.
    // Every value above the threshold bin is > tau; of the candidates, each
    // adds to its owner thread's count of keys > tau or == tau.
    unsigned *t_gt = hist, *t_eq = hist + kThreads;        // hist is free again
    t_gt[threadIdx.x] = 0;
    t_eq[threadIdx.x] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n_cand; j += kThreads) {
        const int slot = cand[j];
        const uint32_t key = score_key(sv[pad(slot)]);
        if (key > tau) atomicAdd(&t_gt[slot / seg], 1u);
        else if (key == tau) atomicAdd(&t_eq[slot / seg], 1u);
    }
    __syncthreads();
    const int gt = above + (int)t_gt[threadIdx.x], eq = (int)t_eq[threadIdx.x];
    int cta_gt, cta_eq;
    block_scan_int(gt, itmp, &cta_gt);
    const int eq_before_me = block_scan_int(eq, itmp, &cta_eq);
    if (threadIdx.x == 0) {
        ctl.n_gt = cta_gt;
        ctl.n_eq = cta_eq;
    }
    cl.sync();                                                            // (7)
    int off = 0, eq_before = 0;
    for (int r = 0; r < p; r++) {
        const ClusterCtl *rc = cl.map_shared_rank(&ctl, r);
        int quota = q - eq_before;
        quota = quota < 0 ? 0 : (quota > rc->n_eq ? rc->n_eq : quota);
        off += rc->n_gt + quota;
        eq_before += rc->n_eq;
    }
    cl.sync();                            // (8) no CTA leaves while others read its counts
    // tau-equal positions this thread takes: the first (q - earlier ones)
    int my_q = q - eq_before - eq_before_me;
    my_q = my_q < 0 ? 0 : (my_q > eq ? eq : my_q);
    int tot;
    int pos = off + block_scan_int(gt + my_q, itmp, &tot);
    for (int i = s0; i < s1; i++) {
        // bins are monotone in the score: above the threshold bin means > tau,
        // below means < tau; only threshold-bin values need their key
        const int bin = bin_of(i);
        if (bin < tb) continue;
        bool take = bin > tb;
        if (!take) {
            const uint32_t key = score_key(sv[pad(i)]);
            take = key > tau;
            if (key == tau && my_q > 0) {
                take = true;
                my_q--;
            }
        }
        if (take && pos < m) {
            dst[pos++] = (int32_t)(t0 + i);
            pf(bseq, t0 + i);
        }
    }
    for (int i = m + p * kThreads + threadIdx.x; i < K; i += CN * kThreads) dst[i] = -1;
}

// One CTA per row, the row read from global memory (rows too long for the
// cluster kernel's shared memory).
__global__ void __launch_bounds__(kThreads)
topk_row_kernel(const float *__restrict__ scores, int S, int64_t T, int64_t start_pos, int K,
                int32_t *__restrict__ idx) {
    __shared__ unsigned hist[256];
    __shared__ int warp_tot[33];
    __shared__ unsigned s_sel, s_remaining;

    const int64_t row = blockIdx.x;
    const int64_t s = row % S;
    int64_t n_valid = start_pos + s + 1;
    if (n_valid > T) n_valid = T;
    const int m = (int64_t)K < n_valid ? K : (int)n_valid;
    const float *src = scores + row * T;
    int32_t *dst = idx + row * K;

    if (m == n_valid) {
        for (int i = threadIdx.x; i < K; i += kThreads) dst[i] = i < m ? i : -1;
        return;
    }
    uint32_t prefix = 0, mask = 0;
    unsigned remaining = (unsigned)m;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int64_t t = threadIdx.x; t < n_valid; t += kThreads) {
            const uint32_t key = score_key(src[t]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned cum = 0;
            int bin = 255;
            for (; bin > 0; bin--) {
                if (cum + hist[bin] >= remaining) break;
                cum += hist[bin];
            }
            s_sel = (unsigned)bin;
            s_remaining = remaining - cum;
        }
        __syncthreads();
        prefix |= s_sel << shift;
        mask |= 255u << shift;
        remaining = s_remaining;
        __syncthreads();
    }
    const uint32_t tau = prefix;
    const int need_eq = (int)remaining;
    int out_base = 0, eq_seen = 0;
    for (int64_t start = 0; start < n_valid; start += kThreads) {
        const int64_t t = start + threadIdx.x;
        const bool in = t < n_valid;
        const uint32_t key = in ? score_key(src[t]) : 0u;
        const bool gt = in && key > tau;
        const bool eq = in && key == tau;
        int eq_total;
        const int eq_rank = block_scan_flag(eq, warp_tot, &eq_total);
        const bool sel = gt || (eq && eq_seen + eq_rank < need_eq);
        int sel_total;
        const int pos = block_scan_flag(sel, warp_tot, &sel_total);
        if (sel && out_base + pos < m) dst[out_base + pos] = (int32_t)t;
        out_base += sel_total;
        eq_seen += eq_total;
    }
    for (int i = m + threadIdx.x; i < K; i += kThreads) dst[i] = -1;
}

// Cluster size and slice length for rows of up to `n` positions; CN = 0 if
// the cluster kernel cannot hold them.
void cluster_plan(int64_t n, int *cn, int *slice) {
    int c = 1;
    while (c < 8 && (n + c - 1) / c > 16384) c *= 2;
    int64_t l = (n + c - 1) / c;
    if (l > kMaxSlice) {
        c = 16;
        l = (n + c - 1) / c;
    }
    if (l > kMaxSlice) {
        *cn = 0;
        *slice = 0;
        return;
    }
    *cn = c;
    *slice = (int)((l + 7) / 8 * 8);
}

}  // namespace

size_t topk_workspace_bytes(int, int, int64_t, int) { return 0; }

dsa_status launch_topk_select(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                              int k, int32_t *idx, void *, cudaStream_t stream,
                              const void *prefetch_rows, int64_t prefetch_t_max,
                              int prefetch_row_bytes) {
    if ((int64_t)B * S * T == 0) return DSA_OK;
    const int K = (int64_t)k < T ? k : (int)T;
    const int64_t rows = (int64_t)B * S;
    const int64_t n_max = T < start_pos + S ? T : start_pos + S;
    int cn, L;
    cluster_plan(n_max, &cn, &L);
    if (cn == 0) {
        topk_row_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(scores, S, T, start_pos, K, idx);
        return launch_status();
    }
    size_t smem = (size_t)(L + L / 32 + 1) * sizeof(float) + kGather * sizeof(uint32_t) +
                  (size_t)L * sizeof(uint16_t);
    // per-value bins too, when they fit beside the static shared memory (~17 KB)
    const size_t bins_bytes = (size_t)((L + kThreads - 1) / kThreads) * kThreads * sizeof(uint16_t);
    const int store_bins = smem + bins_bytes <= (size_t)(208 * 1024) ? 1 : 0;
    if (store_bins) smem += bins_bytes;
    if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (cn > 8 && cudaFuncSetAttribute(topk_cluster_kernel,
                                       cudaFuncAttributeNonPortableClusterSizeAllowed,
                                       1) != cudaSuccess)
        return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * cn));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cn;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic launch: the launch overlaps the preceding kernel's tail; the
    // kernel waits for that grid before reading the scores
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    RowPrefetch pf;
    pf.base = static_cast<const uint8_t *>(prefetch_rows);
    pf.t_max = prefetch_t_max;
    pf.bytes = prefetch_row_bytes;
    if (cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, S, T, start_pos, K, L, store_bins, idx,
                           pf) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa

extern "C" size_t dsa_topk_select_workspace_size(int B, int S, int64_t T, int k) {
    if (B <= 0 || S <= 0 || T <= 0 || k <= 0) return 0;
    return dsa::topk_workspace_bytes(B, S, T, k);
}

extern "C" dsa_status dsa_topk_select(const float *scores, int B, int S, int64_t T,
                                      int64_t start_pos, int k, int32_t *idx, void *workspace,
                                      size_t workspace_bytes, dsa_stream_t stream) {
    if (B < 0 || S < 0 || T < 0 || start_pos < 0 || k < 1) return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * S * T == 0) return DSA_OK;
    if (T > INT32_MAX || start_pos + S > T) return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * S * 16 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::topk_workspace_bytes(B, S, T, k);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DSA_ERR_WORKSPACE;
    return dsa::launch_topk_select(scores, B, S, T, start_pos, k, idx, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
}
