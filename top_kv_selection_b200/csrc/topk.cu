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
// Scores are compared through an order-preserving 32-bit key (score_key).
// Cluster kernel (rows up to ~460K positions): a thread-block cluster of CN
// CTAs owns one row; CTA p keeps the keys of positions [p L, (p+1) L) in
// shared memory.  tau is found by radix rounds on the key bits, each a
// histogram of the keys still in play, merged into CTA 0 with distributed
// shared-memory atomics and read back by every CTA, which all find the same
// threshold bin (no broadcast step):
//   round 0: the top 12 key bits of every key (sign, exponent, 3 mantissa
//            bits: bins an eighth of an octave wide);
//   when the keys in the threshold bin are few enough (kCap), they are
//   gathered with their positions into CTA 0, and every CTA reads them back
//   and finds tau among them by radix passes in its own shared memory;
//   otherwise further 12-bit rounds narrow the prefix first.
// The counts each CTA needs for its output offset (keys above tau, and the
// tau-equal keys of lower CTAs) come from the counts every CTA published and
// from the gathered keys' positions, so that the positions are written in
// ascending order with three cluster barriers on the common path.
//
// Decode kernel (one query per sequence, the scorer's per-row histogram of
// the top 12 key bits at hand): the same cluster layout, but every CTA finds
// the threshold bin from that histogram itself, so round 0 and its merge
// disappear and the scores are read once.
//
// Fallback kernel (longer rows): one CTA per row, four 8-bit radix passes
// over the row in global memory, then the same ordered compaction.
#include <cooperative_groups.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBits = 12;                 // key bits a cluster round resolves
constexpr int kBins = 1 << kBits;         // 4096
constexpr int kCap = 8192;                // keys CTA 0 gathers for the exact selection
constexpr int kMaxSlice = 28672;          // keys per CTA kept in shared memory
constexpr int kMaxCluster = 16;

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

// Block-wide exclusive scan of two ints at once; totals in *ta, *tb.
__device__ __forceinline__ void block_scan2(int a, int b, int *ea, int *eb, int2 *tmp, int *ta,
                                            int *tb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int na = __shfl_up_sync(0xffffffffu, ia, o);
        const int nb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += na;
            ib += nb;
        }
    }
    if (lane == 31) tmp[warp] = make_int2(ia, ib);
    __syncthreads();
    if (warp == 0) {
        const int2 v = tmp[lane];
        int wa = v.x, wb = v.y;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int na = __shfl_up_sync(0xffffffffu, wa, o);
            const int nb = __shfl_up_sync(0xffffffffu, wb, o);
            if (lane >= o) {
                wa += na;
                wb += nb;
            }
        }
        tmp[lane] = make_int2(wa - v.x, wb - v.y);
        if (lane == 31) tmp[32] = make_int2(wa, wb);
    }
    __syncthreads();
    *ea = tmp[warp].x + ia - a;
    *eb = tmp[warp].y + ib - b;
    *ta = tmp[32].x;
    *tb = tmp[32].y;
    __syncthreads();
}

// In a histogram of nb = 4 * kThreads or fewer bins (bin index = key digit,
// larger is better), finds the bin holding the rank-th largest key (1-based)
// and the count of keys in the bins above it.  Thread t owns the 4 bins
// nb - 4t - 4 .. nb - 4t - 1 (descending); get(i) reads bin i.  Every thread
// of the block calls it and gets the same answer.
template <typename Get>
__device__ __forceinline__ void find_rank(Get get, int nb, unsigned rank, unsigned *bin_out,
                                          unsigned *above_out, unsigned *cnt_out, int2 *tmp) {
    const int t = threadIdx.x;
    const int b0 = nb - 4 * t - 1;                 // this thread's highest bin
    unsigned c[4];
#pragma unroll
    for (int j = 0; j < 4; j++) c[j] = b0 - j >= 0 ? get(b0 - j) : 0u;
    const int mine = (int)(c[0] + c[1] + c[2] + c[3]);
    int before, unused, total, unused2;
    block_scan2(mine, 0, &before, &unused, tmp, &total, &unused2);
    unsigned above = (unsigned)before;
    __shared__ unsigned s_out[3];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        if (b0 - j >= 0 && above < rank && above + c[j] >= rank) {
            s_out[0] = (unsigned)(b0 - j);
            s_out[1] = above;
            s_out[2] = c[j];
        }
        above += c[j];
    }
    __syncthreads();
    *bin_out = s_out[0];
    *above_out = s_out[1];
    *cnt_out = s_out[2];
    __syncthreads();
}

// Slice element i lives at sv[pad(i)]: one spare word every 32 keeps the
// per-thread contiguous segments (stride seg words) off a single bank.
__device__ __forceinline__ int pad(int i) { return i + (i >> 5); }

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

// Shared by the CTAs of a cluster through distributed shared memory.  Other
// CTAs only write into CTA 0 (atomics, appends, counts) and CTA 0 only writes
// small results back; nobody reads another CTA's shared memory in bulk.
struct TopkShared {
    unsigned hist[kBins];           // this CTA's histogram; CTA 0's is the cluster's sum
    unsigned res[4];                // from CTA 0: prefix, prefix bits, rank in group, group size
    unsigned out[3];                // from CTA 0: tau, this CTA's output offset, its tau-equal quota
    int n_cand;                     // CTA 0: keys gathered
    int cnt_gt[kMaxCluster];        // CTA 0: per CTA, keys above the prefix group
    int cnt_in[kMaxCluster];        // CTA 0: per CTA, keys inside it
    int sel_gt[kMaxCluster];        // CTA 0: per CTA, gathered keys above tau
    int sel_eq[kMaxCluster];        // CTA 0: per CTA, gathered keys equal to tau
};

// The prefix group's threshold bin in CTA 0's merged histogram, found by CTA
// 0 and written into every CTA's res (call with the whole cluster; a cluster
// barrier must follow before res is read).
__device__ __forceinline__ void cta0_find_and_send(cg::cluster_group &cl, TopkShared &sh, int nb,
                                                   uint32_t prefix, int pbits, unsigned rank,
                                                   int2 *tmp) {
    if (cl.block_rank() != 0) return;
    unsigned bin, above, cnt;
    find_rank([&](int i) { return sh.hist[i]; }, 1 << nb, rank, &bin, &above, &cnt, tmp);
    if (threadIdx.x < cl.num_blocks()) {
        TopkShared *r = cl.map_shared_rank(&sh, (int)threadIdx.x);
        r->res[0] = (prefix << nb) | bin;
        r->res[1] = (unsigned)(pbits + nb);
        r->res[2] = rank - above;
        r->res[3] = cnt;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
topk_cluster_kernel(const float *scores, int S, int64_t T, int64_t start_pos, int K, int L,
                    int32_t *__restrict__ idx, const RowPrefetch pf, int compress) {
    // a kernel launched after this one (the sparse attention) may start its
    // set-up now; it reads the selections only after waiting for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cg::cluster_group cl = cg::this_cluster();
    const int CN = (int)cl.num_blocks();
    const int p = (int)cl.block_rank();
    const int64_t row = blockIdx.x / CN;
    const int64_t s = row % S, bseq = row / S;
    int64_t n_valid = (start_pos + s + 1) / compress;
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

    extern __shared__ uint32_t dyn[];
    uint32_t *keys = dyn;                                           // [pad(L) + 1]
    uint32_t *ck = keys + pad(L) + 1;                               // CTA 0: [kCap] gathered keys
    int32_t *cp = reinterpret_cast<int32_t *>(ck + kCap);           // CTA 0: [kCap] their positions
    __shared__ TopkShared sh;
    __shared__ int2 scan_tmp[33];
    TopkShared *sh0 = cl.map_shared_rank(&sh, 0);

    const int64_t t0 = (int64_t)p * L;
    int64_t t1 = t0 + L;
    if (t1 > n_valid) t1 = n_valid;
    const int len = t1 > t0 ? (int)(t1 - t0) : 0;
    const float *src = scores + row * T + t0;

    // clear, then let the other CTAs know (the barrier's wait comes after the
    // slice is loaded, so its latency is hidden)
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[i] = 0;
    if (threadIdx.x < kMaxCluster) {
        sh.sel_gt[threadIdx.x] = 0;
        sh.sel_eq[threadIdx.x] = 0;
    }
    if (threadIdx.x == 0) sh.n_cand = 0;
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

    // keys of the slice and the histogram of their top 12 bits
    auto put = [&](int i, float x) {
        const uint32_t key = score_key(x);
        keys[pad(i)] = key;
        atomicAdd(&sh.hist[key >> (32 - kBits)], 1u);
    };
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
        const int n4 = len >> 2;
        for (int base = 0; base < n4; base += 4 * kThreads) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int j = base + u * kThreads + threadIdx.x;
                v[u] = j < n4 ? reinterpret_cast<const float4 *>(src)[j] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int j = base + u * kThreads + threadIdx.x;
                if (j >= n4) continue;
                put(4 * j, v[u].x);
                put(4 * j + 1, v[u].y);
                put(4 * j + 2, v[u].z);
                put(4 * j + 3, v[u].w);
            }
        }
        for (int i = (len & ~3) + threadIdx.x; i < len; i += kThreads) put(i, src[i]);
    } else {
        for (int i = threadIdx.x; i < len; i += kThreads) put(i, src[i]);
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");

    // ---- round 0: the 12-bit bin holding the m-th largest key
    uint32_t prefix;
    int pbits;
    unsigned rank, n_group;
    {
        if (p != 0)
            for (int i = threadIdx.x; i < kBins; i += kThreads) {
                const unsigned c = sh.hist[i];
                if (c) atomicAdd(&sh0->hist[i], c);
            }
        cl.sync();
        cta0_find_and_send(cl, sh, kBits, 0u, 0, (unsigned)m, scan_tmp);
        cl.sync();
        prefix = sh.res[0];
        pbits = (int)sh.res[1];
        rank = sh.res[2];
        n_group = sh.res[3];
    }
    // further 12-bit rounds while the group is too large to gather (rare:
    // scores within a few percent of each other, or many exact ties)
    while (n_group > (unsigned)kCap && pbits < 32) {
        const int nb = 32 - pbits < kBits ? 32 - pbits : kBits;
        const int sh_lo = 32 - pbits - nb;
        for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[i] = 0;
        cl.sync();                                  // CTA 0's histogram is clear
        for (int i = threadIdx.x; i < len; i += kThreads) {
            const uint32_t key = keys[pad(i)];
            if ((key >> (32 - pbits)) == prefix)
                atomicAdd(&sh.hist[(key >> sh_lo) & ((1u << nb) - 1u)], 1u);
        }
        __syncthreads();
        if (p != 0)
            for (int i = threadIdx.x; i < (1 << nb); i += kThreads) {
                const unsigned c = sh.hist[i];
                if (c) atomicAdd(&sh0->hist[i], c);
            }
        cl.sync();
        cta0_find_and_send(cl, sh, nb, prefix, pbits, rank, scan_tmp);
        cl.sync();
        prefix = sh.res[0];
        pbits = (int)sh.res[1];
        rank = sh.res[2];
        n_group = sh.res[3];
    }

    // ---- this CTA's keys above the group and inside it, counted into CTA 0;
    // the group's keys themselves are gathered there when they are few
    const bool gather = n_group <= (unsigned)kCap && pbits < 32;
    const int gshift = 32 - pbits;
    int n_gt = 0, n_in = 0;
    uint32_t *rk = cl.map_shared_rank(ck, 0);
    int32_t *rp = cl.map_shared_rank(cp, 0);
    for (int i0 = 0; i0 < len; i0 += kThreads) {
        const int i = i0 + threadIdx.x;
        uint32_t key = 0;
        bool in = false;
        if (i < len) {
            key = keys[pad(i)];
            const uint32_t g = gshift == 32 ? 0u : key >> gshift;
            n_gt += g > prefix;
            in = g == prefix;
            n_in += in;
        }
        if (gather) {
            // warp-aggregated append into CTA 0's list
            const unsigned bal = __ballot_sync(0xffffffffu, in);
            const int lane = threadIdx.x & 31;
            int base = 0;
            if (lane == 0 && bal) base = atomicAdd(&sh0->n_cand, __popc(bal));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (in) {
                const int slot = base + __popc(bal & ((1u << lane) - 1u));
                if (slot < kCap) {
                    rk[slot] = key;
                    rp[slot] = (int32_t)(t0 + i);
                }
            }
        }
    }
    {
        int e_gt, e_in, tot_gt, tot_in;
        block_scan2(n_gt, n_in, &e_gt, &e_in, scan_tmp, &tot_gt, &tot_in);
        if (threadIdx.x == 0) {
            sh0->cnt_gt[p] = tot_gt;
            sh0->cnt_in[p] = tot_in;
        }
    }
    cl.sync();                                                      // counts and keys in CTA 0

    // ---- CTA 0: tau (the rank-th largest key of the group), q (tau-equal keys
    // taken), and every CTA's output offset and tau-equal quota
    if (p == 0) {
        uint32_t tau;
        int q;
        if (gather) {
            // radix passes on the gathered keys' remaining bits (at most 11 at a time)
            const int E = (int)n_group;
            uint32_t tp = prefix;
            int tbits = pbits;
            unsigned rk_left = rank;
            while (tbits < 32) {
                const int nb = 32 - tbits < 11 ? 32 - tbits : 11;
                const int sh_lo = 32 - tbits - nb;
                for (int i = threadIdx.x; i < (1 << nb); i += kThreads) sh.hist[i] = 0;
                __syncthreads();
                for (int j = threadIdx.x; j < E; j += kThreads) {
                    const uint32_t key = ck[j];
                    if ((key >> (32 - tbits)) == tp) atomicAdd(&sh.hist[(key >> sh_lo) & ((1u << nb) - 1u)], 1u);
                }
                __syncthreads();
                unsigned bin, above, cnt;
                find_rank([&](int i) { return sh.hist[i]; }, 1 << nb, rk_left, &bin, &above, &cnt, scan_tmp);
                tp = (tp << nb) | bin;
                tbits += nb;
                rk_left -= above;
            }
            tau = tp;
            q = (int)rk_left;
            // per CTA: gathered keys above tau and equal to tau
            for (int j = threadIdx.x; j < E; j += kThreads) {
                const uint32_t key = ck[j];
                const int c = (int)(cp[j] / L);
                if (key > tau) atomicAdd(&sh.sel_gt[c], 1);
                else if (key == tau) atomicAdd(&sh.sel_eq[c], 1);
            }
            __syncthreads();
        } else {
            // the group is one key value: its keys are all tau-equal
            tau = prefix;
            q = (int)rank;
        }
        if (threadIdx.x < CN) {
            const int t = (int)threadIdx.x;
            int gt = 0, eq = 0;
            for (int r = 0; r < t; r++) {
                gt += sh.cnt_gt[r] + (gather ? sh.sel_gt[r] : 0);
                eq += gather ? sh.sel_eq[r] : sh.cnt_in[r];
            }
            const int mine = gather ? sh.sel_eq[t] : sh.cnt_in[t];
            int my_q = q - eq;
            my_q = my_q < 0 ? 0 : (my_q > mine ? mine : my_q);
            TopkShared *r = cl.map_shared_rank(&sh, t);
            r->out[0] = tau;
            r->out[1] = (unsigned)(gt + (q < eq ? q : eq));
            r->out[2] = (unsigned)my_q;
        }
    }
    cl.sync();                            // results delivered; no CTA touches another's memory after this
    const uint32_t tau = sh.out[0];
    const int off = (int)sh.out[1], my_q = (int)sh.out[2];

    // ---- ordered write: thread i owns the contiguous segment [i seg, (i+1) seg)
    const int seg = (len + kThreads - 1) / kThreads;
    const int s0 = threadIdx.x * seg < len ? threadIdx.x * seg : len;
    const int s1 = s0 + seg < len ? s0 + seg : len;
    int c_gt = 0, c_eq = 0;
    for (int i = s0; i < s1; i++) {
        const uint32_t key = keys[pad(i)];
        c_gt += key > tau;
        c_eq += key == tau;
    }
    int e_gt, e_eq, tot_gt, tot_eq;
    block_scan2(c_gt, c_eq, &e_gt, &e_eq, scan_tmp, &tot_gt, &tot_eq);
    // tau-equal keys this thread takes: the CTA's quota goes to the lowest positions
    int take_eq = my_q - e_eq;
    take_eq = take_eq < 0 ? 0 : (take_eq > c_eq ? c_eq : take_eq);
    int pos = off + e_gt + (my_q < e_eq ? my_q : e_eq);
    for (int i = s0; i < s1; i++) {
        const uint32_t key = keys[pad(i)];
        bool take = key > tau;
        if (key == tau && take_eq > 0) {
            take = true;
            take_eq--;
        }
        if (take && pos < m) {
            dst[pos++] = (int32_t)(t0 + i);
            pf(bseq, t0 + i);
        }
    }
    for (int i = m + p * kThreads + threadIdx.x; i < K; i += CN * kThreads) dst[i] = -1;
}

// ------------------------------------------------------------ decode top-k
// The decode step's top-k, when the scorer's CTAs have counted their scores
// by the top 12 key bits: a cluster of CN CTAs of 512 threads per row, each
// thread owning 32 consecutive positions (their keys in shared memory, loaded
// as coalesced float4s; the thread keeps bitmasks of which are above the
// threshold bin and which fall in it).  CTA p sums its
// slice of the bins over the row's scorer histograms and stores the sums into
// every CTA of the cluster, so that after one cluster barrier every CTA holds
// the row's histogram and finds the same 12-bit threshold bin on its own; the
// scores are read once.  Each warp adds its counts into CTA 0's per-CTA
// totals, reserves a range of CTA 0's candidate list with one atomic and
// stores its keys that fall in the bin there, with their positions
// (distributed shared memory); CTA 0 finds tau among them (a 10-bit histogram pass, then one warp
// ranks the few keys left, or further passes when they are many) and every
// CTA's output offset and tau-equal quota, and sends each CTA its numbers.
// Two cluster barriers on the common path; global memory sees only the
// scores, the histogram and the output.  When the threshold bin holds more
// keys than CTA 0 can gather, 12-bit rounds over the register keys, merged
// into CTA 0, narrow it first.
constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecPer = 32;                         // positions per thread
constexpr int kDecSpan = kDecThreads * kDecPer;     // positions per CTA: 16384
constexpr int kKeyPitch = kDecPer + 1;              // a thread's keys in shared memory (padded)
constexpr int kDecCap = 8192;                       // keys CTA 0 gathers
constexpr int kDecSub = 1024;                       // bins of a 10-bit pass
constexpr int kDecFew = 32;                         // keys one warp ranks directly

struct DecShared {
    unsigned hist[kBins];             // CTA 0: histogram of the current pass or round
    unsigned rowhist[kBins];          // the row's histogram, a slice from each CTA
    uint2 cand[kDecCap];              // CTA 0: gathered (key, position), warp by warp
    int n_cand;                       // CTA 0: slots reserved
    int cnt_gt[kMaxCluster];          // CTA 0: per CTA, keys above the group
    int cnt_in[kMaxCluster];          // CTA 0: per CTA, keys inside it
    int sel_gt[kMaxCluster];          // CTA 0: per CTA, gathered keys above tau
    int sel_eq[kMaxCluster];          // CTA 0: per CTA, gathered keys equal to tau
    unsigned res[4];                  // from CTA 0: prefix, prefix bits, rank in group, group size
    unsigned out[3];                  // from CTA 0: tau, output offset, tau-equal quota
    int n_few;
    uint32_t few[kDecFew];
    unsigned s_out[3];
    int wtmp[kDecWarps];
    int2 wtmp2[kDecWarps];
};

// Sum over lanes 0..n-1 of v (n <= 32), in every lane.
__device__ __forceinline__ int warp_sum_first(int v, int lane, int n) {
    int x = lane < n ? v : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Rank search over register-held counts: thread t holds the N bins
// b0 - N + 1 .. b0 (b0 = nb - N t - 1), c[j] the count of bin b0 - j (zero
// for bins below 0).  Finds the bin holding the rank-th largest key in
// descending bin order, the count above it and its own count; every thread
// gets the answer.
template <int N>
__device__ __forceinline__ void find_rank_regs(const unsigned (&c)[N], int b0, unsigned rank,
                                               unsigned *bin_out, unsigned *above_out,
                                               unsigned *cnt_out, DecShared &sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned mine = 0;
#pragma unroll
    for (int j = 0; j < N; j++) mine += c[j];
    unsigned incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sh.wtmp[warp] = (int)incl;
    __syncthreads();
    unsigned above = incl - mine +
                     (unsigned)warp_sum_first(lane < kDecWarps ? sh.wtmp[lane] : 0, lane, warp);
#pragma unroll
    for (int j = 0; j < N; j++) {
        if (b0 - j >= 0 && above < rank && above + c[j] >= rank) {
            sh.s_out[0] = (unsigned)(b0 - j);
            sh.s_out[1] = above;
            sh.s_out[2] = c[j];
        }
        above += c[j];
    }
    __syncthreads();
    *bin_out = sh.s_out[0];
    *above_out = sh.s_out[1];
    *cnt_out = sh.s_out[2];
    __syncthreads();
}

// Block-wide exclusive scan of two ints, with their totals in every thread.
__device__ __forceinline__ int2 block_scan2_dec(int a, int b, DecShared &sh, int2 *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int na = __shfl_up_sync(0xffffffffu, ia, o);
        const int nb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += na;
            ib += nb;
        }
    }
    if (lane == 31) sh.wtmp2[warp] = make_int2(ia, ib);
    __syncthreads();
    const int2 w = lane < kDecWarps ? sh.wtmp2[lane] : make_int2(0, 0);
    int2 r;
    r.x = ia - a + warp_sum_first(w.x, lane, warp);
    r.y = ib - b + warp_sum_first(w.y, lane, warp);
    total->x = warp_sum_first(w.x, lane, kDecWarps);
    total->y = warp_sum_first(w.y, lane, kDecWarps);
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kDecThreads, 1)
topk_decode_kernel(const float *scores, int64_t T, int K, int32_t *__restrict__ idx,
                   const RowPrefetch pf, const uint32_t *row_hist, int hist_chunks) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cg::cluster_group cl = cg::this_cluster();
    const int CN = (int)cl.num_blocks();
    const int p = (int)cl.block_rank();
    const int64_t row = blockIdx.x / CN;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = (int64_t)K < T ? K : (int)T;
    int32_t *dst = idx + row * K;
    if (m == T) {                          // every position selected (the same for every row)
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int i = p * kDecThreads + tid; i < K; i += CN * kDecThreads) {
            dst[i] = i < m ? i : -1;
            if (i < m) pf(row, i);
        }
        return;
    }
    extern __shared__ __align__(16) uint8_t dec_smem[];
    DecShared &sh = *reinterpret_cast<DecShared *>(dec_smem);
    // this CTA's keys, thread t's 32 positions at skey[t * 33 + j]: the per-key
    // loops below read them from here and stay rolled (one pass per CTA, so
    // unrolled code would be fetched cold on every SM)
    uint32_t *skey = reinterpret_cast<uint32_t *>(dec_smem + sizeof(DecShared));
    DecShared *sh0 = cl.map_shared_rank(&sh, 0);
    if (p == 0) {
        for (int i = tid; i < kBins; i += kDecThreads) sh.hist[i] = 0;
        if (tid == 0) sh.n_cand = 0;
        if (tid < kMaxCluster) {
            sh.cnt_gt[tid] = 0;
            sh.cnt_in[tid] = 0;
            sh.sel_gt[tid] = 0;
            sh.sel_eq[tid] = 0;
        }
    }
    if (tid == 0) sh.n_few = 0;
    __syncthreads();
    // cleared: the other CTAs may write here once they have waited
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    // the scores and the histogram come from the scorer
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // This CTA's scores, loaded first as coalesced float4s (consecutive
    // threads, consecutive 16 bytes; the thread that owns a position is not
    // the one that loads it), then its slice of the bins, summed over the
    // row's scorer histograms (thread t: bins b0 + t, b0 + t + 512, ...), with
    // both sets of loads in flight together.
    const int64_t span0 = (int64_t)p * kDecSpan;
    const int64_t span_n = T - span0 <= 0 ? 0 : (T - span0 >= kDecSpan ? kDecSpan : T - span0);
    const float *src = scores + row * T + span0;
    const bool vec = span_n == kDecSpan && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
    constexpr int kLoads = kDecSpan / 4 / kDecThreads;   // float4s a thread loads
    float4 kv4[kLoads];
    if (vec) {
#pragma unroll
        for (int u = 0; u < kLoads; u++)
            kv4[u] = reinterpret_cast<const float4 *>(src)[tid + u * kDecThreads];
    }
    const int bpc = (kBins + CN - 1) / CN;           // bins per CTA
    const int b_lo = p * bpc, b_hi = b_lo + bpc < kBins ? b_lo + bpc : kBins;
    constexpr int kMaxSlice = kBins / kDecThreads;   // bins a thread sums (CN = 1)
    unsigned bsum[kMaxSlice];
    {
        // up to kSumBatch histograms' loads in flight at once per bin
        constexpr int kSumBatch = 40;
        const uint32_t *rh = row_hist + row * hist_chunks * kBins;
#pragma unroll 1
        for (int u = 0; u < kMaxSlice; u++) {
            const int bb = b_lo + tid + u * kDecThreads;
            unsigned acc = 0;
            if (bb < b_hi) {
                for (int c0 = 0; c0 < hist_chunks; c0 += kSumBatch) {
                    unsigned v[kSumBatch];
#pragma unroll
                    for (int c = 0; c < kSumBatch; c++)
                        v[c] = c0 + c < hist_chunks ? ld_cg_u32(rh + (c0 + c) * kBins + bb) : 0u;
#pragma unroll
                    for (int c = 0; c < kSumBatch; c++) acc += v[c];
                }
            }
            bsum[u] = acc;
        }
    }
    // every CTA has started (and CTA 0 has cleared its merge state): store the
    // slice's sums into every CTA's copy of the row histogram (distributed
    // shared memory), while the score loads are still landing
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    for (int r = 0; r < CN; r++) {
        unsigned *peer = cl.map_shared_rank(sh.rowhist, r);
#pragma unroll
        for (int u = 0; u < kMaxSlice; u++) {
            const int bb = b_lo + tid + u * kDecThreads;
            if (bb < b_hi) peer[bb] = bsum[u];
        }
    }
    // the keys into shared memory: position o of the span at skey[(o / 32) * 33
    // + o % 32] (a warp's stores fall in 32 different banks; so do the owners'
    // reads of their j-th key); positions past T get key 0
#pragma unroll
    for (int u = 0; u < kLoads; u++) {
        const int o = 4 * (tid + u * kDecThreads);
        float4 v;
        if (vec) {
            v = kv4[u];
        } else {
            v.x = o < span_n ? src[o] : 0.f;
            v.y = o + 1 < span_n ? src[o + 1] : 0.f;
            v.z = o + 2 < span_n ? src[o + 2] : 0.f;
            v.w = o + 3 < span_n ? src[o + 3] : 0.f;
        }
        uint32_t *kr = skey + (o / kDecPer) * kKeyPitch + (o % kDecPer);
        kr[0] = o < span_n ? score_key(v.x) : 0u;
        kr[1] = o + 1 < span_n ? score_key(v.y) : 0u;
        kr[2] = o + 2 < span_n ? score_key(v.z) : 0u;
        kr[3] = o + 3 < span_n ? score_key(v.w) : 0u;
    }
    const int64_t t0 = span0 + (int64_t)tid * kDecPer;
    const int nv = T - t0 <= 0 ? 0 : (T - t0 >= kDecPer ? kDecPer : (int)(T - t0));
    auto key_at = [&](int j) { return skey[tid * kKeyPitch + j]; };
    // the row's histogram is complete in every CTA, and every thread's keys
    // are in place before their owners read them
    cl.sync();
    // this thread's 8 bins of the row's histogram (4088 - 8t .. 4095 - 8t)
    unsigned hc[8];
    {
        const uint4 *h4 = reinterpret_cast<const uint4 *>(sh.rowhist + kBins - 8 * (tid + 1));
        const uint4 x0 = h4[0], x1 = h4[1];
        hc[0] = x1.w; hc[1] = x1.z; hc[2] = x1.y; hc[3] = x1.x;
        hc[4] = x0.w; hc[5] = x0.z; hc[6] = x0.y; hc[7] = x0.x;
    }
    unsigned bin, above, n_group;
    find_rank_regs<8>(hc, kBins - 8 * tid - 1, (unsigned)m, &bin, &above, &n_group, sh);
    uint32_t prefix = bin;
    int pbits = kBits;
    unsigned rank = (unsigned)m - above;           // rank of tau within the group

    // too many keys to gather (rare: scores within a few percent of each
    // other, or many exact ties): 12-bit rounds over the register keys,
    // merged into CTA 0's histogram (clear on entry, cleared after each round)
    while (n_group > (unsigned)kDecCap && pbits < 32) {
        const int nb = 32 - pbits < kBits ? 32 - pbits : kBits;
        const int sh_lo = 32 - pbits - nb;
#pragma unroll 1
        for (int j = 0; j < nv; j++) {
            const uint32_t kj = key_at(j);
            if ((kj >> (32 - pbits)) == prefix)
                atomicAdd(&sh0->hist[(kj >> sh_lo) & ((1u << nb) - 1u)], 1u);
        }
        cl.sync();
        if (p == 0) {
            unsigned c8[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int b = kBins - 8 * tid - 1 - j;
                c8[j] = b < (1 << nb) ? sh.hist[b] : 0u;
            }
            unsigned b2, a2, n2;
            find_rank_regs<8>(c8, kBins - 8 * tid - 1, rank, &b2, &a2, &n2, sh);
            for (int i = tid; i < kBins; i += kDecThreads) sh.hist[i] = 0;
            if (tid < CN) {
                DecShared *r = cl.map_shared_rank(&sh, tid);
                r->res[0] = (prefix << nb) | b2;
                r->res[1] = (unsigned)(pbits + nb);
                r->res[2] = rank - a2;
                r->res[3] = n2;
            }
        }
        cl.sync();
        prefix = sh.res[0];
        pbits = (int)sh.res[1];
        rank = sh.res[2];
        n_group = sh.res[3];
    }

    // ---- this CTA's keys above the group and inside it; the group's keys
    // stored into a range of CTA 0's list (one atomic per CTA) when they are
    // few enough to gather
    const bool gather = n_group <= (unsigned)kDecCap && pbits < 32;
    const int gshift = 32 - pbits;
    // this thread's keys above the group and inside it, one bit per position
    uint32_t m_gt = 0, m_in = 0;
#pragma unroll 4
    for (int j = 0; j < nv; j++) {
        const uint32_t g = gshift == 32 ? 0u : key_at(j) >> gshift;
        m_gt |= (uint32_t)(g > prefix) << j;
        m_in |= (uint32_t)(g == prefix) << j;
    }
    const int n_gt = __popc(m_gt), n_in = __popc(m_in);
    // per warp: its counts added into CTA 0's per-CTA totals, and (when the
    // group is gathered) a range of CTA 0's list reserved with one atomic,
    // each lane's keys at its place within the warp's range
    int incl = n_in;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const int w_in = __shfl_sync(0xffffffffu, incl, 31);
    const int w_gt = warp_sum_first(n_gt, lane, 32);
    int wbase = 0;
    if (lane == 0) {
        if (w_gt) atomicAdd(&sh0->cnt_gt[p], w_gt);
        if (w_in) {
            atomicAdd(&sh0->cnt_in[p], w_in);
            if (gather) wbase = atomicAdd(&sh0->n_cand, w_in);
        }
    }
    if (gather && w_in) {
        int slot = __shfl_sync(0xffffffffu, wbase, 0) + incl - n_in;
        for (uint32_t mm = m_in; mm; mm &= mm - 1u) {
            const int j = __ffs(mm) - 1;
            if (slot < kDecCap) sh0->cand[slot] = make_uint2(key_at(j), (uint32_t)(t0 + j));
            slot++;
        }
    }
    cl.sync();                                   // counts and keys in CTA 0

    // ---- CTA 0: tau, q (tau-equal keys taken), every CTA's offset and quota
    if (p == 0) {
        uint32_t tau;
        int q;
        if (gather) {
            const int E = sh.n_cand < kDecCap ? sh.n_cand : kDecCap;
            uint32_t tp = prefix;
            int tb = pbits;
            unsigned rk = rank, cnt = n_group;
            while (tb < 32) {
                if (cnt <= (unsigned)kDecFew) {
                    // at most 32 keys share the prefix: one warp ranks them
                    const int sh_p = 32 - tb;
                    for (int j = tid; j < E; j += kDecThreads) {
                        const uint32_t k = sh.cand[j].x;
                        if ((k >> sh_p) == tp) {
                            const int f = atomicAdd(&sh.n_few, 1);
                            if (f < kDecFew) sh.few[f] = k;
                        }
                    }
                    __syncthreads();
                    if (warp == 0) {
                        const int n = sh.n_few < kDecFew ? sh.n_few : kDecFew;
                        const bool valid = lane < n;
                        const uint32_t kl = valid ? sh.few[lane] : 0u;
                        int gt = 0, eq = 0;
                        for (int i = 0; i < n; i++) {
                            const uint32_t ki = __shfl_sync(0xffffffffu, kl, i);
                            gt += ki > kl;
                            eq += ki == kl;
                        }
                        if (valid && (unsigned)gt < rk && (unsigned)(gt + eq) >= rk) {
                            sh.s_out[0] = kl;
                            sh.s_out[1] = rk - (unsigned)gt;
                        }
                    }
                    __syncthreads();
                    tp = sh.s_out[0];
                    rk = sh.s_out[1];
                    break;
                }
                const int nb = 32 - tb < 10 ? 32 - tb : 10;
                const int sh_lo = 32 - tb - nb;
                for (int i = tid; i < kDecSub; i += kDecThreads) sh.hist[i] = 0;
                __syncthreads();
                for (int j = tid; j < E; j += kDecThreads) {
                    const uint32_t k = sh.cand[j].x;
                    if ((k >> (32 - tb)) == tp) atomicAdd(&sh.hist[(k >> sh_lo) & ((1u << nb) - 1u)], 1u);
                }
                __syncthreads();
                // thread t: bins 1023 - 2t and 1022 - 2t (zero above the pass's range)
                unsigned c2[2];
#pragma unroll
                for (int j = 0; j < 2; j++) {
                    const int b = kDecSub - 2 * tid - 1 - j;
                    c2[j] = b < (1 << nb) ? sh.hist[b] : 0u;
                }
                unsigned b1, a1, n1;
                find_rank_regs<2>(c2, kDecSub - 2 * tid - 1, rk, &b1, &a1, &n1, sh);
                tp = (tp << nb) | b1;
                tb += nb;
                rk -= a1;
                cnt = n1;
            }
            tau = tp;
            q = (int)rk;
            // per CTA (a candidate's CTA is its position / kDecSpan): keys above
            // tau, and equal to it
            for (int j = tid; j < E; j += kDecThreads) {
                const uint2 cj = sh.cand[j];
                const int r = (int)(cj.y / (uint32_t)kDecSpan);
                if (cj.x > tau) atomicAdd(&sh.sel_gt[r], 1);
                else if (cj.x == tau) atomicAdd(&sh.sel_eq[r], 1);
            }
            __syncthreads();
        } else {
            // the group is one key value: its keys are all tau-equal
            tau = prefix;
            q = (int)rank;
        }
        if (warp == 0) {
            // exclusive prefix over the CTAs of (keys above tau, tau-equal keys)
            const bool in = lane < CN;
            const int gt_r = in ? sh.cnt_gt[lane] + (gather ? sh.sel_gt[lane] : 0) : 0;
            const int eq_r = in ? (gather ? sh.sel_eq[lane] : sh.cnt_in[lane]) : 0;
            int g = gt_r, e = eq_r;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int ng = __shfl_up_sync(0xffffffffu, g, o);
                const int ne = __shfl_up_sync(0xffffffffu, e, o);
                if (lane >= o) {
                    g += ng;
                    e += ne;
                }
            }
            if (in) {
                const int gt_below = g - gt_r, eq_below = e - eq_r;
                int my_q = q - eq_below;
                my_q = my_q < 0 ? 0 : (my_q > eq_r ? eq_r : my_q);
                DecShared *r = cl.map_shared_rank(&sh, lane);
                r->out[0] = tau;
                r->out[1] = (unsigned)(gt_below + (q < eq_below ? q : eq_below));
                r->out[2] = (unsigned)my_q;
            }
        }
    }
    cl.sync();                  // results delivered; no CTA touches another's memory after this
    const uint32_t tau = sh.out[0];
    const int off = (int)sh.out[1], my_q = (int)sh.out[2];

    // ---- ordered write of this thread's 32 positions: every key above the
    // group is above tau; of the group's keys (few), those above tau and the
    // lowest positions of the tau-equal ones within the quota
    uint32_t m_sel = m_gt, m_eq = 0;
    for (uint32_t mm = m_in; mm; mm &= mm - 1u) {
        const int j = __ffs(mm) - 1;
        const uint32_t kj = key_at(j);
        if (kj > tau) m_sel |= 1u << j;
        else if (kj == tau) m_eq |= 1u << j;
    }
    const int c_gt = __popc(m_sel), c_eq = __popc(m_eq);
    int2 tot2;
    const int2 e2 = block_scan2_dec(c_gt, c_eq, sh, &tot2);
    int take_eq = my_q - e2.y;
    take_eq = take_eq < 0 ? 0 : (take_eq > c_eq ? c_eq : take_eq);
    for (uint32_t mm = m_eq; take_eq > 0 && mm; mm &= mm - 1u, take_eq--) m_sel |= mm & (0u - mm);
    int pos = off + e2.x + (my_q < e2.y ? my_q : e2.y);
    for (uint32_t mm = m_sel; mm && pos < m; mm &= mm - 1u) {
        const int j = __ffs(mm) - 1;
        dst[pos++] = (int32_t)(t0 + j);
        pf(row, t0 + j);
    }
    for (int i = m + p * kDecThreads + tid; i < K; i += CN * kDecThreads) dst[i] = -1;
}

// One CTA per row, the row read from global memory (rows too long for the
// cluster kernel's shared memory).
__global__ void __launch_bounds__(kThreads)
topk_row_kernel(const float *__restrict__ scores, int S, int64_t T, int64_t start_pos, int K,
                int32_t *__restrict__ idx, int compress) {
    __shared__ unsigned hist[256];
    __shared__ int warp_tot[33];
    __shared__ unsigned s_sel, s_remaining;

    const int64_t row = blockIdx.x;
    const int64_t s = row % S;
    int64_t n_valid = (start_pos + s + 1) / compress;
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
                              int prefetch_row_bytes, const uint32_t *row_hist, int hist_chunks,
                              int compress) {
    if ((int64_t)B * S * T == 0) return DSA_OK;
    const int K = (int64_t)k < T ? k : (int)T;
    const int64_t rows = (int64_t)B * S;
    const int64_t avail_max = (start_pos + S) / compress;
    const int64_t n_max = T < avail_max ? T : avail_max;
    RowPrefetch pf;
    pf.base = static_cast<const uint8_t *>(prefetch_rows);
    pf.t_max = prefetch_t_max;
    pf.bytes = prefetch_row_bytes;
    if (row_hist && hist_chunks > 0 && compress == 1 && S == 1 && start_pos == T - 1 &&
        (T + kDecSpan - 1) / kDecSpan <= kMaxCluster) {
        // the decode top-k: one cluster per row, the threshold bin from the scorer's histogram
        const int dcn = (int)((T + kDecSpan - 1) / kDecSpan);
        const int dsmem = (int)sizeof(DecShared) + kDecThreads * kKeyPitch * (int)sizeof(uint32_t);
        if (cudaFuncSetAttribute(topk_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsmem) != cudaSuccess ||
            (dcn > 8 && cudaFuncSetAttribute(topk_decode_kernel,
                                             cudaFuncAttributeNonPortableClusterSizeAllowed,
                                             1) != cudaSuccess))
            return DSA_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(rows * dcn));
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = (size_t)dsmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)dcn;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        // programmatic launch: the set-up overlaps the scorer's tail
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        if (cudaLaunchKernelEx(&cfg, topk_decode_kernel, scores, T, K, idx, pf, row_hist,
                               hist_chunks) != cudaSuccess)
            return DSA_ERR_CUDA;
        return launch_status();
    }
    int cn, L;
    cluster_plan(n_max, &cn, &L);
    if (cn == 0) {
        topk_row_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(scores, S, T, start_pos, K, idx,
                                                                  compress);
        return launch_status();
    }
    // keys of the slice (padded) and the gathered keys with their positions
    const size_t smem = (size_t)(L + L / 32 + 1) * sizeof(uint32_t) + (size_t)kCap * 8;
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
    if (cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, S, T, start_pos, K, L, idx, pf,
                           compress) != cudaSuccess)
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

extern "C" dsa_status dsa_topk_select_csa(const float *scores, int B, int S, int64_t T,
                                          int64_t start_pos, int compress, int k, int32_t *idx,
                                          void *workspace, size_t workspace_bytes,
                                          dsa_stream_t stream) {
    if (B < 0 || S < 0 || T < 0 || start_pos < 0 || k < 1 || compress < 1)
        return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * S * T == 0) return DSA_OK;
    if (T > INT32_MAX || (start_pos + S) / compress > T) return DSA_ERR_INVALID_ARG;
    if ((int64_t)B * S * 16 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::topk_workspace_bytes(B, S, T, k);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DSA_ERR_WORKSPACE;
    return dsa::launch_topk_select(scores, B, S, T, start_pos, k, idx, workspace,
                                   reinterpret_cast<cudaStream_t>(stream), nullptr, 0, 0,
                                   nullptr, 0, compress);
}
