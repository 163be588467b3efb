// topk.cu -- per-query top-k selection over the causal positions.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward:
//   topk_indices = index_score.topk(min(index_topk, end_pos), dim=-1)[1]
// with the causal mask of "DeepSeek-V3.2-Exp - Causal mask" applied first.
// Rows with fewer causal positions than K are padded with -1 (the warm-up
// sentinel of the DeepSeek-V4 mask visualiser) instead of masked positions.
//
// Selection = exact radix select on order-preserving 32-bit keys:
//   pass p (p = 0..3) histograms byte (3-p) of the keys that match the
//   prefix chosen so far and keeps the bin holding the m-th largest key;
//   after four passes the threshold key tau and the number of tau-equal keys
//   still needed are known.  A final pass writes every position with
//   key > tau plus the first `need` positions with key == tau, in ascending
//   position order (block-wide ballot scans), so ties go to the lower
//   position and the output is deterministic.
#include "common.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Block-wide exclusive scan of a 0/1 flag; returns the exclusive prefix and
// writes the block total to *total.  All threads must call it.
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
        if (lane < kWarps) warp_tot[lane] = incl - v;   // exclusive
        if (lane == 31) warp_tot[32] = incl;
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    *total = warp_tot[32];
    __syncthreads();
    return r;
}

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

    if (m == n_valid) {                       // every causal position is selected
        for (int i = threadIdx.x; i < K; i += kThreads) dst[i] = i < m ? i : -1;
        return;
    }

    uint32_t prefix = 0, mask = 0;
    unsigned remaining = (unsigned)m;         // rank still to find among matching keys
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

}  // namespace

size_t topk_workspace_bytes(int, int, int64_t, int) { return 0; }

dsa_status launch_topk_select(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                              int k, int32_t *idx, void *, cudaStream_t stream) {
    if ((int64_t)B * S * T == 0) return DSA_OK;
    const int K = (int64_t)k < T ? k : (int)T;
    topk_row_kernel<<<(unsigned)(B * S), kThreads, 0, stream>>>(scores, S, T, start_pos, K, idx);
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
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::topk_workspace_bytes(B, S, T, k);
    if (need > 0 && (!workspace || workspace_bytes < need)) return DSA_ERR_WORKSPACE;
    return dsa::launch_topk_select(scores, B, S, T, start_pos, k, idx, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
}
