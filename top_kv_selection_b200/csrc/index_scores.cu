// index_scores.cu -- fp8_index scoring with the weight fold and the causal mask.
//
// Page: "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward, weight
// and scoring steps: the per-head weights are scaled by H^-1/2, by each
// head's query scale and by the indexer's softmax scale; fp8_index then
// scores every cached key, and the additive mask is applied.  The scoring
// formula is the one of the diagram "DeepSeek Sparse Attention, one decode
// step in one layer (V3.2 sizes)": a weighted sum over heads of the ReLU of
// the query-key dot products.
//
// Tensor-core scorer (sm_100a).  One CTA owns a contiguous range of 128-token
// tiles of one query row (b, s) and streams them once from HBM:
//   warp 0      TMA producer: 128 x D FP8 key tiles (swizzled) into a ring of
//               shared-memory stages, L2 evict-first;
//   warp 1      allocates TMEM and issues tcgen05.mma kind::f8f6f4 with
//               M = 128 tokens, N = heads (padded to 16), K = D in steps of 32,
//               accumulating fp32 in a double-buffered TMEM tile;
//   warps 2..5  epilogue: each thread owns one token (one TMEM lane), reads its
//               N head dot products, and computes
//               k_scale[t] * sum_h w'_h * max(dot_h, 0)  (ReLU, weighted head
//               sum, key scale), storing one fp32 score per token.
// The key cache is the only large operand: 132 bytes per token (D + 4).
//
// The producer starts streaming at once; the query operand is built in
// parallel by the epilogue warps, either from given FP8 codes or -- in the
// decode step -- by rotating and quantising the new token's fp32 queries
// (rotate_activation + act_quant, bit-identical to dsa_indexer_quant).  The
// fp32 query row arrives by TMA (swizzled boxes) right after the dependency
// wait, ahead of the key stream, and the rotation keeps 64 elements per lane
// so that it is almost all register arithmetic.  In the decode step the CTA
// holding position T-1 also quantises the new key and appends it to the cache
// (the cache write of Indexer.forward) before its last tile is fetched.
#include "common.cuh"
#include "quant.cuh"
#include "tc_ptx.cuh"
#include "scorer.cuh"
#include "tmap.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kMaxHeads = 256;

struct ScoreArgs {
    const uint8_t *q_fp8;      // query codes [rows, H, D] and scales, or ...
    const float *q_scale;
    const float *q_raw;        // ... the new token's fp32 queries [B, H, D] (decode)
    const float *k_new;        // decode: new key [B, D], appended at position T-1
    uint8_t *k_cache_w;
    float *k_scale_w;
    const float *w;
    const float *k_scale;
    float *scores;
    uint32_t *row_hist;        // decode: per (row, chunk) CTA, the histogram of its scores'
                               //   12-bit key bins ([rows][chunks][kHistBins], every bin
                               //   written), or null
    int64_t t_max;
    int64_t start_pos;
    int64_t T;
    int B, S, H, NH, chunks;
    int compress;              // keys are compressed entries of this many tokens (1: tokens)
    int q_copies;              // decode: the fp32 query row arrives in this many TMA boxes
    int q_box_bytes;           //   of this size into shared memory (0 boxes: direct loads)
    uint32_t tmem_cols;
    float head_scale, softmax_scale;
    int *err;
};

// Key-tile ring depth: the decode scorer gives one stage's shared memory to
// the histogram of its scores (two CTAs must still fit on an SM).
template <bool kRaw> constexpr int ring_stages() { return kRaw ? kStages - 1 : kStages; }
constexpr int kHistBits = 12;                      // top key bits the histogram resolves
static_assert(kHistBins == 1 << kHistBits, "histogram bins");

template <int D, bool kRaw>
__host__ __device__ constexpr size_t score_smem_bytes(int NH) {
    return 1024 + (size_t)ring_stages<kRaw>() * kTile * D + (size_t)NH * D +
           kMaxHeads * sizeof(float) + (2 * ring_stages<kRaw>() + 2 * kAcc + 3) * sizeof(uint64_t) +
           16 + (kRaw ? kHistBins * sizeof(uint32_t) : 0);
}

// Decode: the fp32 query row [H, D] of a sequence reaches shared memory as
// 8 KB TMA boxes of 64 rows x 128 bytes, 128-byte swizzled (16-byte chunk c of
// row r lands at chunk c ^ (r % 8)), so that the lanes of a head-slice read it
// back with at most two-way bank conflicts; global loads of 64 contiguous
// floats per lane would touch 32 cache lines per warp instruction.  Boxes 0
// and 1 land in the histogram's region, the rest in the last key stage.
constexpr int kQBoxRows = 64;
constexpr int kQBoxBytes = kQBoxRows * 128;

// Query operand (K-major, swizzled, padded heads zero) and folded weights
// w' = ((w * H^-1/2) * q_scale) * softmax_scale, built by the four epilogue
// warps.  G = D / 64 adjacent lanes own one head, 64 bytes of its row each, so
// one pass over the warps covers 4 * 32 / G heads.  The first pass's global
// loads are issued at kernel entry (QueryPrefetch), ahead of the key stream
// that would otherwise queue in front of them.
template <int D, bool kRaw> struct QueryPrefetch {
    static constexpr int G = D / 64;            // lanes per head
    static constexpr int kPass = 4 * 32 / G;    // heads per pass
    float r[kRaw ? 64 : 1];                     // fp32 query slice (decode)
    uint4 c[4];                                 // FP8 code slice (64 bytes)
    float w, qs;

    __device__ __forceinline__ static int head(int pass) {
        const int t = threadIdx.x - 64;
        return pass * kPass + (t >> 5) * (32 / G) + (t & 31) / G;
    }
    // the head's weight only (the query itself comes from shared memory)
    __device__ __forceinline__ void load_w(const ScoreArgs &a, int64_t row, int pass) {
        const int h = head(pass), part = (threadIdx.x - 64) % G;
        w = h < a.H && part == 0 ? a.w[row * a.H + h] : 0.f;
        qs = 0.f;
    }
    // this lane's 64 floats from the staged, swizzled query row (decode)
    __device__ __forceinline__ void load_staged(const ScoreArgs &a, const uint8_t *box01,
                                                const uint8_t *box2, int pass) {
        const int h = head(pass), part = (threadIdx.x - 64) % G;
        const bool ok = h < a.H;
        const int slice = h * G + part;             // 256-byte slice of the row
#pragma unroll
        for (int half = 0; half < 2; half++) {
            const int R = slice * 2 + half;         // 128-byte row of the query
            const int c = R / kQBoxRows, rr = R % kQBoxRows;
            const uint8_t *line = (c < 2 ? box01 + c * kQBoxBytes : box2 + (c - 2) * kQBoxBytes) +
                                  rr * 128;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float4 v = ok ? *reinterpret_cast<const float4 *>(line + ((j ^ (rr & 7)) << 4))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                float *d = r + 32 * half + 4 * j;
                d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
            }
        }
    }
    __device__ __forceinline__ void load(const ScoreArgs &a, int64_t row, int pass) {
        const int h = head(pass), part = (threadIdx.x - 64) % G;
        const bool ok = h < a.H;
        w = ok && part == 0 ? a.w[row * a.H + h] : 0.f;
        if constexpr (kRaw) {
            qs = 0.f;
            const float4 *src =
                reinterpret_cast<const float4 *>(a.q_raw + (row * a.H + h) * D + part * 64);
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const float4 v = ok ? src[j] : make_float4(0.f, 0.f, 0.f, 0.f);
                r[4 * j] = v.x; r[4 * j + 1] = v.y; r[4 * j + 2] = v.z; r[4 * j + 3] = v.w;
            }
        } else {
            qs = ok && part == 0 ? a.q_scale[row * a.H + h] : 0.f;
            const uint4 *src =
                reinterpret_cast<const uint4 *>(a.q_fp8 + (row * a.H + h) * D + part * 64);
#pragma unroll
            for (int j = 0; j < 4; j++) c[j] = ok ? src[j] : make_uint4(0, 0, 0, 0);
        }
    }
    // Rotates / quantises (decode) or copies (codes) the loaded slice into the
    // operand and writes the head's folded weight.
    __device__ __forceinline__ void store(const ScoreArgs &a, int pass, uint8_t *sq, float *wf) {
        const int h = head(pass), part = (threadIdx.x - 64) % G;
        float scale = qs;
        if constexpr (kRaw) {
            uint32_t codes[16];
            rotate_quant_lanes<D>(r, codes, &scale);
#pragma unroll
            for (int j = 0; j < 4; j++)
                c[j] = make_uint4(codes[4 * j], codes[4 * j + 1], codes[4 * j + 2],
                                  codes[4 * j + 3]);
        }
        if (h < a.NH) {
#pragma unroll
            for (int j = 0; j < 4; j++)
                *reinterpret_cast<uint4 *>(sq + h * D + KSwizzle<D>::chunk(h, part * 4 + j) * 16) =
                    c[j];
        }
        if (h < a.H && part == 0) {
            float x = __fmul_rn(w, a.head_scale);
            x = __fmul_rn(x, scale);
            wf[h] = __fmul_rn(x, a.softmax_scale);
        }
    }
};

// Decode: quantise the new key and append it at position T-1 of the cache
// (one warp, the lane layout of rotate_quant_warp); its TMA read follows.
template <int D>
__device__ __forceinline__ void append_key(const ScoreArgs &a, int64_t b, float (&kr)[D / 32],
                                           float *knew_scale, uint64_t *k_ready) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    float ks;
    const uint32_t packed = rotate_quant_warp<D>(kr, &ks);
    uint8_t *dst = a.k_cache_w + (b * a.t_max + a.T - 1) * D + lane * E;
    if constexpr (E == 4) *reinterpret_cast<uint32_t *>(dst) = packed;
    else *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(packed);
    if (lane == 0) {
        a.k_scale_w[b * a.t_max + a.T - 1] = ks;
        *knew_scale = ks;
    }
    // the key row is read next by TMA (async proxy)
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(k_ready);
}

template <int D, bool kRaw>
__global__ void __launch_bounds__(kThreads, 2)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_q, const ScoreArgs a) {
    constexpr int NS = ring_stages<kRaw>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sk = smem;
    uint8_t *sq = sk + NS * kTile * D;
    // decode: histogram of this CTA's scores by the top 12 bits of their key
    // (1024-byte aligned: before the query operand is built it holds the
    // first two boxes of the staged fp32 query row)
    uint32_t *s_hist = reinterpret_cast<uint32_t *>(sq + a.NH * D);
    float *wf = reinterpret_cast<float *>(sq + a.NH * D + (kRaw ? kHistBins * sizeof(uint32_t) : 0));
    uint64_t *full = reinterpret_cast<uint64_t *>(wf + kMaxHeads);
    uint64_t *empty = full + NS;
    uint64_t *accf = empty + NS;
    uint64_t *acce = accf + kAcc;
    uint64_t *q_ready = acce + kAcc, *k_ready = q_ready + 1, *q_full = k_ready + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(q_full + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    float *knew_scale = reinterpret_cast<float *>(tmem_holder + 2);
    // decode with a staged query: its boxes 2.. occupy the last key stage
    // until the query operand is built
    const bool staged = kRaw && a.q_copies > 0;
    uint8_t *q_box01 = reinterpret_cast<uint8_t *>(s_hist);
    uint8_t *q_box2 = sk + (NS - 1) * kTile * D;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // causal rows are taken longest first (query s = S-1 of every sequence,
    // then S-2, ...), so the short rows fill the last wave
    const int64_t ri = blockIdx.x / a.chunks;
    const int chunk = blockIdx.x - (int)(ri * a.chunks);
    const int64_t b = ri % a.B, s = a.S - 1 - ri / a.B;
    const int64_t row = b * a.S + s;
    // keys visible to this query: positions <= start_pos + s, or with compressed
    // entries of m tokens, the entries whose m tokens are all in
    const int64_t avail = (a.start_pos + s + 1) / (a.compress > 1 ? a.compress : 1);
    const int64_t n_vis = a.T < avail ? a.T : avail;
    const int64_t n_tiles = (n_vis + kTile - 1) / kTile;
    const int64_t tile_lo = chunk * n_tiles / a.chunks;
    const int64_t tile_hi = (chunk + 1) * n_tiles / a.chunks;
    const int n_my = (int)(tile_hi - tile_lo);
    // decode: this CTA appends the new key if its last tile holds position T-1
    const bool append = kRaw && n_my > 0 && tile_hi == n_tiles;

    // a kernel launched after this one (the top-k) may be scheduled now; it
    // waits for this grid before reading the scores
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // causally masked positions of this row (prefill only), shared by the chunks
    auto write_masked = [&]() {
        for (int64_t t = n_vis + (int64_t)chunk * kThreads + threadIdx.x; t < a.T;
             t += (int64_t)a.chunks * kThreads)
            a.scores[row * a.T + t] = -INFINITY;
    };
    if (n_my <= 0) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        write_masked();
        // no tiles: an empty histogram for this CTA's slot
        if (kRaw && a.row_hist)
            for (int i = threadIdx.x; i < kHistBins; i += kThreads)
                a.row_hist[(row * a.chunks + chunk) * kHistBins + i] = 0u;
        return;
    }

    using Prefetch = QueryPrefetch<D, kRaw>;
    Prefetch pf;
    float kr[D / 32];
    const int tok = (warp & 3) * 32 + lane;       // token within a tile (epilogue)
    const float *ks_row = a.k_scale + b * a.t_max;
    // key scales are loaded three tiles ahead so their HBM latency is hidden
    auto load_ks = [&](int ii) -> float {
        const int64_t tt = (tile_lo + ii) * kTile + tok;
        if (ii >= n_my || tt >= n_vis) return 0.f;
        return (append && tt == a.T - 1) ? *knew_scale : ld_cg_f32(ks_row + tt);
    };
    // the epilogue warp whose tokens include position T-1 appends the new key,
    // so the key's scale passes between lanes of one warp
    const bool appender = append && warp >= 2 && (warp & 3) == (int)(((a.T - 1) % kTile) >> 5);
    float ks0 = 0.f, ks1 = 0.f, ks2 = 0.f;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < kAcc; i++) {
            tc::mbar_init(&accf[i], 1);
            tc::mbar_init(&acce[i], 4 * 32);
        }
        tc::mbar_init(q_ready, 4 * 32);
        tc::mbar_init(k_ready, 1);
        tc::mbar_init(q_full, 1);
        *abort = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap_k);
        if (staged) tc::tma_prefetch_desc(&tmap_q);
    }
    __syncthreads();        // the barriers are initialised
    // The accumulators: warp 1 allocates them while the epilogue warps build
    // the query operand; the two meet at named barrier 3 (warps 1..5) before
    // either touches TMEM.  Allocation is the last thing done before the wait
    // below, so with a programmatic launch it overlaps the preceding kernel.
    if (warp == 1) {
        tc::tmem_alloc(tmem_holder, a.tmem_cols);
        tc::tmem_relinquish();
    }
    // Everything below reads the step's inputs (queries, weights, the key
    // cache) or writes its outputs: wait for the preceding kernel (a no-op
    // without a programmatic launch).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    write_masked();
    // the staged query row first, ahead of every other request of the CTA
    if (staged && threadIdx.x == 0) {
        tc::mbar_arrive_expect_tx(q_full, (uint32_t)(a.q_copies * a.q_box_bytes));
        const uint64_t keep = tc::l2_evict_last_policy();   // every chunk of the row reads it
        for (int c = 0; c < a.q_copies; c++)
            tc::tma_load_3d(c < 2 ? q_box01 + c * kQBoxBytes : q_box2 + (c - 2) * kQBoxBytes,
                            &tmap_q, 0, c * kQBoxRows, (int)b, q_full, keep);
    }
    // epilogue warps: issue the query (unless staged), weight, first key-scale
    // and new-key loads before the key stream starts (named barrier 4, warps 0
    // and 2..5: the first ring of key tiles is issued only after them, so that
    // these loads are not queued behind every CTA's ring in HBM)
    if (warp >= 2) {
        if (staged) pf.load_w(a, row, 0);
        else pf.load(a, row, 0);
        if (appender) load_lane_slice<D, float>(a.k_new + b * D, kr);
        ks0 = load_ks(0);     // the new key's entry is reloaded once it is appended
        ks1 = load_ks(1);
        ks2 = load_ks(2);
    }
    if (warp != 1) asm volatile("bar.sync 4, 160;" ::: "memory");
    // the first ring of key tiles (the tile holding the appended key waits
    // for it in the loop below; with a staged query the last stage waits
    // until the query operand is built)
    const int ring0 = staged ? NS - 1 : NS;
    const int early = n_my - (append ? 1 : 0) < ring0 ? n_my - (append ? 1 : 0) : ring0;
    const uint64_t pol = tc::l2_evict_first_policy();
    if (threadIdx.x == 0)
        for (int i = 0; i < early; i++) {
            tc::mbar_arrive_expect_tx(&full[i], kTile * D);
            tc::tma_load_3d(sk + i * kTile * D, &tmap_k, 0, (int)((tile_lo + i) * kTile), (int)b,
                            &full[i], pol);
        }
    uint32_t tmem_base = 0;
    if (warp == 1) {
        tc::tc_fence_before();
        asm volatile("bar.sync 3, 160;" ::: "memory");
        tc::tc_fence_after();
        tmem_base = *tmem_holder;
    }

    if (warp == 0) {
        if (lane == 0) {
            int issued = early;
            for (int i = early; i < n_my; i++) {
                const int st = i % NS;
                const uint32_t ph = (uint32_t)(i / NS) & 1u;
                if (!tc::mbar_wait(&empty[st], ph ^ 1u, a.err, abort)) break;
                if (staged && i == NS - 1 && !tc::mbar_wait(q_ready, 0, a.err, abort)) break;
                if (append && i == n_my - 1 && !tc::mbar_wait(k_ready, 0, a.err, abort)) break;
                tc::mbar_arrive_expect_tx(&full[st], kTile * D);
                tc::tma_load_3d(sk + st * kTile * D, &tmap_k, 0, (int)((tile_lo + i) * kTile),
                                (int)b, &full[st], pol);
                issued = i + 1;
            }
            // wait (bounded) for the last loads still landing in shared memory
            for (int j = issued > NS ? issued - NS : 0; j < issued; j++)
                tc::mbar_wait(&full[j % NS], (uint32_t)(j / NS) & 1u, a.err, abort);
            if (staged) tc::mbar_wait(q_full, 0, a.err, abort);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::instr_desc(tc::kFmtE4M3, tc::kFmtE4M3, kTile, a.NH);
            const uint32_t sk_addr = tc::smem_u32(sk), sq_addr = tc::smem_u32(sq);
            const bool q_ok = tc::mbar_wait(q_ready, 0, a.err, abort);
            for (int i = 0; q_ok && i < n_my; i++) {
                const int st = i % NS, ac = i % kAcc;
                if (!tc::mbar_wait(&full[st], (uint32_t)(i / NS) & 1u, a.err, abort)) break;
                if (!tc::mbar_wait(&acce[ac], ((uint32_t)(i / kAcc) & 1u) ^ 1u, a.err, abort))
                    break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(ac * a.NH);
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
        for (int pass = 0; pass * Prefetch::kPass < a.NH; pass++) {
            if constexpr (kRaw) {
                if (staged) {
                    if (pass > 0) pf.load_w(a, row, pass);
                    if (tc::mbar_wait(q_full, 0, a.err, abort)) {
                        pf.load_staged(a, q_box01, q_box2, pass);
                    } else {
#pragma unroll
                        for (int e = 0; e < 64; e++) pf.r[e] = 0.f;
                    }
                } else if (pass > 0) {
                    pf.load(a, row, pass);
                }
            } else {
                if (pass > 0) pf.load(a, row, pass);
            }
            pf.store(a, pass, sq, wf);
        }
        for (int h = a.H + (threadIdx.x - 64); h < kMaxHeads; h += 128) wf[h] = 0.f;
        tc::fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");   // folded weights of all heads
        tc::mbar_arrive(q_ready);
        if (appender) {
            append_key<D>(a, b, kr, knew_scale, k_ready);
            __syncwarp();
            ks0 = load_ks(0);
            ks1 = load_ks(1);
            ks2 = load_ks(2);
        }
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        float *out = a.scores + row * a.T;
        const bool hist = kRaw && a.row_hist != nullptr;
        if (hist) {
            for (int i = threadIdx.x - 64; i < kHistBins; i += 128) s_hist[i] = 0;
            asm volatile("bar.sync 2, 128;" ::: "memory");
        }
        // the accumulators' TMEM address, from warp 1
        asm volatile("bar.sync 3, 160;" ::: "memory");
        tc::tc_fence_after();
        tmem_base = *tmem_holder;
        for (int i = 0; i < n_my; i++) {
            const int ac = i % kAcc;
            const int64_t t = (tile_lo + i) * kTile + tok;
            const float ks = ks0;
            ks0 = ks1;
            ks1 = ks2;
            ks2 = load_ks(i + 3);
            if (!tc::mbar_wait(&accf[ac], (uint32_t)(i / kAcc) & 1u, a.err, abort)) break;
            tc::tc_fence_after();
            const uint32_t taddr = tmem_base + lane_addr + (uint32_t)(ac * a.NH);
            // four independent partial sums keep the FMA chain short
            float acc4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c0 = 0; c0 < a.NH; c0 += 64) {
                uint32_t r[4][16];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    if (c0 + 16 * j < a.NH) tc::tmem_ld16(taddr + c0 + 16 * j, r[j]);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    if (c0 + 16 * j >= a.NH) break;
                    const float4 *w4 = reinterpret_cast<const float4 *>(wf + c0 + 16 * j);
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float4 wv = w4[e];
                        acc4[0] = fmaf(wv.x, fmaxf(__uint_as_float(r[j][4 * e + 0]), 0.f), acc4[0]);
                        acc4[1] = fmaf(wv.y, fmaxf(__uint_as_float(r[j][4 * e + 1]), 0.f), acc4[1]);
                        acc4[2] = fmaf(wv.z, fmaxf(__uint_as_float(r[j][4 * e + 2]), 0.f), acc4[2]);
                        acc4[3] = fmaf(wv.w, fmaxf(__uint_as_float(r[j][4 * e + 3]), 0.f), acc4[3]);
                    }
                }
            }
            const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
            tc::tc_fence_before();
            tc::mbar_arrive(&acce[ac]);
            if (t < n_vis) {
                const float sc = ks * acc;
                out[t] = sc;
                if (hist) atomicAdd(&s_hist[score_key(sc) >> (32 - kHistBits)], 1u);
            }
        }
        if (hist) {
            // this CTA's histogram, every bin, into its own slot (nothing has
            // to be zeroed before the launch; the top-k sums a row's slots)
            asm volatile("bar.sync 2, 128;" ::: "memory");
            uint32_t *rh = a.row_hist + (row * a.chunks + chunk) * kHistBins;
            for (int i = threadIdx.x - 64; i < kHistBins; i += 128) rh[i] = s_hist[i];
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, a.tmem_cols);
    }
}

uint32_t pow2_cols(int n) {
    uint32_t c = 32;
    while (c < (uint32_t)n) c <<= 1;
    return c;
}

// CTAs per query row: enough to fill the SMs once (two per SM when their
// shared memory and TMEM allow), at most one per 128-token tile.
template <int D, bool kRaw>
int score_chunks(int64_t rows, int NH, int64_t vis_max) {
    const size_t smem = score_smem_bytes<D, kRaw>(NH);
    const int per_sm = smem * 2 <= 227 * 1024 && pow2_cols(kAcc * NH) <= 256 ? 2 : 1;
    const int64_t max_tiles = (vis_max + kTile - 1) / kTile;
    int64_t chunks = (int64_t)num_sms() * per_sm / rows;
    if (chunks > max_tiles) chunks = max_tiles;
    if (chunks < 1) chunks = 1;
    return (int)chunks;
}

template <int D, bool kRaw>
dsa_status launch_tc(ScoreArgs a, const uint8_t *k_cache, int B, int S, int64_t start_pos,
                     int64_t T, cudaStream_t stream) {
    CUtensorMap tmap, tmap_q;
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.t_max, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)D, (uint64_t)a.t_max * D};
    const uint32_t box[3] = {(uint32_t)D, (uint32_t)kTile, 1};
    const CUtensorMapSwizzle swz =
        D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    if (!encode_tmap(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k_cache, dims, strides, box, swz))
        return DSA_ERR_CUDA;
    tmap_q = tmap;      // unused unless the decode query is staged
    a.q_copies = 0;
    if (kRaw) {
        // the query row [H, D] fp32 as rows of 128 bytes; staged when its
        // boxes fit the histogram region (2 boxes) and the last key stage
        const int64_t q_rows = (int64_t)a.H * D / 32;
        const int64_t copies = (q_rows + kQBoxRows - 1) / kQBoxRows;
        const int64_t room = 2 + (int64_t)kTile * D / kQBoxBytes;
        if (copies <= room) {
            const uint64_t qd[3] = {32, (uint64_t)q_rows, (uint64_t)B};
            const uint64_t qs[2] = {128, (uint64_t)q_rows * 128};
            const uint32_t box_rows = (uint32_t)(q_rows < kQBoxRows ? q_rows : kQBoxRows);
            const uint32_t qb[3] = {32, box_rows, 1};
            if (!encode_tmap(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.q_raw, qd, qs, qb,
                             CU_TENSOR_MAP_SWIZZLE_128B))
                return DSA_ERR_CUDA;
            a.q_copies = (int)copies;
            a.q_box_bytes = (int)box_rows * 128;
        }
    }
    a.start_pos = start_pos;
    a.T = T;
    a.B = B;
    a.S = S;
    a.NH = (a.H + 15) / 16 * 16;
    a.tmem_cols = pow2_cols(kAcc * a.NH);
    a.head_scale = (float)(1.0 / sqrt((double)a.H));
    a.err = device_error_word();

    const size_t smem = score_smem_bytes<D, kRaw>(a.NH);
    const int64_t rows = (int64_t)B * S;
    const int64_t avail_max = (start_pos + S) / (a.compress > 1 ? a.compress : 1);
    const int64_t vis_max = T < avail_max ? T : avail_max;
    a.chunks = score_chunks<D, kRaw>(rows, a.NH, vis_max);
    const int64_t chunks = a.chunks;
    if (cudaFuncSetAttribute(score_tc_kernel<D, kRaw>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DSA_ERR_CUDA;
    // programmatic launch: the CTAs' set-up (barriers, TMEM) overlaps the
    // preceding kernel's tail; the kernel waits for it before touching memory
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * chunks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, score_tc_kernel<D, kRaw>, tmap, tmap_q, a) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace

dsa_status launch_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                               const uint8_t *k_cache, const float *k_scale, int64_t t_max, int B,
                               int S, int H, int D, int64_t start_pos, int64_t T,
                               float softmax_scale, float *scores, cudaStream_t stream,
                               int compress) {
    if ((int64_t)B * S * T == 0) return DSA_OK;
    ScoreArgs a = {};
    a.q_fp8 = q_fp8;
    a.q_scale = q_scale;
    a.w = w;
    a.k_scale = k_scale;
    a.scores = scores;
    a.t_max = t_max;
    a.H = H;
    a.softmax_scale = softmax_scale;
    a.compress = compress;
    if (compress == 1 && prefill_group_rows(B, S, H))
        return launch_prefill_scores(q_fp8, q_scale, w, k_cache, k_scale, t_max, B, S, H, D,
                                     start_pos, T, softmax_scale, scores, stream);
    return D == 128 ? launch_tc<128, false>(a, k_cache, B, S, start_pos, T, stream)
                    : launch_tc<64, false>(a, k_cache, B, S, start_pos, T, stream);
}

int decode_hist_chunks(int B, int H, int D, int64_t T) {
    if (B <= 0 || T <= 0) return 0;
    const int NH = (H + 15) / 16 * 16;
    return D == 128 ? score_chunks<128, true>(B, NH, T) : score_chunks<64, true>(B, NH, T);
}

dsa_status launch_decode_scores(const float *q_raw, const float *w, const float *k_new,
                                uint8_t *k_cache, float *k_scale, int64_t t_max, int B, int H,
                                int D, int64_t T, float softmax_scale, float *scores,
                                cudaStream_t stream, uint32_t *row_hist) {
    if ((int64_t)B * T == 0) return DSA_OK;
    ScoreArgs a = {};
    a.row_hist = row_hist;
    a.q_raw = q_raw;
    a.k_new = k_new;
    a.k_cache_w = k_cache;
    a.k_scale_w = k_scale;
    a.w = w;
    a.k_scale = k_scale;
    a.scores = scores;
    a.t_max = t_max;
    a.H = H;
    a.softmax_scale = softmax_scale;
    a.compress = 1;
    return D == 128 ? launch_tc<128, true>(a, k_cache, B, 1, T - 1, T, stream)
                    : launch_tc<64, true>(a, k_cache, B, 1, T - 1, T, stream);
}

}  // namespace dsa

extern "C" dsa_status dsa_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                                       const uint8_t *k_cache, const float *k_scale,
                                       int64_t t_max, int B, int S, int H, int D,
                                       int64_t start_pos, int64_t T, float softmax_scale,
                                       float *scores, dsa_stream_t stream) {
    if (B < 0 || S < 0 || T < 0 || start_pos < 0 || H < 1) return DSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
    if (H > 256) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S * T == 0) return DSA_OK;
    if (T > t_max || start_pos + S > T) return DSA_ERR_INVALID_ARG;
    if (t_max > INT32_MAX || B > 65535 || (int64_t)B * S > INT32_MAX / 512)
        return DSA_ERR_UNSUPPORTED;
    if (!q_fp8 || !q_scale || !w || !k_cache || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q_fp8) || !dsa::aligned16(k_cache)) return DSA_ERR_INVALID_ARG;
    return dsa::launch_index_scores(q_fp8, q_scale, w, k_cache, k_scale, t_max, B, S, H, D,
                                    start_pos, T, softmax_scale, scores,
                                    reinterpret_cast<cudaStream_t>(stream), 1);
}

extern "C" dsa_status dsa_index_scores_csa(const uint8_t *q_fp8, const float *q_scale,
                                           const float *w, const uint8_t *k_cache,
                                           const float *k_scale, int64_t t_max, int B, int S,
                                           int H, int D, int64_t start_pos, int64_t T,
                                           int compress, float softmax_scale, float *scores,
                                           dsa_stream_t stream) {
    if (B < 0 || S < 0 || T < 0 || start_pos < 0 || H < 1 || compress < 1)
        return DSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
    if (H > 256) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)B * S * T == 0) return DSA_OK;
    // every entry the last query may see must be in the cache
    if (T > t_max || (start_pos + S) / compress > T) return DSA_ERR_INVALID_ARG;
    if (t_max > INT32_MAX || B > 65535 || (int64_t)B * S > INT32_MAX / 512)
        return DSA_ERR_UNSUPPORTED;
    if (!q_fp8 || !q_scale || !w || !k_cache || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q_fp8) || !dsa::aligned16(k_cache)) return DSA_ERR_INVALID_ARG;
    return dsa::launch_index_scores(q_fp8, q_scale, w, k_cache, k_scale, t_max, B, S, H, D,
                                    start_pos, T, softmax_scale, scores,
                                    reinterpret_cast<cudaStream_t>(stream), compress);
}

extern "C" dsa_status dsa_decode_index_scores(const float *q_idx, const float *w,
                                              const float *k_new, uint8_t *k_cache,
                                              float *k_scale, int64_t t_max, int B, int H, int D,
                                              int64_t T, float softmax_scale, float *scores,
                                              dsa_stream_t stream) {
    if (B < 0 || T < 1 || H < 1 || T > t_max) return DSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
    if (H > 256 || t_max > INT32_MAX || B > 65535) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (!q_idx || !w || !k_new || !k_cache || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q_idx) || !dsa::aligned16(k_new) || !dsa::aligned16(k_cache) ||
        ((t_max * D) & 15))
        return DSA_ERR_INVALID_ARG;
    return dsa::launch_decode_scores(q_idx, w, k_new, k_cache, k_scale, t_max, B, H, D, T,
                                     softmax_scale, scores, reinterpret_cast<cudaStream_t>(stream));
}
