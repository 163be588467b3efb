// decode_step.cu -- one DSA decode step for a batch of sequences.
//
// Order of Indexer.forward ("DeepSeek-V3.2-Exp - Split indexer heads") with
// seqlen == 1 (no mask, "DeepSeek-V3.2-Exp - Causal mask"), followed by the
// diagram's sparse core attention in MQA mode:
//   rotate+quantise q and k_new, append k_new at T-1, fp8_index over the T
//   cached keys (one fused tensor-core kernel), top-min(index_topk, T), sparse
//   latent attention.
// Everything is enqueued on one stream; nothing synchronises with the host.
#include "common.cuh"

namespace dsa {
namespace {

struct DecodeWs {
    float *scores;     // [B,T]
    uint32_t *hist;    // [B][chunks][kHistBins]: each scorer CTA's scores counted by their
                       //   top 12 key bits
    int hist_chunks;
    void *attn_ws;
    size_t total;
};


DecodeWs carve(void *base, int B, int H, int D, int64_t T, int index_topk, int Hq, int dc, int dr,
               dsa_dtype dt) {
    DecodeWs w{};
    size_t off = 0;
    char *p = static_cast<char *>(base);
    auto take = [&](size_t bytes) {
        char *r = p ? p + off : nullptr;
        off = align_up(off + bytes, 256);
        return r;
    };
    w.scores = reinterpret_cast<float *>(take((size_t)B * T * sizeof(float)));
    // the scorer CTAs' histograms (each slot fully written every step)
    w.hist_chunks = decode_hist_chunks(B, H, D, T);
    w.hist = reinterpret_cast<uint32_t *>(
        take((size_t)B * w.hist_chunks * kHistBins * sizeof(uint32_t)));
    const int K = (int64_t)index_topk < T ? index_topk : (int)T;
    w.attn_ws = take(dt == DSA_FP8_LATENT ? sparse_mla_fp8_workspace_bytes(B, 1, Hq, dc, dr, K)
                                          : sparse_mla_workspace_bytes(B, 1, Hq, dc, dr, K, dt));
    w.total = off;
    return w;
}

}  // namespace
}  // namespace dsa

extern "C" size_t dsa_decode_step_workspace_size(int B, int H, int D, int64_t T, int index_topk,
                                                 int Hq, int dc, int dr, dsa_dtype dt) {
    if (B <= 0 || H <= 0 || T <= 0 || index_topk <= 0) return 0;
    return dsa::carve(nullptr, B, H, D, T, index_topk, Hq, dc, dr, dt).total;
}

extern "C" dsa_status dsa_decode_step(const float *q_idx, const float *w, const float *k_new,
                                      uint8_t *k_cache, float *k_scale, int64_t t_max,
                                      const void *kv_cache, const void *q_mla, int B, int H,
                                      int D, int Hq, int dc, int dr, int64_t T, int index_topk,
                                      float softmax_scale, float sm_scale, dsa_dtype dt,
                                      int32_t *idx, void *out, float *lse, void *workspace,
                                      size_t workspace_bytes, dsa_stream_t stream) {
    if (B < 0 || H < 1 || Hq < 1 || index_topk < 1 || T < 1 || T > t_max || T > INT32_MAX)
        return DSA_ERR_INVALID_ARG;
    if (dt != DSA_F32 && dt != DSA_BF16 && dt != DSA_FP8_LATENT) return DSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
    if (H > 256) return DSA_ERR_UNSUPPORTED;
    if (dc == 0 || dc % 32 != 0 || dc > 512 || dr < 0 || dr % 8 != 0 || dc + dr > 576)
        return DSA_ERR_UNSUPPORTED;
    if (dt == DSA_FP8_LATENT && !dsa::latent_fp8_shape_ok(dc, dr)) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (!q_idx || !w || !k_new || !k_cache || !k_scale || !kv_cache || !q_mla || !idx || !out)
        return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned16(q_idx) || !dsa::aligned16(k_new) || !dsa::aligned16(k_cache) ||
        !dsa::aligned16(kv_cache) || !dsa::aligned16(q_mla) || !dsa::aligned16(out) ||
        ((t_max * D) & 15))
        return DSA_ERR_INVALID_ARG;
    const dsa::DecodeWs ws = dsa::carve(workspace, B, H, D, T, index_topk, Hq, dc, dr, dt);
    if (!workspace || workspace_bytes < ws.total || !dsa::aligned16(workspace))
        return DSA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    dsa_status st;
    if ((st = dsa::launch_decode_scores(q_idx, w, k_new, k_cache, k_scale, t_max, B, H, D, T,
                                        softmax_scale, ws.scores, s, ws.hist)) != DSA_OK)
        return st;
    // (the attention prefetches its own rows into L2; a prefetch issued by the
    // top-k as it writes each position measured slower in the chained step)
    if ((st = dsa::launch_topk_select(ws.scores, B, 1, T, T - 1, index_topk, idx, nullptr, s,
                                      nullptr, 0, 0, ws.hist, ws.hist_chunks)) != DSA_OK)
        return st;
    const int K = (int64_t)index_topk < T ? index_topk : (int)T;
    if (dt == DSA_FP8_LATENT)
        return dsa::launch_sparse_mla_fp8(q_mla, static_cast<const uint8_t *>(kv_cache), t_max,
                                          idx, B, 1, Hq, dc, dr, K, T - 1, sm_scale, out, lse,
                                          ws.attn_ws, s);
    return dsa::launch_sparse_mla(q_mla, kv_cache, t_max, idx, B, 1, Hq, dc, dr, K, T - 1,
                                  sm_scale, dt, out, lse, ws.attn_ws, s);
}
