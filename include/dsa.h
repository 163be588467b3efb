/*
 * dsa.h -- C ABI of libdsa: the data-parallel hot path of DeepSeek Sparse
 * Attention on NVIDIA B200 (sm_100a).
 *
 * The path (lightning indexer, top-k token selection, sparse latent attention)
 * follows these pages:
 *   "DeepSeek-V3.2-Exp - Split indexer heads": the Indexer.forward excerpt:
 *       the non-interleaved rotary embedding of q_pe / k_pe, rotate_activation,
 *       act_quant (with its scale_fmt), the key-cache write, the weight fold,
 *       fp8_index, the additive mask and the top-k of min(index_topk, end_pos)
 *       positions.
 *   "DeepSeek-V3.2-Exp - Causal mask": Transformer.forward (a -inf mask above
 *       the diagonal when more than one token is new) and the MLA prefill
 *       excerpt (an index mask, -inf except at the selected positions, plus
 *       that causal mask).
 *   "DeepSeek Sparse Attention, one decode step in one layer (V3.2 sizes)"
 *       diagram: I(t,s) = sum_j w_j ReLU(q_j . k_s), k = 2048, core attention
 *       in MQA mode over the gathered latents, each latent row key and value,
 *       latents cached as "FP8 + bf16 RoPE" in 656-byte rows.
 *
 * Conventions for every entry point:
 *   - Memory: every tensor argument is a caller-owned DEVICE pointer, row-major
 *     and contiguous with the layout stated below, 16-byte aligned unless the
 *     entry point states a weaker alignment.  The library allocates nothing.  Scratch memory is passed in as `workspace`
 *     (size from the matching *_workspace_size call); it need not be zeroed.
 *   - Execution: every call only enqueues kernels on `stream` and returns; it
 *     never synchronises.  Calls on one stream run in order.  Two calls that
 *     share a workspace must not run concurrently.
 *   - Errors: argument checks run on the host before anything is launched and
 *     return DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED / DSA_ERR_WORKSPACE with
 *     nothing enqueued.  A failed launch returns DSA_ERR_CUDA.  Problems found
 *     on the device (an index out of range) never trap: the kernel skips the
 *     access and records a code in a sticky device word that
 *     dsa_get_device_error() reads.
 *   - Empty problems (a zero batch or zero vectors) return DSA_OK without a
 *     launch.
 *   - Indices are int32; -1 marks an empty selection slot.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *dsa_stream_t;

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer  */
    DSA_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. D not 64 or 128)  */
    DSA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed        */
    DSA_ERR_TIMEOUT = 4,       /* a bounded device-side wait expired          */
    DSA_ERR_DEVICE = 5,        /* device-side check failed (see device word)  */
    DSA_ERR_WORKSPACE = 6      /* workspace missing or smaller than required  */
} dsa_status;

typedef enum dsa_dtype {
    DSA_F32 = 0,               /* IEEE binary32 */
    DSA_BF16 = 1,              /* bfloat16      */
    /* The FP8 latent cache layout of dsa_latent_row_bytes (656-byte rows at
     * the V3.2 sizes).  Accepted only by dsa_decode_step(_noalloc) as the
     * kv_cache type; q_mla and out are then bf16. */
    DSA_FP8_LATENT = 2
} dsa_dtype;

/* act_quant's scale_fmt: a plain fp32 scale, or ue8m0 (a bare power of two). */
typedef enum dsa_scale_fmt {
    DSA_SCALE_F32 = 0,
    DSA_SCALE_UE8M0 = 1
} dsa_scale_fmt;

/* Text for a status code (static storage, never NULL). */
const char *dsa_status_string(dsa_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
int dsa_version(void);

/*
 * Waits for `stream`, then returns in *device_status the first code a kernel
 * of this library recorded on the current device since the last call (DSA_OK
 * if none) and clears it.  Returns DSA_ERR_INVALID_ARG if device_status is
 * NULL, DSA_ERR_CUDA if the wait or the read fails.
 */
dsa_status dsa_get_device_error(dsa_stream_t stream, int32_t *device_status);

/*
 * Diagnostic of the bounded device waits (failure detection; the pages have
 * no counterpart).  Every wait of this library's kernels on a barrier (a TMA
 * load, a tensor-core commit, a peer CTA) gives up after a budget of SM clock
 * cycles, records DSA_ERR_TIMEOUT in the device word above and lets the kernel
 * return normally: no trap, and the context stays usable.  This call launches
 * one CTA that waits through that same routine on a shared-memory barrier,
 * with a budget of budget_cycles (1 .. 2e9, about a second at 2 GHz, the
 * budget the kernels use).  With complete = 0 nobody arrives, so the wait
 * expires after about budget_cycles and DSA_ERR_TIMEOUT is recorded; with
 * complete != 0 the barrier completes at once and nothing is recorded.
 * Returns DSA_ERR_INVALID_ARG for a budget outside that range (nothing
 * launched), DSA_ERR_CUDA if the launch fails.
 */
dsa_status dsa_wait_selftest(int64_t budget_cycles, int complete, dsa_stream_t stream);

/*
 * rotate_activation + act_quant (Indexer.forward, "Split indexer heads"):
 * each d-vector is rotated by the orthonormal Walsh-Hadamard transform
 * (butterflies in fp32 with strides 1, 2, ..., d/2, then one multiply by
 * fp32(d^-1/2)) and quantised to FP8 e4m3 with one scale per vector:
 * scale = max(amax, 1e-4) / 448, code = e4m3_rn_satfinite(x / scale), both
 * divisions correctly rounded.
 *
 *   x          [n_rows, n_vec, d]  F32 or BF16 (x_dtype), contiguous
 *   out_fp8    vector (r, v) -> out_fp8 + r * out_row_stride + v * d  (bytes)
 *   out_scale  vector (r, v) -> out_scale + r * scale_row_stride + v  (floats)
 *
 * Queries: n_rows = 1, n_vec = B*S*H, strides unused (pass 0).
 * Keys appended to a cache k_cache[B, t_max, d] / k_scale[B, t_max] at
 * start_pos: x = keys[B, S, d], n_rows = B, n_vec = S, out_fp8 = k_cache +
 * start_pos * d, out_row_stride = t_max * d, out_scale = k_scale + start_pos,
 * scale_row_stride = t_max.
 * d must be 64 or 128 (else DSA_ERR_UNSUPPORTED).  out_row_stride must be a
 * multiple of 16 when n_rows > 1.
 */
dsa_status dsa_indexer_quant(const void *x, dsa_dtype x_dtype, int64_t n_rows, int64_t n_vec,
                             int d, uint8_t *out_fp8, int64_t out_row_stride, float *out_scale,
                             int64_t scale_row_stride, dsa_stream_t stream);

/*
 * The indexer's query and key preparation in one pass (Indexer.forward,
 * "Split indexer heads": split off the first rope_head_dim elements, rotary
 * embedding with interleaved = False, concatenate, rotate_activation,
 * act_quant(x, block_size, scale_fmt), k_cache / k_scale_cache append at
 * start_pos .. start_pos + S - 1).
 * Rotary part, for every query head vector and key vector: element j and
 * element j + rope_dim/2 (j < rope_dim/2) are the real and imaginary parts of
 * one complex number, multiplied by rope_cs[s][j] = (cos, sin) of the token's
 * angle for frequency j: x1' = x1*c - x2*s, x2' = x1*s + x2*c, each product
 * and sum rounded to fp32 (bf16 inputs are widened to fp32 first; the result
 * stays fp32).  Then rotation and quantisation as dsa_indexer_quant, except
 * that with DSA_SCALE_UE8M0 the scale max(amax, 1e-4) / 448 is rounded up to
 * the smallest power of two not below it.
 *
 *   q        [B,S,H,d] F32 or BF16 (x_dtype), contiguous, 16-byte aligned
 *   k        [B,S,d]   same dtype, contiguous, 16-byte aligned
 *   rope_cs  [S, rope_dim/2, 2] fp32, 16-byte aligned: row s is the angle of
 *            position start_pos + s (the caller's freqs_cis[start_pos + s] as
 *            (re, im)); unused (may be NULL) when rope_dim = 0
 *   q_fp8    [B,S,H,d] e4m3 codes (16-byte aligned), q_scale [B,S,H] fp32
 *   k_cache  [B,t_max,d] e4m3 codes (16-byte aligned), k_scale [B,t_max] fp32:
 *            rows start_pos .. start_pos + S - 1 of each sequence are
 *            written, nothing else
 * d must be 64 or 128 and rope_dim one of 0, 8, 16, 32, 64 (or 128 when
 * d = 128), else DSA_ERR_UNSUPPORTED; start_pos + S <= t_max, else
 * DSA_ERR_INVALID_ARG, as are NULL or misaligned buffers.  H may be 0 (keys
 * only; q, q_fp8 and q_scale may then be NULL).  All buffers are caller-owned
 * device memory; the call is asynchronous on `stream`.
 */
dsa_status dsa_indexer_prologue(const void *q, const void *k, dsa_dtype x_dtype, int B, int S,
                                int H, int d, int rope_dim, const float *rope_cs,
                                dsa_scale_fmt scale_fmt, int64_t start_pos, int64_t t_max,
                                uint8_t *q_fp8, float *q_scale, uint8_t *k_cache,
                                float *k_scale, dsa_stream_t stream);

/*
 * The FP8 latent cache ("DeepSeek Sparse Attention, one decode step in one
 * layer (V3.2 sizes)": latents stored as "FP8 + bf16 RoPE", 656 B per row).
 * Row layout, latent_row_bytes(dc, dr) = dc + 4*dc/128 + 2*dr bytes:
 *   [dc e4m3 codes | dc/128 fp32 scales | dr bf16 rotary values]
 * The latent part is quantised in blocks of 128 exactly as act_quant does
 * (scale = max(amax, 1e-4) / 448, code = e4m3_rn_satfinite(x / scale), both
 * divisions correctly rounded); the rotary part is rounded to bf16 (nearest
 * even).  Supported: dc in {128, 256, 384, 512}, dr a multiple of 8 up to 64,
 * dc + dr <= 576 (else DSA_ERR_UNSUPPORTED).
 */
int64_t dsa_latent_row_bytes(int dc, int dr);

/*
 * Quantise latent rows into the FP8 cache layout above.
 *   kv   [n_rows, n_vec, dc + dr] F32 or BF16 (x_dtype), contiguous, 4-byte aligned
 *   out  row (r, v) -> out + r * out_row_stride + v * latent_row_bytes(dc, dr)
 * A cache append at start_pos: kv = new rows [B, S, dc + dr], n_rows = B, n_vec = S,
 * out = cache + start_pos * row_bytes, out_row_stride = t_max * row_bytes.
 * out and out_row_stride must be multiples of 4.
 */
dsa_status dsa_latent_quant(const void *kv, dsa_dtype x_dtype, int64_t n_rows, int64_t n_vec,
                            int dc, int dr, uint8_t *out, int64_t out_row_stride,
                            dsa_stream_t stream);

/*
 * Sparse latent attention (as dsa_sparse_mla_attn, bf16) over the FP8 latent
 * cache kv_fp8 [B, t_max, latent_row_bytes(dc, dr)].  Each query row's selected
 * rows are decoded (code * block scale, rounded to bf16; rotary part as
 * stored) into the workspace, then attended with the bf16 sparse attention.
 *   q    [B,S,Hq,dc+dr] bf16 (16-byte aligned), idx [B,S,k] int32 (-1 = empty)
 *   out  [B,S,Hq,dc] bf16 (16-byte aligned), lse [B,S,Hq] fp32 or NULL
 * Workspace: dsa_sparse_mla_attn_fp8_workspace_size bytes (16-byte aligned),
 * else DSA_ERR_WORKSPACE.  Masking as dsa_sparse_mla_attn (indices > start_pos + s
 * and -1 slots are skipped; indices >= t_max set DSA_ERR_DEVICE).
 */
size_t dsa_sparse_mla_attn_fp8_workspace_size(int B, int S, int Hq, int dc, int dr, int k);
dsa_status dsa_sparse_mla_attn_fp8(const void *q, const uint8_t *kv_fp8, int64_t t_max,
                                   const int32_t *idx, int B, int S, int Hq, int dc, int dr,
                                   int k, int64_t start_pos, float sm_scale, void *out,
                                   float *lse, void *workspace, size_t workspace_bytes,
                                   dsa_stream_t stream);

/*
 * fp8_index with the weight fold and the additive causal mask
 * (Indexer.forward; mask from Transformer.forward; formula from the diagram):
 *   w'[b,s,h]  = fp32(fp32(fp32(w * fp32(H^-1/2)) * q_scale) * softmax_scale)
 *   I[b,s,t]   = k_scale[b,t] * sum_h w'[b,s,h] * ReLU(q_fp8[b,s,h,:] . k_cache[b,t,:])
 *   I[b,s,t]   = -inf for t > start_pos + s
 * Dot products of the decoded FP8 values accumulate in fp32.
 *
 *   q_fp8   [B,S,H,D] e4m3 codes     q_scale [B,S,H] fp32     w [B,S,H] fp32
 *   k_cache [B,t_max,D] e4m3 codes   k_scale [B,t_max] fp32
 *   scores  [B,S,T] fp32 (T = end_pos <= t_max; start_pos + S <= T)
 * D must be 64 or 128; 1 <= H <= 256.
 */
dsa_status dsa_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                            const uint8_t *k_cache, const float *k_scale, int64_t t_max, int B,
                            int S, int H, int D, int64_t start_pos, int64_t T,
                            float softmax_scale, float *scores, dsa_stream_t stream);

/*
 * The indexer half of a decode step (Indexer.forward with seqlen == 1): rotate
 * and quantise the new token's queries q_idx [B,H,D] fp32 and key k_new [B,D]
 * fp32 exactly as dsa_indexer_quant does, append the key's codes and scale to
 * k_cache / k_scale at position T-1, and write scores [B,T] fp32 for positions
 * 0..T-1 as dsa_index_scores does (start_pos = T-1, no mask).  One kernel.
 * Same constraints as dsa_index_scores; t_max * D must be a multiple of 16.
 */
dsa_status dsa_decode_index_scores(const float *q_idx, const float *w, const float *k_new,
                                   uint8_t *k_cache, float *k_scale, int64_t t_max, int B, int H,
                                   int D, int64_t T, float softmax_scale, float *scores,
                                   dsa_stream_t stream);

/*
 * The top-k step of Indexer.forward (min(index_topk, end_pos) positions), restricted to the causal
 * positions t <= start_pos + s of each row:
 *   idx[b,s,:] holds the m = min(K, start_pos+s+1, T) positions with the
 *   largest scores, K = min(k, T), ties broken towards the lower position,
 *   written in ascending position order; slots m..K-1 hold -1.
 * Scores are compared as fp32 values (-0 equals +0; NaN ranks below -inf).
 *
 *   scores [B,S,T] fp32     idx [B,S,K] int32
 */
size_t dsa_topk_select_workspace_size(int B, int S, int64_t T, int k);
dsa_status dsa_topk_select(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                           int k, int32_t *idx, void *workspace, size_t workspace_bytes,
                           dsa_stream_t stream);

/*
 * The indexer of DeepSeek-V4's compressed sparse attention (CSA branch of
 * "visualize_attention_masks.py (DeepSeek-V4)"): the keys are compressed
 * entries of `compress` (m >= 1) tokens each, and entry e is causally
 * available to the query at absolute position i = start_pos + s once all its
 * tokens are in, i.e. e < (i + 1) / m (integer division).  The page shows only
 * this availability rule and the -1 warm-up sentinel of the top-k; how the
 * compressor builds an entry's key is not shown, so the entries' indexer keys
 * are an input, in the cache layout of dsa_index_scores.  With m = 1 these two
 * calls are dsa_index_scores and dsa_topk_select.
 *
 * dsa_index_scores_csa: as dsa_index_scores over T entries (k_cache / k_scale
 * rows are entries), scores [B,S,T] fp32, entry e of query s masked (-inf)
 * unless e < (start_pos + s + 1) / m.  (start_pos + S) / m must not exceed T.
 *
 * dsa_topk_select_csa: idx[b,s,:] (K = min(k, T) slots) holds the
 * min(K, available entries) entry ids with the largest scores among the row's
 * available entries, ties towards the lower entry, in ascending order; the
 * other slots hold -1 (warm-up: fewer entries than k available yet).
 * Workspace as dsa_topk_select.  Both return DSA_ERR_INVALID_ARG for m < 1.
 */
dsa_status dsa_index_scores_csa(const uint8_t *q_fp8, const float *q_scale, const float *w,
                                const uint8_t *k_cache, const float *k_scale, int64_t t_max,
                                int B, int S, int H, int D, int64_t start_pos, int64_t T,
                                int compress, float softmax_scale, float *scores,
                                dsa_stream_t stream);
dsa_status dsa_topk_select_csa(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                               int compress, int k, int32_t *idx, void *workspace,
                               size_t workspace_bytes, dsa_stream_t stream);

/*
 * Sparse latent attention, MQA mode (diagram "core attention"; semantics of
 * the MLA prefill excerpt with the index mask and the causal mask):
 *   for each (b, s, head) over the selected rows c_j = kv_cache[b, idx_j, :]:
 *   z_j = sm_scale * (q[:dc] . c_j[:dc] + q[dc:] . c_j[dc:])
 *   out = sum_j softmax(z)_j * c_j[:dc],   lse = log sum_j exp(z_j)
 * Slots with idx < 0 or idx > start_pos + s are skipped (the -1 sentinel and
 * the causal mask).  A row with no valid slot gives out = 0, lse = -inf.
 * Indices must be distinct within a row and below t_max; an index >= t_max
 * is skipped and recorded as DSA_ERR_DEVICE in the device word.
 *
 *   q        [B,S,Hq,dc+dr]   kv_cache [B,t_max,dc+dr]   (dtype dt)
 *   idx      [B,S,k] int32
 *   out      [B,S,Hq,dc] (dtype dt)     lse [B,S,Hq] fp32 or NULL
 * dt = DSA_BF16 (tensor-core path, fp32 softmax and accumulation) or DSA_F32
 * (test mode: fp32 FMA throughout).
 */
size_t dsa_sparse_mla_attn_workspace_size(int B, int S, int Hq, int dc, int dr, int k,
                                          dsa_dtype dt);
dsa_status dsa_sparse_mla_attn(const void *q, const void *kv_cache, int64_t t_max,
                               const int32_t *idx, int B, int S, int Hq, int dc, int dr, int k,
                               int64_t start_pos, float sm_scale, dsa_dtype dt, void *out,
                               float *lse, void *workspace, size_t workspace_bytes,
                               dsa_stream_t stream);

/*
 * One DSA decode step for B sequences that each see T tokens (end_pos = T,
 * the new token at position T-1; no mask, as seqlen == 1):
 *   1. rotate + quantise the new token's indexer queries and key; append the
 *      key to k_cache / k_scale at position T-1 (Indexer.forward cache write);
 *   2. score all T cached keys (fp8_index with the weight fold);
 *   3. select the top K = min(index_topk, T) positions into idx;
 *   4. sparse latent attention of q_mla over the selected latent rows.
 *
 *   q_idx [B,H,D] fp32   w [B,H] fp32   k_new [B,D] fp32
 *   k_cache [B,t_max,D] e4m3 (written at T-1)   k_scale [B,t_max] fp32
 *   kv_cache [B,t_max,dc+dr] (dt): row T-1 must already hold the new latent
 *   q_mla [B,Hq,dc+dr] (dt)   idx [B,K] int32   out [B,Hq,dc] (dt)
 *   lse [B,Hq] fp32 or NULL
 * dt = DSA_FP8_LATENT: kv_cache is the FP8 latent cache [B, t_max,
 * dsa_latent_row_bytes(dc, dr)] (16-byte aligned), attended as
 * dsa_sparse_mla_attn_fp8 does; q_mla and out are bf16.
 */
size_t dsa_decode_step_workspace_size(int B, int H, int D, int64_t T, int index_topk, int Hq,
                                      int dc, int dr, dsa_dtype dt);
dsa_status dsa_decode_step(const float *q_idx, const float *w, const float *k_new,
                           uint8_t *k_cache, float *k_scale, int64_t t_max,
                           const void *kv_cache, const void *q_mla, int B, int H, int D, int Hq,
                           int dc, int dr, int64_t T, int index_topk, float softmax_scale,
                           float sm_scale, dsa_dtype dt, int32_t *idx, void *out, float *lse,
                           void *workspace, size_t workspace_bytes, dsa_stream_t stream);

/*
 * The decode step without a workspace, for callers that cannot allocate device
 * memory (a plugin living in another engine's memory pool, code launched while
 * a CUDA graph owned by someone else is being captured, a host that links only
 * this library).  The pages have no counterpart: this is a packaging variant
 * of dsa_decode_step, with the same arguments minus the workspace and the same
 * results.
 *
 * Scratch comes from a fixed device array of DSA_NOALLOC_SCRATCH_BYTES inside
 * the library; every GPU that loads the library holds it until the process
 * exits.  No call allocates or frees memory.  A problem whose
 * dsa_decode_step_workspace_size() exceeds DSA_NOALLOC_SCRATCH_BYTES is
 * rejected with DSA_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device resolves the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     A call that finds a different CUDA context current on the device (after
 *     cudaDeviceReset, say) resolves it again, so that call too should come
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents (nothing in it needs to start at zero).  Calls that
 *     overlap on the GPU (other streams, other threads) race on it: serialise
 *     them, e.g. by issuing them on one stream.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (32u << 20)
dsa_status dsa_decode_step_noalloc(const float *q_idx, const float *w, const float *k_new,
                                   uint8_t *k_cache, float *k_scale, int64_t t_max,
                                   const void *kv_cache, const void *q_mla, int B, int H, int D,
                                   int Hq, int dc, int dr, int64_t T, int index_topk,
                                   float softmax_scale, float sm_scale, dsa_dtype dt,
                                   int32_t *idx, void *out, float *lse, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
