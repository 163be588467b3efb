"""GPU-side drivers for the parity tests: put seeded workloads on the device and
run whole passes through the C ABI (no oracle code here)."""
import torch

import workloads


def decode_batch(dsa, wl, T=None, B=None, t_max=None, fp8_latent=False):
    """Build a decode step's device state for sequences 0..B-1 and run it once.

    The cache holds positions 0..T-2 quantised by dsa_indexer_quant; the step
    appends the new key at T-1.  With fp8_latent the latent rows are quantised
    by dsa_latent_quant into the FP8 latent cache, which the step attends over.
    Returns (host inputs per sequence, device results).
    """
    T = wl.T if T is None else T
    B = wl.B if B is None else B
    t_max = T if t_max is None else t_max
    dt = torch.bfloat16 if wl.attn_dtype == "bf16" else torch.float32
    seqs = [workloads.decode_sequence(wl, b, T=T) for b in range(B)]
    dev = "cuda"
    k_cache = torch.zeros(B, t_max, wl.D, dtype=torch.uint8, device=dev)
    k_scale = torch.zeros(B, t_max, dtype=torch.float32, device=dev)
    kv = torch.zeros(B, t_max, wl.dqk, dtype=dt, device=dev)
    q_idx = torch.stack([s["q_idx"] for s in seqs]).to(dev)
    w = torch.stack([s["w"] for s in seqs]).to(dev)
    k_new = torch.stack([s["keys"][T - 1] for s in seqs]).to(dev)
    q_mla = torch.stack([s["q_mla"] for s in seqs]).to(dev)
    for b, s in enumerate(seqs):
        if T > 1:
            dsa.dsa_indexer_quant(s["keys"][:T - 1].to(dev), k_cache[b], k_scale[b])
        kv[b, :T] = s["kv"].to(dev)
    kv_dt = dsa.DSA_BF16 if dt == torch.bfloat16 else dsa.DSA_F32
    if fp8_latent:
        rb = dsa.dsa_latent_row_bytes(wl.dc, wl.dr)
        kv8 = torch.zeros(B, t_max, rb, dtype=torch.uint8, device=dev)
        dsa.dsa_latent_quant(kv, kv8, wl.dc, n_rows=B, out_row_stride=t_max * rb)
        kv, kv_dt = kv8, dsa.DSA_FP8_LATENT
    K = min(wl.topk, T)
    idx = torch.empty(B, K, dtype=torch.int32, device=dev)
    out = torch.empty(B, wl.Hq, wl.dc, dtype=dt, device=dev)
    lse = torch.empty(B, wl.Hq, dtype=torch.float32, device=dev)
    need = dsa.dsa_decode_step_workspace_size(B, wl.H, wl.D, T, wl.topk, wl.Hq, wl.dc, wl.dr,
                                              kv_dt)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    state = dict(q_idx=q_idx, w=w, k_new=k_new, k_cache=k_cache, k_scale=k_scale, kv=kv,
                 q_mla=q_mla, idx=idx, out=out, lse=lse, ws=ws, T=T)
    run_decode(dsa, wl, state)
    torch.cuda.synchronize()
    return seqs, state


def run_decode(dsa, wl, st, stream=None):
    dsa.dsa_decode_step(st["q_idx"], st["w"], st["k_new"], st["k_cache"], st["k_scale"], st["kv"],
                        st["q_mla"], st["T"], wl.topk, wl.softmax_scale_idx, wl.sm_scale,
                        st["idx"], st["out"], st["lse"], st["ws"], stream=stream)


def prefill(dsa, wl, inp, T=None):
    """Prefill of B sequences (start_pos = 0, S = T) chained through the C ABI."""
    T = inp["keys"].shape[1] if T is None else T
    B, H, D = wl.B, wl.H, wl.D
    dev = "cuda"
    dt = torch.bfloat16 if wl.attn_dtype == "bf16" else torch.float32
    q = inp["q_idx"][:, :T].contiguous().to(dev)
    keys = inp["keys"][:, :T].contiguous().to(dev)
    w = inp["w"][:, :T].contiguous().to(dev)
    q_fp8 = torch.empty(B, T, H, D, dtype=torch.uint8, device=dev)
    q_scale = torch.empty(B, T, H, dtype=torch.float32, device=dev)
    k_cache = torch.empty(B, T, D, dtype=torch.uint8, device=dev)
    k_scale = torch.empty(B, T, dtype=torch.float32, device=dev)
    dsa.dsa_indexer_quant(q, q_fp8, q_scale)
    dsa.dsa_indexer_quant(keys, k_cache, k_scale, n_rows=B, out_row_stride=T * D,
                          scale_row_stride=T)
    scores = torch.empty(B, T, T, dtype=torch.float32, device=dev)
    dsa.dsa_index_scores(q_fp8, q_scale, w, k_cache, k_scale, 0, T, wl.softmax_scale_idx, scores)
    K = min(wl.topk, T)
    idx = torch.empty(B, T, K, dtype=torch.int32, device=dev)
    need = dsa.dsa_topk_select_workspace_size(B, T, T, wl.topk)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dsa.dsa_topk_select(scores, 0, wl.topk, idx, ws)
    q_mla = inp["q_mla"][:, :T].contiguous().to(dev)
    kv = inp["kv"][:, :T].contiguous().to(dev)
    out = torch.empty(B, T, wl.Hq, wl.dc, dtype=dt, device=dev)
    lse = torch.empty(B, T, wl.Hq, dtype=torch.float32, device=dev)
    need = dsa.dsa_sparse_mla_attn_workspace_size(
        B, T, wl.Hq, wl.dc, wl.dr, K, dsa.DSA_BF16 if dt == torch.bfloat16 else dsa.DSA_F32)
    ws2 = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dsa.dsa_sparse_mla_attn(q_mla, kv, idx, 0, wl.sm_scale, out, lse, ws2)
    torch.cuda.synchronize()
    return dict(q_fp8=q_fp8, q_scale=q_scale, k_cache=k_cache, k_scale=k_scale, scores=scores,
                idx=idx, out=out, lse=lse)
