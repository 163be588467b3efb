"""A prefill in two chunks through the C ABI: the second chunk (start_pos > 0,
S > 1) runs against a cache the first chunk filled.

Chunk 1 (positions 0 .. C-1) only appends its keys; chunk 2 (positions C .. T-1)
appends its keys, scores its queries against all T cached keys with the causal
mask offset by start_pos = C, selects, and attends.  Every step is the fused
prologue (RoPE on 64 of 128 dims, rotate_activation, act_quant), fp8_index,
top-k and sparse attention of libdsa, compared with the oracle run on the
unchunked sequence (each query and key vector is prepared independently, so
the chunking must not change any code)."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_attention_close, assert_scores_close, assert_selection_matches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _angles(T, R, base=10000.0):
    pos = np.arange(T, dtype=np.float64)[:, None]
    th = pos * base ** (-np.arange(0, R, 2, dtype=np.float64) / R)[None, :]
    return np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32)


@pytest.mark.parametrize("fmt", [0, 1])
def test_two_chunk_prefill_matches_oracle(dsa, fmt):
    T, C, H, D, R, topk = 900, 600, 64, 128, 64, 256
    Hq, dc, dr = 128, 512, 64
    S2 = T - C
    g = torch.Generator().manual_seed(77 + fmt)
    q = torch.randn(1, T, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(1, T, D, generator=g).to(torch.bfloat16)
    w = torch.randn(1, T, H, generator=g)
    q_mla = torch.randn(1, T, Hq, dc + dr, generator=g).to(torch.bfloat16)
    kv = torch.randn(1, T, dc + dr, generator=g).to(torch.bfloat16)
    cs = _angles(T, R)
    sm_idx, sm = D ** -0.5, (dc + dr) ** -0.5
    dev = "cuda"

    k_cache = torch.zeros(1, T, D, dtype=torch.uint8, device=dev)
    k_scale = torch.zeros(1, T, dtype=torch.float32, device=dev)
    cs_d = torch.from_numpy(cs).to(dev)
    # chunk 1: its keys only (its own queries are not part of this check)
    dsa.dsa_indexer_prologue(None, k[:, :C].contiguous().to(dev), cs_d[:C].contiguous(), 0,
                             None, None, k_cache, k_scale, scale_fmt=fmt)
    # chunk 2
    q2_fp8 = torch.empty(1, S2, H, D, dtype=torch.uint8, device=dev)
    q2_scale = torch.empty(1, S2, H, dtype=torch.float32, device=dev)
    dsa.dsa_indexer_prologue(q[:, C:].contiguous().to(dev), k[:, C:].contiguous().to(dev),
                             cs_d[C:].contiguous(), C, q2_fp8, q2_scale, k_cache, k_scale,
                             scale_fmt=fmt)
    scores = torch.empty(1, S2, T, dtype=torch.float32, device=dev)
    dsa.dsa_index_scores(q2_fp8, q2_scale, w[:, C:].contiguous().to(dev), k_cache, k_scale, C, T,
                         sm_idx, scores)
    idx = torch.empty(1, S2, topk, dtype=torch.int32, device=dev)
    need = dsa.dsa_topk_select_workspace_size(1, S2, T, topk)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dsa.dsa_topk_select(scores, C, topk, idx, ws)
    out = torch.empty(1, S2, Hq, dc, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, S2, Hq, dtype=torch.float32, device=dev)
    need = dsa.dsa_sparse_mla_attn_workspace_size(1, S2, Hq, dc, dr, topk, dsa.DSA_BF16)
    ws2 = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dsa.dsa_sparse_mla_attn(q_mla[:, C:].contiguous().to(dev), kv.to(dev), idx, C, sm, out, lse,
                            ws2)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == dsa.DSA_OK

    # the oracle on the unchunked sequence
    rq, rqs, rk, rks = oracle.indexer_prologue(q.float().numpy(), k.float().numpy(), cs, fmt)
    assert np.array_equal(k_cache.cpu().numpy(), rk)
    assert np.array_equal(k_scale.cpu().numpy(), rks)
    assert np.array_equal(q2_fp8.cpu().numpy(), rq[:, C:])
    assert np.array_equal(q2_scale.cpu().numpy(), rqs[:, C:])
    ref_scores = oracle.index_scores(rq[:, C:], rqs[:, C:], w[:, C:].numpy(), rk, rks, C, T, sm_idx)
    assert_scores_close(scores.cpu().numpy(), ref_scores)
    ref_idx = oracle.topk_select(ref_scores, C, topk)
    gi = idx.cpu().numpy()
    for s in range(S2):
        assert_selection_matches(gi[0, s], ref_idx[0, s], ref_scores[0, s])
        assert (gi[0, s][gi[0, s] >= 0] <= C + s).all()           # never a future position
    rows = [0, 1, 2, 127, 128, 255, 256, S2 - 1]
    ref_out = np.empty((1, len(rows), Hq, dc), np.float64)
    ref_lse = np.empty((1, len(rows), Hq), np.float64)
    # each sampled row keeps its own causal limit C + s: evaluate it as a one-row chunk
    for j, s in enumerate(rows):
        o1, l1 = oracle.sparse_mla(q_mla[:, C + s:C + s + 1].float().numpy(), kv.float().numpy(),
                                   ref_idx[:, s:s + 1], C + s, sm, dc)
        ref_out[:, j], ref_lse[:, j] = o1[:, 0], l1[:, 0]
    assert_attention_close(out.float().cpu().numpy()[:, rows], ref_out, "bf16",
                           lse.cpu().numpy()[:, rows], ref_lse)
