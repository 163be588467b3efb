"""fp8_index scoring on the GPU vs the oracle (1e-3 relative, exact mask)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_scores_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _quantised_case(B, S, H, D, t_max, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, S, H, D, generator=g)
    w = torch.randn(B, S, H, generator=g)
    keys = torch.randn(B, t_max, D, generator=g)
    qf, qs = oracle.indexer_quant(q.numpy())
    kf, ks = oracle.indexer_quant(keys.numpy())
    return qf, qs, w.numpy(), kf, ks


def _run(dsa, qf, qs, w, kf, ks, start_pos, T, sm):
    B, S = qf.shape[:2]
    out = torch.empty(B, S, T, dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores(torch.from_numpy(qf).cuda(), torch.from_numpy(qs).cuda(),
                         torch.from_numpy(w).cuda(), torch.from_numpy(kf).cuda(),
                         torch.from_numpy(ks).cuda(), start_pos, T, sm, out)
    return out.cpu().numpy()


@pytest.mark.parametrize("B,S,H,D,t_max,T,sp", [
    (1, 1, 64, 128, 5000, 4999, 4998),      # decode, ragged tail of the 128-token tiles
    (2, 1, 64, 128, 700, 513, 512),         # decode, t_max > T
    (1, 1, 64, 128, 1, 1, 0),               # single cached token
    (3, 1, 4, 64, 300, 300, 299),           # tiny heads
    (1, 20, 64, 128, 400, 400, 380),        # chunk of queries against a cache
    (1, 130, 4, 64, 130, 130, 0),           # prefill with the causal mask
])
def test_scores_match_oracle(dsa, B, S, H, D, t_max, T, sp):
    qf, qs, w, kf, ks = _quantised_case(B, S, H, D, t_max, seed=B * 1000 + T)
    sm = D ** -0.5
    got = _run(dsa, qf, qs, w, kf, ks, sp, T, sm)
    ref = oracle.index_scores(qf, qs, w, kf, ks, sp, T, sm)
    assert_scores_close(got, ref)


def test_scores_prefill_full_size_sampled_rows(dsa):
    """T = 8192 prefill scoring (64 x 128 heads); rows compared one by one."""
    wl = workloads.WORKLOADS[3]
    inp = workloads.prefill_inputs(wl)
    T = wl.T
    qf, qs = oracle.indexer_quant(inp["q_idx"].numpy())
    kf, ks = oracle.indexer_quant(inp["keys"].numpy())
    w = inp["w"].numpy()
    got = _run(dsa, qf, qs, w, kf, ks, 0, T, wl.softmax_scale_idx)
    for s in (0, 1, 127, 128, 2047, 2048, 5000, 8191):
        ref = oracle.index_scores(qf[:, s:s + 1], qs[:, s:s + 1], w[:, s:s + 1], kf, ks, s, T,
                                  wl.softmax_scale_idx)
        assert_scores_close(got[:, s:s + 1], ref)


@pytest.mark.parametrize("cfg,B,T,t_max,H", [
    (1, 3, 5000, 5003, None),
    (1, 1, 1, 8, None),
    (0, 2, 300, 300, None),        # D = 64, 4 heads: one lane per head, padded heads
    (1, 2, 4193, 4200, 128),       # two passes over the heads; T-1 in the last quarter
    (1, 1, 2081, 2081, 256),       # four passes; T-1 in the second quarter
    (1, 2, 129, 129, 64),          # T-1 opens a tile of its own
    (0, 2, 3000, 3001, 96),        # D = 64: the staged query's third box in the last key stage
    (1, 2, 700, 700, 20),          # staged query rows end inside its second box
])
def test_decode_index_scores_matches_oracle(dsa, cfg, B, T, t_max, H):
    """The indexer half of a decode step: quantise the new queries and key, append
    the key at T-1, score every cached position."""
    wl = workloads.WORKLOADS[cfg]
    if H is not None:
        wl = dataclasses.replace(wl, H=H)
    D, H = wl.D, wl.H
    seqs = [workloads.decode_sequence(wl, b, T=T) for b in range(B)]
    k_cache = torch.zeros(B, t_max, D, dtype=torch.uint8, device="cuda")
    k_scale = torch.zeros(B, t_max, dtype=torch.float32, device="cuda")
    for b, s in enumerate(seqs):
        if T > 1:
            dsa.dsa_indexer_quant(s["keys"][:T - 1].cuda(), k_cache[b], k_scale[b])
    q = torch.stack([s["q_idx"] for s in seqs]).cuda()
    w = torch.stack([s["w"] for s in seqs]).cuda()
    k_new = torch.stack([s["keys"][T - 1] for s in seqs]).cuda()
    scores = torch.empty(B, T, dtype=torch.float32, device="cuda")
    dsa.dsa_decode_index_scores(q, w, k_new, k_cache, k_scale, T, wl.softmax_scale_idx, scores)
    for b, s in enumerate(seqs):
        kf, ks = oracle.indexer_quant(s["keys"].numpy())
        qf, qs = oracle.indexer_quant(s["q_idx"].numpy())
        assert np.array_equal(k_cache[b, T - 1].cpu().numpy(), kf[T - 1])
        assert k_scale[b, T - 1].item() == ks[T - 1]
        ref = oracle.index_scores(qf[None, None], qs[None, None], s["w"].numpy()[None, None],
                                  kf[None], ks[None], T - 1, T, wl.softmax_scale_idx)
        assert_scores_close(scores[b:b + 1].cpu().numpy()[:, None], ref)


@pytest.mark.parametrize("B,S,H,D,T,sp,rows", [
    (1, 702, 64, 128, 702, 0, (0, 1, 3, 4, 127, 128, 351, 697, 700, 701)),   # ragged last group
    (2, 1195, 4, 64, 1195, 0, (0, 15, 16, 600, 1183, 1184, 1194)),          # 16 rows per group
    (1, 600, 64, 128, 1000, 400, (0, 3, 4, 199, 599)),                      # chunk on a cache
])
def test_prefill_groups_match_oracle(dsa, B, S, H, D, T, sp, rows):
    """Enough causal query rows for the grouped prefill scorer (several rows of
    one sequence per CTA, the key tile shared); rows compared one by one."""
    qf, qs, w, kf, ks = _quantised_case(B, S, H, D, T, seed=S + H)
    sm = D ** -0.5
    got = _run(dsa, qf, qs, w, kf, ks, sp, T, sm)
    for s in rows:
        ref = oracle.index_scores(qf[:, s:s + 1], qs[:, s:s + 1], w[:, s:s + 1], kf, ks, sp + s, T,
                                  sm)
        assert_scores_close(got[:, s:s + 1], ref)
