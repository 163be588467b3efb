"""The V4 compressed-sparse-attention (CSA) indexer on the GPU vs the oracle:
fp8_index over compressed entries with their causal availability
(entry < (i + 1) // m), and the top-k over the available entries with -1
warm-up sentinels ("visualize_attention_masks.py (DeepSeek-V4)", CSA branch)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_scores_close, assert_selection_matches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _case(B, S, H, D, t_max, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, S, H, D, generator=g)
    w = torch.randn(B, S, H, generator=g)
    keys = torch.randn(B, t_max, D, generator=g)
    qf, qs = oracle.indexer_quant(q.numpy())
    kf, ks = oracle.indexer_quant(keys.numpy())
    return qf, qs, w.numpy(), kf, ks


def _scores(dsa, qf, qs, w, kf, ks, sp, T, m, sm):
    B, S = qf.shape[:2]
    out = torch.empty(B, S, T, dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores_csa(torch.from_numpy(qf).cuda(), torch.from_numpy(qs).cuda(),
                             torch.from_numpy(w).cuda(), torch.from_numpy(kf).cuda(),
                             torch.from_numpy(ks).cuda(), sp, T, m, sm, out)
    return out


def _topk(dsa, scores, sp, m, k):
    B, S, T = scores.shape
    K = min(k, T)
    idx = torch.empty(B, S, K, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, dsa.dsa_topk_select_workspace_size(B, S, T, k)), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_topk_select_csa(scores, sp, m, k, idx, ws)
    return idx.cpu().numpy()


# (B, S, H, D, t_max, T entries, start_pos, m): (start_pos + S) // m <= T
CASES = [
    (2, 1, 64, 128, 1100, 1000, 3999, 4),     # decode: 1000 entries of 4 tokens
    (1, 1, 64, 128, 40, 33, 4224, 128),       # decode at an HCA-like rate
    (1, 64, 64, 128, 200, 200, 736, 4),       # prefill chunk against a compressed cache
    (1, 32, 4, 64, 8, 8, 0, 4),               # warm-up: the first queries see no entry yet
    (3, 5, 4, 64, 300, 257, 1023, 4),         # ragged tile tail
    (1, 40, 8, 128, 600, 600, 560, 1),        # m = 1: the token-level indexer
]


@pytest.mark.parametrize("B,S,H,D,t_max,T,sp,m", CASES)
def test_csa_scores_match_oracle(dsa, B, S, H, D, t_max, T, sp, m):
    qf, qs, w, kf, ks = _case(B, S, H, D, t_max, seed=B * 7919 + T + m)
    sm = D ** -0.5
    got = _scores(dsa, qf, qs, w, kf, ks, sp, T, m, sm).cpu().numpy()
    ref = oracle.index_scores_csa(qf, qs, w, kf, ks, sp, T, m, sm)
    assert_scores_close(got, ref)


@pytest.mark.parametrize("B,S,H,D,t_max,T,sp,m", CASES)
def test_csa_topk_identical_to_oracle_on_the_same_scores(dsa, B, S, H, D, t_max, T, sp, m):
    qf, qs, w, kf, ks = _case(B, S, H, D, t_max, seed=B * 7919 + T + m)
    ref_sc = oracle.index_scores_csa(qf, qs, w, kf, ks, sp, T, m, D ** -0.5)
    for k in (16, 2048):
        got = _topk(dsa, torch.from_numpy(ref_sc).cuda(), sp, m, k)
        ref = oracle.topk_select_csa(ref_sc, sp, m, k)
        assert np.array_equal(got, ref)


def test_csa_chained_decode_long_cache(dsa):
    """Decode over 32768 entries (131072 tokens at m = 4), k = 2048: the GPU's own
    scores and selection against the oracle's, ties at the k-th score allowed."""
    B, H, D, T, m, k = 2, 64, 128, 32768, 4, 2048
    sp = T * m - 1
    qf, qs, w, kf, ks = _case(B, 1, H, D, T, seed=4242)
    sm = D ** -0.5
    sc = _scores(dsa, qf, qs, w, kf, ks, sp, T, m, sm)
    idx = _topk(dsa, sc, sp, m, k)
    ref_sc = oracle.index_scores_csa(qf, qs, w, kf, ks, sp, T, m, sm)
    assert_scores_close(sc.cpu().numpy(), ref_sc)
    ref_idx = oracle.topk_select_csa(ref_sc, sp, m, k)
    for b in range(B):
        assert_selection_matches(idx[b, 0], ref_idx[b, 0], ref_sc[b, 0])


def test_csa_warmup_rows_pad_with_sentinels(dsa):
    """Prefill from position 0 at m = 4: row s sees (s + 1) // 4 entries; the
    rest of its k slots are -1."""
    B, S, H, D, m, k = 1, 48, 4, 64, 4, 8
    T = S // m
    qf, qs, w, kf, ks = _case(B, S, H, D, T, seed=77)
    sc = _scores(dsa, qf, qs, w, kf, ks, 0, T, m, D ** -0.5)
    idx = _topk(dsa, sc, 0, m, k)
    for s in range(S):
        avail = (s + 1) // m
        n = min(avail, min(k, T))
        assert np.all(idx[0, s, :n] >= 0) and np.all(idx[0, s, :n] < avail)
        assert np.all(idx[0, s, n:] == -1)
