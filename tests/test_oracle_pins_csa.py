"""Pins of the oracle's V4 compressed-sparse-attention (CSA) indexer.

Page: "visualize_attention_masks.py (DeepSeek-V4)", CSA branch: the indexer
scores compressed entries of m tokens (m = the compress rate), an entry is
causally available to the query at position i once its m tokens are in, and
the top-k lists entry ids with -1 as the warm-up sentinel.  The pins derive
availability from token coverage (not from the oracle's formula), recompute the
scores with numpy einsums in fp64, and rank with numpy's lexsort.
"""
import numpy as np
import pytest

import oracle
import workloads
from test_oracle_pins import _rand_codes, _brute_scores, _lexsort_select


def _available_by_coverage(i: int, m: int) -> int:
    """Entries e (tokens e*m .. e*m + m - 1) whose every token is at or before i."""
    n = 0
    e = 0
    while True:
        tokens = range(e * m, (e + 1) * m)
        if all(t <= i for t in tokens):
            n += 1
            e += 1
        else:
            return n


@pytest.mark.parametrize("m", [1, 2, 3, 4, 7, 128])
def test_availability_from_token_coverage(m):
    for i in range(0, 3 * m + 40):
        assert oracle.csa_available(i, m) == _available_by_coverage(i, m)
    # m = 1: every position up to i, the token-level causal count
    if m == 1:
        assert all(oracle.csa_available(i, 1) == i + 1 for i in range(500))


def test_csa_scores_brute_force_tiny():
    rng = np.random.default_rng(21)
    B, S, H, D, t_max, T, sp, m = 2, 5, 4, 64, 12, 10, 9, 4
    q = _rand_codes(rng, (B, S, H, D))
    qs = (rng.random((B, S, H)) * 0.01 + 1e-3).astype(np.float32)
    w = rng.standard_normal((B, S, H)).astype(np.float32)
    k = _rand_codes(rng, (B, t_max, D))
    ks = (rng.random((B, t_max)) * 0.01 + 1e-3).astype(np.float32)
    got = oracle.index_scores_csa(q, qs, w, k, ks, sp, T, m, 0.125)
    # scores with no mask at all (start_pos past every entry), then the
    # availability of each query from token coverage
    ref = _brute_scores(q, qs, w, k, ks, T, T, 0.125)
    for s in range(S):
        avail = _available_by_coverage(sp + s, m)
        assert np.all(np.isfinite(got[:, s, :avail]))
        assert np.all(got[:, s, avail:] == -np.inf)
        assert np.allclose(got[:, s, :avail], ref[:, s, :avail], rtol=1e-6, atol=0)


def test_csa_scores_equal_token_scores_when_m_is_one():
    rng = np.random.default_rng(22)
    B, S, H, D, T, sp = 1, 4, 2, 64, 20, 12
    q = _rand_codes(rng, (B, S, H, D))
    qs = (rng.random((B, S, H)) * 0.01 + 1e-3).astype(np.float32)
    w = rng.standard_normal((B, S, H)).astype(np.float32)
    k = _rand_codes(rng, (B, T, D))
    ks = (rng.random((B, T)) * 0.01 + 1e-3).astype(np.float32)
    a = oracle.index_scores_csa(q, qs, w, k, ks, sp, T, 1, 0.09)
    b = oracle.index_scores(q, qs, w, k, ks, sp, T, 0.09)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("m,sp,k", [(4, 0, 8), (4, 37, 8), (4, 399, 16), (7, 100, 5), (1, 50, 20),
                                    (128, 2000, 4)])
def test_csa_topk_matches_lexsort_and_pads_warmup(m, sp, k):
    T = max(1, (sp + 6) // m)
    S = 6
    sc = workloads.score_rows(S, T, seed=m * 1000 + sp).numpy()[None]      # [1,S,T]
    idx = oracle.topk_select_csa(sc, sp, m, k)
    K = min(k, T)
    assert idx.shape == (1, S, K)
    for r in range(S):
        avail = min(T, _available_by_coverage(sp + r, m))
        sel = _lexsort_select(sc[0, r], avail, K)
        assert np.array_equal(idx[0, r, :len(sel)], sel)
        # warm-up sentinels: fewer available entries than slots
        assert np.all(idx[0, r, len(sel):] == -1)
        assert len(sel) == min(K, avail)
        # never an entry that is not yet complete
        assert np.all(idx[0, r, :len(sel)] < avail)


def test_csa_topk_ties_take_lower_entry():
    sc = np.zeros((1, 2, 12), dtype=np.float32)
    sc[0, :, ::3] = 1.0                     # ties at 0, 3, 6, 9
    idx = oracle.topk_select_csa(sc, 40, 4, 3)          # avail = 41 // 4 = 10 entries
    assert idx[0, 0].tolist() == [0, 3, 6]
    assert idx[0, 1].tolist() == [0, 3, 6]


def test_csa_topk_equals_token_topk_when_m_is_one():
    sc = workloads.score_rows(5, 200, seed=77, tie_frac=0.2).numpy()[None]
    for sp, k in ((10, 30), (150, 64), (195, 250)):
        S = 5
        a = oracle.topk_select_csa(sc, sp, 1, k)
        b = oracle.topk_select(sc, sp, k)
        assert np.array_equal(a, b)
