"""Top-k selection on the GPU: identical to the oracle when both see the same fp32 scores."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _gpu_topk(dsa, scores, start_pos, k):
    B, S, T = scores.shape
    K = min(k, T)
    sc = torch.from_numpy(np.ascontiguousarray(scores)).cuda()
    idx = torch.empty(B, S, K, dtype=torch.int32, device="cuda")
    need = dsa.dsa_topk_select_workspace_size(B, S, T, k)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    dsa.dsa_topk_select(sc, start_pos, k, idx, ws)
    return idx.cpu().numpy()


@pytest.mark.parametrize("B,S,T,sp,k,ties", [
    (1, 1, 4096, 4095, 2048, 0.0),       # V3.2 decode, 4K context
    (4, 1, 5003, 5002, 2048, 0.0),       # ragged
    (2, 1, 1500, 1499, 2048, 0.0),       # T < k: everything selected
    (2, 1, 2048, 2047, 2048, 0.0),       # T == k
    (3, 1, 9000, 8999, 2048, 0.3),       # many exact ties, also at the boundary
    (1, 1, 3000, 2999, 1, 0.0),          # k = 1
    (1, 64, 64, 0, 16, 0.0),             # prefill causal rows, short rows padded with -1
    (1, 40, 600, 560, 100, 0.1),         # query chunk with start_pos > 0
])
def test_topk_identical_to_oracle(dsa, B, S, T, sp, k, ties):
    sc = workloads.score_rows(B * S, T, seed=T + k, tie_frac=ties).numpy().reshape(B, S, T)
    got = _gpu_topk(dsa, sc, sp, k)
    ref = oracle.topk_select(sc, sp, k)
    assert np.array_equal(got, ref)


def test_topk_special_values(dsa):
    T = 3000
    sc = workloads.score_rows(4, T, seed=9).numpy()
    sc[0, ::3] = -np.inf                 # masked-looking entries inside the causal range
    sc[1, :] = 0.0
    sc[1, ::2] = -0.0                    # signed zeros tie
    sc[2, :2500] = -np.inf               # fewer finite scores than k
    sc[3] = np.abs(sc[3])                # all positive
    sc = sc.reshape(4, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)


def test_topk_long_context_rows(dsa):
    """Rows of 131072 scores (the 128K decode) with k = 2048."""
    T = 131072
    sc = workloads.score_rows(8, T, seed=4).numpy().reshape(8, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)


def test_topk_prefill_full_size_sampled_rows(dsa):
    """8192 causal rows of 8192 scores, top-2048 each; rows compared one by one."""
    T = 8192
    sc = workloads.score_rows(T, T, seed=8).numpy().reshape(1, T, T)
    got = _gpu_topk(dsa, sc, 0, 2048)
    for s in (0, 1, 2046, 2047, 2048, 4000, 8191):
        ref = oracle.topk_select(sc[:, s:s + 1], s, 2048)
        assert np.array_equal(got[:, s:s + 1], ref)


def test_topk_deterministic(dsa):
    sc = workloads.score_rows(4, 20000, seed=11, tie_frac=0.2).numpy().reshape(4, 1, 20000)
    a = _gpu_topk(dsa, sc, 19999, 2048)
    b = _gpu_topk(dsa, sc, 19999, 2048)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("T", [20000, 40000, 70000, 300000, 700000])
def test_topk_every_cluster_size_and_fallback(dsa, T):
    """Row lengths that take 2, 4, 8 and 16 CTAs per row, and the one-CTA
    global-memory kernel beyond that."""
    sc = workloads.score_rows(2, T, seed=T % 997, tie_frac=0.05).numpy().reshape(2, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)


def test_topk_outlier_and_flat_rows(dsa):
    """A huge outlier squeezes every other score into one linear bin; a flat
    row has no spread at all; both must still select exactly."""
    T = 50000
    sc = workloads.score_rows(3, T, seed=12).numpy()
    sc[0, 777] = 3.0e38
    sc[1, :] = 0.25
    sc[2, 5] = -3.0e38
    sc[2, 9] = np.inf
    sc = sc.reshape(3, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)


def test_topk_query_chunk_rows_of_different_lengths(dsa):
    """S rows of a chunk share a cluster size but see different causal prefixes."""
    B, S, T = 2, 6, 40000
    sp = T - S
    sc = workloads.score_rows(B * S, T, seed=13, tie_frac=0.02).numpy().reshape(B, S, T)
    got = _gpu_topk(dsa, sc, sp, 2048)
    ref = oracle.topk_select(sc, sp, 2048)
    assert np.array_equal(got, ref)


def _tied_block_row(T, n_top, n_tied, tied_positions, seed):
    """Uniform [0, 1) scores, n_top of them in [6, 7) and n_tied exactly 5.0 at
    the given positions: with k between n_top and n_top + n_tied the k-th
    largest is 5.0 and only the lowest-positioned ties are taken."""
    rng = np.random.default_rng(seed)
    row = rng.random(T, dtype=np.float32)
    rest = np.setdiff1d(np.arange(T), tied_positions)
    top = rng.choice(rest, n_top, replace=False)
    row[top] = 6.0 + rng.random(n_top, dtype=np.float32)
    row[tied_positions] = 5.0
    return row


def test_topk_many_tied_candidates_spread_over_the_cluster(dsa):
    """4000 ties at the threshold, spread over the row: every CTA sends a few
    hundred candidates and CTA 0 radix-selects among them."""
    T = 131072
    rows = [_tied_block_row(T, 1500, 4000, np.linspace(0, T - 1, 4000).astype(np.int64), s)
            for s in range(2)]
    sc = np.stack(rows).reshape(2, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)


def test_topk_tied_candidates_crowded_into_one_slice(dsa):
    """1000 ties in the first 1000 positions: one CTA holds more threshold-bin
    candidates than it may send to CTA 0, so the cluster-wide radix rounds run."""
    T = 131072
    rows = [_tied_block_row(T, 1500, 1000, np.arange(1000), s) for s in range(2)]
    sc = np.stack(rows).reshape(2, 1, T)
    got = _gpu_topk(dsa, sc, T - 1, 2048)
    ref = oracle.topk_select(sc, T - 1, 2048)
    assert np.array_equal(got, ref)
