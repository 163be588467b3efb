"""fp8_index scoring on the GPU vs the oracle (1e-3 relative, exact mask)."""
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
