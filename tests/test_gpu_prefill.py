"""Prefill (start_pos = 0, causal) through the C ABI vs the oracle."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_pipelines import prefill
from parity import assert_attention_close, assert_scores_close, assert_selection_matches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _check_rows(wl, inp, res, rows):
    r = oracle.prefill_rows(inp["q_idx"][0].numpy(), inp["w"][0].numpy(), inp["keys"][0].numpy(),
                            inp["q_mla"][0].float().numpy(), inp["kv"][0].float().numpy(), rows,
                            topk=wl.topk, softmax_scale_idx=wl.softmax_scale_idx,
                            sm_scale=wl.sm_scale, dc=wl.dc)
    assert np.array_equal(res["k_cache"][0].cpu().numpy(), r["k_fp8"])
    assert np.array_equal(res["k_scale"][0].cpu().numpy(), r["k_scale"])
    assert np.array_equal(res["q_fp8"][0].cpu().numpy()[rows], r["q_fp8"])
    assert_scores_close(res["scores"][0].cpu().numpy()[rows], r["scores"])
    idx = res["idx"][0].cpu().numpy()
    out = res["out"][0].float().cpu().numpy()
    lse = res["lse"][0].cpu().numpy()
    for j, s in enumerate(rows):
        assert_selection_matches(idx[s], r["idx"][j], r["scores"][j])
        assert (idx[s][idx[s] >= 0] <= s).all()
    assert_attention_close(out[rows], r["out"], wl.attn_dtype, lse[rows], r["lse"])


def test_prefill_tiny_full(dsa):
    wl = workloads.WORKLOADS[0]
    inp = workloads.prefill_inputs(wl)
    res = prefill(dsa, wl, inp)
    _check_rows(wl, inp, res, list(range(wl.T)))


def test_prefill_ragged_v32_shapes(dsa):
    wl = workloads.WORKLOADS[3]
    inp = workloads.prefill_inputs(wl, T=2500)
    res = prefill(dsa, wl, inp)
    _check_rows(wl, inp, res, [0, 1, 127, 128, 2046, 2047, 2048, 2499])


def test_prefill_8k_full_size_sampled_rows(dsa):
    wl = workloads.WORKLOADS[3]
    inp = workloads.prefill_inputs(wl)
    res = prefill(dsa, wl, inp)
    _check_rows(wl, inp, res, [0, 1, 2046, 2047, 2048, 4095, 6001, 8191])
