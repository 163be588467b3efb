"""The fused decode step on the GPU vs the oracle's decode pass, sequence by sequence."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_pipelines import decode_batch, run_decode
from parity import assert_attention_close, assert_selection_matches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _check_sequence(wl, seq, state, b, T):
    r = oracle.decode_step(seq["q_idx"].numpy(), seq["w"].numpy(), seq["keys"].numpy(),
                           seq["q_mla"].float().numpy(), seq["kv"].float().numpy(), topk=wl.topk,
                           softmax_scale_idx=wl.softmax_scale_idx, sm_scale=wl.sm_scale, dc=wl.dc)
    # the appended key
    assert np.array_equal(state["k_cache"][b, T - 1].cpu().numpy(), r["k_fp8"][T - 1])
    assert state["k_scale"][b, T - 1].item() == r["k_scale"][T - 1]
    assert_selection_matches(state["idx"][b].cpu().numpy(), r["idx"], r["scores"])
    assert_attention_close(state["out"][b].float().cpu().numpy(), r["out"], wl.attn_dtype,
                           state["lse"][b].cpu().numpy(), r["lse"])
    return r


@pytest.mark.parametrize("cfg,T,B", [
    (1, 5000, 2),      # V3.2 shapes, ragged context
    (1, 1, 1),         # a single token: K = 1
    (1, 2048, 2),      # T == k: every position
    (1, 700, 1),       # T < k: K = min(k, T) = T slots, all filled
    (0, 300, 2),       # tiny heads, fp32 test mode
])
def test_decode_step_small(dsa, cfg, T, B):
    wl = workloads.WORKLOADS[cfg]
    if cfg == 0:
        wl = dataclasses.replace(wl, mode="decode")
    seqs, st = decode_batch(dsa, wl, T=T, B=B)
    for b in range(B):
        _check_sequence(wl, seqs[b], st, b, T)
    assert dsa.dsa_get_device_error() == 0


def test_decode_step_cache_capacity_larger_than_context(dsa):
    wl = workloads.WORKLOADS[1]
    seqs, st = decode_batch(dsa, wl, T=3000, B=2, t_max=4096)
    for b in range(2):
        _check_sequence(wl, seqs[b], st, b, 3000)


def test_decode_step_v32_4k_full(dsa):
    wl = workloads.WORKLOADS[1]
    seqs, st = decode_batch(dsa, wl)
    _check_sequence(wl, seqs[0], st, 0, wl.T)


def test_decode_step_batched_32k_sampled(dsa):
    wl = workloads.WORKLOADS[2]
    seqs, st = decode_batch(dsa, wl)
    for b in (0, 17, 31):
        _check_sequence(wl, seqs[b], st, b, wl.T)


def test_decode_step_long_context_128k(dsa):
    """B = 8 at 131072 tokens with 1% planted keys: every planted position is
    selected in every sequence; two sequences compared in full with the oracle."""
    wl = workloads.WORKLOADS[4]
    seqs, st = decode_batch(dsa, wl)
    idx = st["idx"].cpu().numpy()
    for b in range(wl.B):
        assert np.isin(seqs[b]["planted"].numpy(), idx[b]).all()
        assert len(np.unique(idx[b])) == wl.topk and (idx[b] >= 0).all()
    for b in (0, 7):
        _check_sequence(wl, seqs[b], st, b, wl.T)


def test_decode_step_deterministic(dsa):
    wl = workloads.WORKLOADS[1]
    seqs, st = decode_batch(dsa, wl, T=6000, B=2)
    idx1, out1 = st["idx"].clone(), st["out"].clone()
    run_decode(dsa, wl, st)
    torch.cuda.synchronize()
    assert torch.equal(idx1, st["idx"]) and torch.equal(out1, st["out"])


def test_decode_step_repeats_bitwise_50_steps(dsa):
    """50 back-to-back decode steps on one state at the long-context shapes
    (B = 8, T = 131072, the launch configuration the benchmark times): the
    selections, outputs and lse are bitwise the first step's every time (the
    re-appended key writes the same codes; the scorer's histogram atomics, the
    cluster top-k and the split merge are order-independent)."""
    wl = workloads.WORKLOADS[4]
    _, st = decode_batch(dsa, wl)
    idx1, out1, lse1 = st["idx"].clone(), st["out"].clone(), st["lse"].clone()
    outs = []
    for i in range(50):
        run_decode(dsa, wl, st)
        outs.append((st["idx"].clone(), st["out"].clone(), st["lse"].clone()))
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
    for i, (idx, out, lse) in enumerate(outs):
        assert torch.equal(idx, idx1), f"step {i}: selection differs"
        assert torch.equal(out, out1), f"step {i}: output differs"
        assert torch.equal(lse, lse1), f"step {i}: lse differs"


@pytest.mark.parametrize("T,B", [(5000, 2), (131072, 8)])
def test_decode_step_fp8_latent_cache(dsa, T, B):
    """The decode step over the FP8 latent cache (656-byte rows): the selection
    is the bf16 step's, the attention matches the oracle's attention over its
    own FP8 rows at the oracle's selection."""
    wl = workloads.WORKLOADS[1 if T < 100000 else 4]
    seqs, st = decode_batch(dsa, wl, T=T, B=B, fp8_latent=True)
    rows = st["kv"].cpu().numpy()
    for b in (0, B - 1):
        seq = seqs[b]
        k_fp8, k_sc = oracle.indexer_quant(seq["keys"].numpy())
        q_fp8, q_sc = oracle.indexer_quant(seq["q_idx"].numpy())
        sc = oracle.index_scores(q_fp8[None, None], q_sc[None, None], seq["w"].numpy()[None, None],
                                 k_fp8[None], k_sc[None], start_pos=T - 1, T=T,
                                 softmax_scale=wl.softmax_scale_idx)
        ref_idx = oracle.topk_select(sc, start_pos=T - 1, k=wl.topk)
        assert_selection_matches(st["idx"][b].cpu().numpy(), ref_idx[0, 0], sc[0, 0])
        assert np.array_equal(rows[b, :T], oracle.latent_quant(seq["kv"].float().numpy(), wl.dc))
        ref, ref_lse = oracle.sparse_mla_fp8(seq["q_mla"].float().numpy()[None, None], rows[b:b + 1],
                                             ref_idx, T - 1, wl.sm_scale, wl.dc, wl.dr)
        assert_attention_close(st["out"][b].float().cpu().numpy(), ref[0, 0], "bf16",
                               st["lse"][b].cpu().numpy(), ref_lse[0, 0])
    assert dsa.dsa_get_device_error() == 0


def test_decode_steps_growing_context(dsa):
    """Four decode steps launched back to back on one stream, the context growing
    by one token each step (T0 .. T0 + 3), with nothing between the launches:
    every step's scorer reads the keys that the previous steps appended while the
    kernels overlap through their programmatic launches.  Each step's selection,
    output and appended key match the oracle's decode pass over the cache as it
    stood at that step."""
    wl = workloads.WORKLOADS[1]
    B, T0, n = 2, 3000, 4
    t_max = T0 + n - 1
    dev = "cuda"
    dt = torch.bfloat16
    base = [workloads.decode_sequence(wl, b, T=t_max) for b in range(B)]
    # per step: the new token's queries, weights and attention query
    stepq = [[workloads.decode_sequence(wl, 100 + 10 * i + b, T=1) for b in range(B)]
             for i in range(n)]
    k_cache = torch.zeros(B, t_max, wl.D, dtype=torch.uint8, device=dev)
    k_scale = torch.zeros(B, t_max, dtype=torch.float32, device=dev)
    kv = torch.zeros(B, t_max, wl.dqk, dtype=dt, device=dev)
    for b, s in enumerate(base):
        dsa.dsa_indexer_quant(s["keys"][:T0 - 1].to(dev), k_cache[b], k_scale[b])
        kv[b] = s["kv"].to(dev)
    q_idx = torch.stack([torch.stack([stepq[i][b]["q_idx"] for b in range(B)])
                         for i in range(n)]).to(dev)
    w = torch.stack([torch.stack([stepq[i][b]["w"] for b in range(B)]) for i in range(n)]).to(dev)
    q_mla = torch.stack([torch.stack([stepq[i][b]["q_mla"] for b in range(B)])
                         for i in range(n)]).to(dev)
    k_new = torch.stack([torch.stack([base[b]["keys"][T0 - 1 + i] for b in range(B)])
                         for i in range(n)]).to(dev)
    K = min(wl.topk, T0)
    idx = torch.empty(n, B, K, dtype=torch.int32, device=dev)
    out = torch.empty(n, B, wl.Hq, wl.dc, dtype=dt, device=dev)
    lse = torch.empty(n, B, wl.Hq, dtype=torch.float32, device=dev)
    need = max(dsa.dsa_decode_step_workspace_size(B, wl.H, wl.D, T0 + i, wl.topk, wl.Hq, wl.dc,
                                                  wl.dr, dsa.DSA_BF16) for i in range(n))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    for i in range(n):
        dsa.dsa_decode_step(q_idx[i], w[i], k_new[i], k_cache, k_scale, kv, q_mla[i], T0 + i,
                            wl.topk, wl.softmax_scale_idx, wl.sm_scale, idx[i], out[i], lse[i],
                            ws)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
    for i in range(n):
        T = T0 + i
        for b in range(B):
            r = oracle.decode_step(stepq[i][b]["q_idx"].numpy(), stepq[i][b]["w"].numpy(),
                                   base[b]["keys"][:T].numpy(),
                                   stepq[i][b]["q_mla"].float().numpy(),
                                   base[b]["kv"][:T].float().numpy(), topk=wl.topk,
                                   softmax_scale_idx=wl.softmax_scale_idx, sm_scale=wl.sm_scale,
                                   dc=wl.dc)
            assert np.array_equal(k_cache[b, T - 1].cpu().numpy(), r["k_fp8"][T - 1])
            assert k_scale[b, T - 1].item() == r["k_scale"][T - 1]
            assert_selection_matches(idx[i, b].cpu().numpy(), r["idx"], r["scores"])
            assert_attention_close(out[i, b].float().cpu().numpy(), r["out"], wl.attn_dtype,
                                   lse[i, b].cpu().numpy(), r["lse"])
