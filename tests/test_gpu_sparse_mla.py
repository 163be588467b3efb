"""Sparse latent attention on the GPU vs the oracle (bf16: 2e-2 abs, fp32: 1e-4 abs)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _case(B, S, Hq, dc, dr, t_max, k, sp, dtype, seed, fill=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, S, Hq, dc + dr, generator=g).to(dtype)
    kv = torch.randn(B, t_max, dc + dr, generator=g).to(dtype)
    idx = workloads.random_indices(B, S, k, t_max, sp, seed=seed, fill=fill)
    return q, kv, idx


def _gpu(dsa, q, kv, idx, sp, sm, dc):
    B, S, Hq, _ = q.shape
    k = idx.shape[-1]
    dt = dsa.DSA_BF16 if q.dtype == torch.bfloat16 else dsa.DSA_F32
    need = dsa.dsa_sparse_mla_attn_workspace_size(B, S, Hq, dc, q.shape[-1] - dc, k, dt)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, S, Hq, dc, dtype=q.dtype, device="cuda")
    lse = torch.empty(B, S, Hq, dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_attn(q.cuda(), kv.cuda(), idx.cuda(), sp, sm, out, lse, ws)
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("B,S,Hq,dc,dr,t_max,k,sp,dtype,fill", [
    (1, 1, 8, 64, 16, 128, 16, 127, "f32", 1.0),        # tiny config, fp32 test mode
    (1, 5, 8, 64, 16, 128, 16, 20, "f32", 0.5),         # half-empty rows
    (1, 1, 128, 512, 64, 4096, 2048, 4095, "bf16", 1.0),  # V3.2 decode shape
    (2, 1, 128, 512, 64, 3000, 2048, 2999, "bf16", 0.6),  # rows with -1 slots
    (3, 1, 128, 512, 64, 300, 2048, 299, "bf16", 1.0),  # fewer rows than k
    (1, 1, 128, 512, 64, 5000, 1, 4999, "bf16", 1.0),   # a single selected row
    (1, 3, 128, 512, 64, 4096, 2048, 3000, "f32", 1.0),  # V3.2 shape in fp32 test mode
    (4, 1, 128, 512, 64, 4096, 2048, 4095, "bf16", 1.0),  # 128-row units
    (5, 1, 128, 512, 64, 3000, 2048, 2999, "bf16", 0.8),  # 192-row units, -1 slots
    (8, 1, 128, 512, 64, 4096, 2048, 4095, "bf16", 1.0),  # 256-row units (the decode bench's B)
])
def test_sparse_mla_matches_oracle(dsa, B, S, Hq, dc, dr, t_max, k, sp, dtype, fill):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, kv, idx = _case(B, S, Hq, dc, dr, t_max, k, sp, tdt, seed=B + S + k + t_max, fill=fill)
    sm = (dc + dr) ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, sp, sm, dc)
    ref, ref_lse = oracle.sparse_mla(q.float().numpy(), kv.float().numpy(), idx.numpy(), sp, sm,
                                     dc)
    assert_attention_close(out, ref, dtype, lse, ref_lse)


def test_sparse_mla_masks_future_and_sentinels(dsa):
    """Entries past start_pos + s and -1 slots contribute nothing (index mask + causal mask)."""
    B, S, Hq, dc, dr, t_max = 1, 4, 128, 512, 64, 600
    q, kv, _ = _case(B, S, Hq, dc, dr, t_max, 64, 500, torch.bfloat16, seed=3)
    g = torch.Generator().manual_seed(5)
    idx = torch.randperm(t_max, generator=g)[:64].to(torch.int32).reshape(1, 1, 64).repeat(1, S, 1)
    idx[0, :, ::7] = -1
    sm = 576 ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, 500, sm, dc)
    ref, ref_lse = oracle.sparse_mla(q.float().numpy(), kv.float().numpy(), idx.numpy(), 500, sm,
                                     dc)
    assert_attention_close(out, ref, "bf16", lse, ref_lse)
    empty = torch.full((1, 1, 8), -1, dtype=torch.int32)
    out0, lse0 = _gpu(dsa, q[:, :1], kv, empty, 500, sm, dc)
    assert np.all(out0 == 0) and np.all(lse0 == -np.inf)


def test_sparse_mla_single_split_many_rows(dsa):
    """Enough rows that each (row, half) gets one CTA: output written directly."""
    B, Hq, dc, dr, t_max, k = 80, 128, 512, 64, 700, 256
    q, kv, idx = _case(B, 1, Hq, dc, dr, t_max, k, t_max - 1, torch.bfloat16, seed=21, fill=0.9)
    sm = 576 ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, t_max - 1, sm, dc)
    for b in (0, 41, 79):
        ref, ref_lse = oracle.sparse_mla(q[b:b + 1].float().numpy(), kv[b:b + 1].float().numpy(),
                                         idx[b:b + 1].numpy(), t_max - 1, sm, dc)
        assert_attention_close(out[b:b + 1], ref, "bf16", lse[b:b + 1], ref_lse)


def test_sparse_mla_growing_logits_force_rescale(dsa):
    """Logits grow along the (ascending) selection, so the running max keeps
    rising by more than the lazy-rescale threshold from tile to tile."""
    B, Hq, dc, dr, t_max, k = 2, 128, 512, 64, 4096, 2048
    g = torch.Generator().manual_seed(22)
    q = torch.randn(B, 1, Hq, dc + dr, generator=g)
    base = torch.randn(B, t_max, dc + dr, generator=g)
    ramp = torch.linspace(0, 6, t_max).reshape(1, t_max, 1)
    kv = base * 0.3 + ramp * q[:, 0, :1, :].sign()      # aligned with head 0's query signs
    q, kv = q.to(torch.bfloat16), kv.to(torch.bfloat16)
    idx = torch.sort(torch.randperm(t_max, generator=g)[:k].to(torch.int32)).values
    idx = idx.reshape(1, 1, k).repeat(B, 1, 1)
    sm = 576 ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, t_max - 1, sm, dc)
    ref, ref_lse = oracle.sparse_mla(q.float().numpy(), kv.float().numpy(), idx.numpy(),
                                     t_max - 1, sm, dc)
    assert_attention_close(out, ref, "bf16", lse, ref_lse)


def test_sparse_mla_all_slots_empty_bf16(dsa):
    B, Hq, dc, dr, t_max = 3, 128, 512, 64, 300
    q, kv, _ = _case(B, 1, Hq, dc, dr, t_max, 8, t_max - 1, torch.bfloat16, seed=23)
    idx = torch.full((B, 1, 2048), -1, dtype=torch.int32)
    out, lse = _gpu(dsa, q, kv, idx, t_max - 1, 0.04, dc)
    assert np.all(out == 0) and np.all(lse == -np.inf)


def test_sparse_mla_prefill_rows_bf16(dsa):
    """S > 1 query rows with their own causal limits (start_pos + s)."""
    B, S, Hq, dc, dr, t_max, k, sp = 1, 5, 128, 512, 64, 2000, 512, 1500
    q, kv, idx = _case(B, S, Hq, dc, dr, t_max, k, sp, torch.bfloat16, seed=24)
    sm = 576 ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, sp, sm, dc)
    ref, ref_lse = oracle.sparse_mla(q.float().numpy(), kv.float().numpy(), idx.numpy(), sp, sm, dc)
    assert_attention_close(out, ref, "bf16", lse, ref_lse)


def test_sparse_mla_split_partials_keep_range(dsa):
    """Latent values far beyond the fp16 range of the split partials.

    The cache is scaled by 2^20 and the query by 2^-20 (exact in bf16), so the
    logits, the softmax and the log-sum-exp are unchanged and the output is
    2^20 times the unscaled one; one row over 2048 selections runs as many
    splits, whose partials are stored in fp16 with a power-of-two scale.
    """
    B, S, Hq, dc, dr, t_max, k = 1, 1, 128, 512, 64, 4096, 2048
    q, kv, idx = _case(B, S, Hq, dc, dr, t_max, k, t_max - 1, torch.bfloat16, seed=33)
    sm = (dc + dr) ** -0.5
    big = 2.0 ** 20
    out, lse = _gpu(dsa, (q.float() / big).to(torch.bfloat16), (kv.float() * big).to(torch.bfloat16),
                    idx, t_max - 1, sm, dc)
    assert np.all(np.isfinite(out))
    ref, ref_lse = oracle.sparse_mla(q.float().numpy(), kv.float().numpy(), idx.numpy(), t_max - 1,
                                     sm, dc)
    assert_attention_close(out / big, ref, "bf16", lse, ref_lse)


@pytest.mark.parametrize("B,k", [(40, 512), (20, 1024)])
def test_sparse_mla_rows_of_two_and_four_units(dsa, B, k):
    """Rows whose selections span 2 (k = 512) or 4 (k = 1024) units of 256 rows
    when the rows fill the GPU, merged by the split combine."""
    Hq, dc, dr, t_max = 128, 512, 64, 3000
    q, kv, idx = _case(B, 1, Hq, dc, dr, t_max, k, t_max - 1, torch.bfloat16, seed=B + k, fill=0.9)
    sm = 576 ** -0.5
    out, lse = _gpu(dsa, q, kv, idx, t_max - 1, sm, dc)
    for b in (0, B // 2, B - 1):
        ref, ref_lse = oracle.sparse_mla(q[b:b + 1].float().numpy(), kv[b:b + 1].float().numpy(),
                                         idx[b:b + 1].numpy(), t_max - 1, sm, dc)
        assert_attention_close(out[b:b + 1], ref, "bf16", lse[b:b + 1], ref_lse)
