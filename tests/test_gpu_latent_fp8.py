"""The FP8 latent cache on the GPU against the oracle: row quantisation
bit-identical (codes, block scales, bf16 rotary part), and sparse attention
over FP8 rows within the bf16 attention tolerance.  Both sides decode a row
as code * block scale rounded to bf16 (the attention's operand type), so the
decoded operands are identical and only the attention's arithmetic differs."""
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


def _gpu_rows(dsa, kv, dc, t_max=None, start=0):
    """Quantise kv [B, n, dc+dr] into a cache [B, t_max, row_bytes] at rows start..start+n-1."""
    B, n, dqk = kv.shape
    rb = dsa.dsa_latent_row_bytes(dc, dqk - dc)
    t_max = n if t_max is None else t_max
    cache = torch.full((B, t_max, rb), 0x5A, dtype=torch.uint8, device="cuda")
    dsa.dsa_latent_quant(kv.cuda(), cache[:, start:], dc, n_rows=B, out_row_stride=t_max * rb)
    torch.cuda.synchronize()
    return cache


@pytest.mark.parametrize("dtype,dc,dr", [(torch.bfloat16, 512, 64), (torch.float32, 512, 64),
                                         (torch.bfloat16, 256, 32), (torch.float32, 128, 8)])
def test_latent_quant_matches_oracle(dsa, dtype, dc, dr):
    g = torch.Generator().manual_seed(dc + dr)
    B, n, t_max, start = 2, 300, 400, 37
    kv = (torch.randn(B, n, dc + dr, generator=g) *
          torch.exp2(torch.randint(-10, 10, (B, n, 1), generator=g).float())).to(dtype)
    cache = _gpu_rows(dsa, kv, dc, t_max=t_max, start=start).cpu().numpy()
    ref = oracle.latent_quant(kv.float().numpy(), dc)
    assert ref.shape[-1] == dsa.dsa_latent_row_bytes(dc, dr)
    assert np.array_equal(cache[:, start:start + n], ref)
    assert np.all(cache[:, :start] == 0x5A) and np.all(cache[:, start + n:] == 0x5A)


@pytest.mark.parametrize("B,S,t_max,k,sp,fill", [
    (2, 1, 5000, 2048, 4999, 1.0),        # decode at the V3.2 sizes
    (2, 1, 3000, 2048, 2999, 0.6),        # -1 slots
    (1, 5, 2000, 512, 1500, 1.0),         # query rows with their own causal limits
    (3, 1, 300, 2048, 299, 1.0),          # fewer cached rows than k
    (1, 1, 5000, 1, 4999, 1.0),           # a single selected row
    (8, 1, 4096, 2048, 4095, 1.0),        # 256-row units (the decode bench's B)
    (5, 1, 3000, 2048, 2999, 0.8),        # 192-row units
])
def test_sparse_mla_fp8_matches_oracle(dsa, B, S, t_max, k, sp, fill):
    Hq, dc, dr = 128, 512, 64
    g = torch.Generator().manual_seed(B * 7 + S + k)
    q = torch.randn(B, S, Hq, dc + dr, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, t_max, dc + dr, generator=g).to(torch.bfloat16)
    idx = workloads.random_indices(B, S, k, t_max, sp, seed=B + S + k, fill=fill)
    cache = _gpu_rows(dsa, kv, dc)
    rows = cache.cpu().numpy()
    assert np.array_equal(rows, oracle.latent_quant(kv.float().numpy(), dc))
    sm = (dc + dr) ** -0.5
    need = dsa.dsa_sparse_mla_attn_fp8_workspace_size(B, S, Hq, dc, dr, k)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty(B, S, Hq, dc, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, S, Hq, dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_attn_fp8(q.cuda(), cache, idx.cuda(), sp, sm, dc, out, lse, ws)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
    ref, ref_lse = oracle.sparse_mla_fp8(q.float().numpy(), rows, idx.numpy(), sp, sm, dc, dr)
    assert_attention_close(out.float().cpu().numpy(), ref, "bf16", lse.cpu().numpy(), ref_lse)


def test_sparse_mla_fp8_empty_rows(dsa):
    B, Hq, dc, dr, t_max, k = 2, 128, 512, 64, 300, 64
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, 1, Hq, dc + dr, generator=g).to(torch.bfloat16).cuda()
    kv = torch.randn(B, t_max, dc + dr, generator=g).to(torch.bfloat16)
    cache = _gpu_rows(dsa, kv, dc)
    idx = torch.full((B, 1, k), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.dsa_sparse_mla_attn_fp8_workspace_size(B, 1, Hq, dc, dr, k),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(B, 1, Hq, dc, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, 1, Hq, dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_attn_fp8(q, cache, idx, t_max - 1, 0.04, dc, out, lse, ws)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isinf(lse) & (lse < 0))


def test_sparse_mla_fp8_other_shape_two_launch_path(dsa):
    """dc = 256: decoded into the workspace, then the bf16 attention."""
    B, S, Hq, dc, dr, t_max, k, sp = 1, 2, 16, 256, 32, 800, 128, 700
    g = torch.Generator().manual_seed(9)
    q = torch.randn(B, S, Hq, dc + dr, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, t_max, dc + dr, generator=g).to(torch.bfloat16)
    idx = workloads.random_indices(B, S, k, t_max, sp, seed=9, fill=0.9)
    cache = _gpu_rows(dsa, kv, dc)
    rows = cache.cpu().numpy()
    sm = (dc + dr) ** -0.5
    ws = torch.empty(max(dsa.dsa_sparse_mla_attn_fp8_workspace_size(B, S, Hq, dc, dr, k), 1),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(B, S, Hq, dc, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, S, Hq, dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_attn_fp8(q.cuda(), cache, idx.cuda(), sp, sm, dc, out, lse, ws)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.sparse_mla_fp8(q.float().numpy(), rows, idx.numpy(), sp, sm, dc, dr)
    assert_attention_close(out.float().cpu().numpy(), ref, "bf16", lse.cpu().numpy(), ref_lse)
