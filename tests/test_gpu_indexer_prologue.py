"""The fused indexer prologue on the GPU against the oracle: RoPE (not
interleaved) + rotate_activation + act_quant (fp32 or ue8m0 scale) + the key
cache append.  FP8 codes and scales must be bit-identical; cache rows outside
[start_pos, start_pos + S) must be left as they were."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _angles(S, R, start_pos, base=10000.0):
    """cos / sin of position * base^(-2j/R), as a rotary table is built."""
    pos = np.arange(start_pos, start_pos + S, dtype=np.float64)[:, None]
    inv = base ** (-np.arange(0, R, 2, dtype=np.float64) / R)[None, :]
    th = pos * inv
    return np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32)   # [S, R/2, 2]


def _run(dsa, B, S, H, d, R, dtype, fmt, start_pos, t_max, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, S, H, d, generator=g) * scale).to(dtype) if H else None
    k = (torch.randn(B, S, d, generator=g) * scale).to(dtype)
    cs = _angles(S, R, start_pos) if R else None
    q_fp8 = torch.empty(B, S, H, d, dtype=torch.uint8, device="cuda") if H else None
    q_scale = torch.empty(B, S, H, dtype=torch.float32, device="cuda") if H else None
    k_cache = torch.full((B, t_max, d), 0xAB, dtype=torch.uint8, device="cuda")
    k_scale = torch.full((B, t_max), -1.0, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_prologue(q.cuda() if H else None, k.cuda(),
                             torch.from_numpy(cs).cuda() if R else None, start_pos,
                             q_fp8, q_scale, k_cache, k_scale, scale_fmt=fmt)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
    qn = q.float().numpy() if H else np.zeros((B, S, 0, d), np.float32)
    rq, rqs, rk, rks = oracle.indexer_prologue(qn, k.float().numpy(), cs, fmt)
    if H:
        assert np.array_equal(q_fp8.cpu().numpy(), rq)
        assert np.array_equal(q_scale.cpu().numpy(), rqs)
    kc, ksc = k_cache.cpu().numpy(), k_scale.cpu().numpy()
    rows = slice(start_pos, start_pos + S)
    assert np.array_equal(kc[:, rows], rk)
    assert np.array_equal(ksc[:, rows], rks)
    outside = np.ones(t_max, bool)
    outside[rows] = False
    assert np.all(kc[:, outside] == 0xAB) and np.all(ksc[:, outside] == -1.0)
    if fmt == dsa.DSA_SCALE_UE8M0 and H:
        m, _ = np.frexp(q_scale.cpu().numpy().astype(np.float64))
        assert np.all(m == 0.5)                       # bare powers of two


@pytest.mark.parametrize("B,S,H,d,R,dtype,fmt,start_pos,t_max", [
    (1, 1, 64, 128, 64, torch.float32, 0, 4095, 4096),     # decode token, V3.2 sizes
    (2, 5, 64, 128, 64, torch.bfloat16, 1, 100, 200),      # chunk of a prefill, ue8m0, bf16
    (1, 3, 4, 64, 16, torch.float32, 1, 0, 8),             # tiny sizes
    (2, 7, 3, 128, 128, torch.float32, 0, 10, 30),         # rotary over the whole vector
    (1, 4, 8, 128, 8, torch.bfloat16, 0, 2, 9),            # smallest rotary part
    (1, 4, 8, 128, 0, torch.float32, 1, 2, 10),            # no rotary part, ue8m0
    (3, 2, 0, 64, 32, torch.bfloat16, 0, 5, 9),            # keys only
    (1, 6, 16, 128, 32, torch.bfloat16, 0, 3, 12),         # lanes split on bit 3, angles staged
    (1, 6, 16, 128, 32, torch.float32, 1, 3, 12),          # rotary 32 in fp32: contiguous halves
    (2, 3, 5, 128, 16, torch.bfloat16, 0, 0, 5),           # few heads: angles read from the table
])
def test_prologue_matches_oracle(dsa, B, S, H, d, R, dtype, fmt, start_pos, t_max):
    _run(dsa, B, S, H, d, R, dtype, fmt, start_pos, t_max, seed=B * 100 + S * 10 + H + R)


@pytest.mark.parametrize("fmt", [0, 1])
def test_prologue_prefill_chunk_full_size(dsa, fmt):
    """2048 new tokens x 64 heads (131,072 query vectors) appended after 1000 cached ones."""
    _run(dsa, 1, 2048, 64, 128, 64, torch.float32, fmt, 1000, 4096, seed=7 + fmt)


def test_prologue_wide_dynamic_range(dsa):
    """Vectors scaled over 2^-20 .. 2^20: scales in both formats, tiny and large."""
    for i, sc in enumerate((2.0 ** -20, 2.0 ** -6, 2.0 ** 9, 2.0 ** 20)):
        _run(dsa, 1, 6, 16, 128, 64, torch.float32, i % 2, 0, 6, seed=30 + i, scale=sc)


def test_prologue_then_indexer_quant_agree_without_rotary(dsa):
    """With no rotary part and fp32 scales the prologue equals dsa_indexer_quant."""
    g = torch.Generator().manual_seed(9)
    q = torch.randn(2, 3, 8, 128, generator=g).cuda()
    k = torch.randn(2, 3, 128, generator=g).cuda()
    a_q = torch.empty(2, 3, 8, 128, dtype=torch.uint8, device="cuda")
    a_s = torch.empty(2, 3, 8, device="cuda")
    kc = torch.zeros(2, 8, 128, dtype=torch.uint8, device="cuda")
    ks = torch.zeros(2, 8, device="cuda")
    dsa.dsa_indexer_prologue(q, k, None, 4, a_q, a_s, kc, ks)
    b_q = torch.empty_like(a_q)
    b_s = torch.empty_like(a_s)
    dsa.dsa_indexer_quant(q, b_q, b_s)
    kc2 = torch.zeros_like(kc)
    ks2 = torch.zeros_like(ks)
    dsa.dsa_indexer_quant(k, kc2[:, 4:], ks2[:, 4:], n_rows=2, out_row_stride=8 * 128,
                          scale_row_stride=8)
    torch.cuda.synchronize()
    assert torch.equal(a_q, b_q) and torch.equal(a_s, b_s)
    assert torch.equal(kc, kc2) and torch.equal(ks, ks2)
