"""rotate_activation + act_quant on the GPU: codes and scales bit-identical to the oracle."""
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


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n_vec", [1, 7, 33, 4099])
def test_indexer_quant_bit_exact(dsa, D, dtype, n_vec):
    g = torch.Generator().manual_seed(D * 7 + n_vec)
    x = torch.randn(n_vec, D, generator=g) * torch.exp2(torch.randint(-8, 8, (n_vec, 1),
                                                                      generator=g).float())
    x = x.to(dtype)
    out = torch.empty(n_vec, D, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n_vec, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(x.cuda(), out, sc)
    ref_c, ref_s = oracle.indexer_quant(x.float().numpy())
    assert np.array_equal(out.cpu().numpy(), ref_c)
    assert np.array_equal(sc.cpu().numpy(), ref_s)


def test_indexer_quant_special_values(dsa):
    D = 128
    x = torch.zeros(6, D)
    x[1, 5] = 1e-30                      # below the 1e-4 clamp
    x[2] = 3.0                           # constant vector: one nonzero Hadamard output
    x[3, ::2] = -2.5
    x[4] = torch.linspace(-1e6, 1e6, D)  # large range
    x[5, 0] = 1.0                        # a single spike
    out = torch.empty(6, D, dtype=torch.uint8, device="cuda")
    sc = torch.empty(6, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(x.cuda(), out, sc)
    ref_c, ref_s = oracle.indexer_quant(x.numpy())
    assert np.array_equal(out.cpu().numpy(), ref_c)
    assert np.array_equal(sc.cpu().numpy(), ref_s)


@pytest.mark.parametrize("cfg", [0, 1])
def test_cache_append_with_strides(dsa, cfg):
    """Keys [B,S,D] appended to k_cache [B,t_max,D] at start_pos, as the cache write does."""
    wl = workloads.WORKLOADS[cfg]
    B, S, t_max, sp, D = 3, 5, 40, 17, wl.D
    g = torch.Generator().manual_seed(cfg)
    keys = torch.randn(B, S, D, generator=g)
    k_cache = torch.full((B, t_max, D), 0xAB, dtype=torch.uint8, device="cuda")
    k_scale = torch.full((B, t_max), -1.0, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(keys.cuda(), k_cache[:, sp:], k_scale[:, sp:], n_rows=B,
                          out_row_stride=t_max * D, scale_row_stride=t_max)
    ref_c, ref_s = oracle.indexer_quant(keys.numpy())
    kc, ks = k_cache.cpu().numpy(), k_scale.cpu().numpy()
    assert np.array_equal(kc[:, sp:sp + S], ref_c)
    assert np.array_equal(ks[:, sp:sp + S], ref_s)
    assert np.all(kc[:, :sp] == 0xAB) and np.all(kc[:, sp + S:] == 0xAB)
    assert np.all(ks[:, :sp] == -1.0) and np.all(ks[:, sp + S:] == -1.0)


def test_indexer_quant_prefill_queries_full_size(dsa):
    """All 8192 x 64 query vectors of the T=8192 prefill, checked on a row sample."""
    wl = workloads.WORKLOADS[3]
    inp = workloads.prefill_inputs(wl)
    q = inp["q_idx"][0]                          # [T,H,D]
    out = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(q.cuda(), out, sc)
    rows = np.array([0, 1, 2047, 2048, 4095, 8191])
    ref_c, ref_s = oracle.indexer_quant(q[rows].numpy())
    assert np.array_equal(out.cpu().numpy()[rows], ref_c)
    assert np.array_equal(sc.cpu().numpy()[rows], ref_s)


def test_indexer_quant_bit_exact_many_vectors(dsa):
    """200,000 vectors of 128 (25.6 M quotients) over 2^-20 .. 2^20: every code and
    scale equals the oracle's, which divides with C's correctly rounded division."""
    n_vec, D = 200_000, 128
    g = torch.Generator().manual_seed(20)
    x = torch.randn(n_vec, D, generator=g) * torch.exp2(torch.randint(-20, 21, (n_vec, 1),
                                                                      generator=g).float())
    out = torch.empty(n_vec, D, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n_vec, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(x.cuda(), out, sc)
    ref_c, ref_s = oracle.indexer_quant(x.numpy())
    assert np.array_equal(sc.cpu().numpy(), ref_s)
    assert np.array_equal(out.cpu().numpy(), ref_c)
