"""The decode step without a workspace (for callers that cannot allocate device
memory): same results as the workspace entry point, on two calls in a row.

Named so that pytest collects it last: its scratch array is shared by every
call on the device and keeps the previous call's contents, so this also checks
that nothing in it has to start at zero after the other tests ran.
"""
import ctypes

import pytest
import torch

import workloads
from gpu_pipelines import decode_batch
from parity import ATTN_ATOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def test_noalloc_decode_matches_workspace_entry_point(dsa):
    wl = workloads.WORKLOADS[1]
    T, B = 5000, 2
    _, st = decode_batch(dsa, wl, T=T, B=B)          # runs dsa_decode_step (workspace)
    ref_idx, ref_out, ref_lse = st["idx"].clone(), st["out"].clone(), st["lse"].clone()
    for _ in range(2):                                # two calls in a row
        idx = torch.full_like(ref_idx, -7)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        # re-appending the same new key at T-1 writes the same codes again
        dsa.dsa_decode_step_noalloc(st["q_idx"], st["w"], st["k_new"], st["k_cache"],
                                    st["k_scale"], st["kv"], st["q_mla"], T, wl.topk,
                                    wl.softmax_scale_idx, wl.sm_scale, idx, out, lse)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert (out.float() - ref_out.float()).abs().max().item() <= ATTN_ATOL["bf16"]
        assert (lse - ref_lse).abs().max().item() <= 1e-3
    assert dsa.dsa_get_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(dsa):
    wl = workloads.WORKLOADS[2]
    B, T = 64, 1 << 20                               # 256 MiB of score rows
    need = dsa.dsa_decode_step_workspace_size(B, wl.H, wl.D, T, wl.topk, wl.Hq, wl.dc, wl.dr,
                                              dsa.DSA_BF16)
    assert need > dsa.DSA_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    rc = dsa._lib.dsa_decode_step_noalloc(fake, fake, fake, fake, fake, T, fake, fake, B, wl.H,
                                          wl.D, wl.Hq, wl.dc, wl.dr, T, wl.topk, 0.08, 0.04,
                                          dsa.DSA_BF16, fake, fake, None, None)
    assert rc == dsa.DSA_ERR_WORKSPACE
