"""Pins of the oracle's FP8 latent row (the diagram "DeepSeek Sparse Attention,
one decode step in one layer (V3.2 sizes)": latents stored as "FP8 + bf16
RoPE", 656 B per row).  Reading: the 512 latent values in four blocks of 128,
each quantised like act_quant with its own fp32 scale, then the four scales,
then the 64 rotary values in bf16.  Checked against torch's e4m3 and bf16
casts, the e4m3 half-ulp bound and the diagram's byte counts."""
import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_latent_row_is_the_diagram_size():
    g = json.load(open(os.path.join(GOLDEN, "v32_decode_sizes.json")))
    dc = g["latent_width"] - g["rope_width_bf16"]
    assert oracle.latent_row_bytes(dc, g["rope_width_bf16"]) == g["latent_row_bytes"]
    x = np.random.default_rng(50).standard_normal((3, g["latent_width"])).astype(np.float32)
    assert oracle.latent_quant(x, dc).shape == (3, g["latent_row_bytes"])


def test_latent_row_layout_matches_library_casts():
    rng = np.random.default_rng(51)
    x = (rng.standard_normal((64, 576)) * np.exp2(rng.integers(-6, 6, (64, 1)))).astype(np.float32)
    rows = oracle.latent_quant(x, 512)
    codes, scales = rows[:, :512], rows[:, 512:528].copy().view(np.float32)
    rope = rows[:, 528:656].copy().view(np.uint16)
    for b in range(4):
        blk = x[:, 128 * b:128 * (b + 1)]
        amax = np.maximum(np.abs(blk).max(axis=1), np.float32(1e-4))
        assert np.array_equal(scales[:, b], (amax / np.float32(448.0)).astype(np.float32))
        q = blk / scales[:, b:b + 1]
        ref = torch.from_numpy(np.ascontiguousarray(q)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes[:, 128 * b:128 * (b + 1)], ref)
    ref_rope = torch.from_numpy(x[:, 512:]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(rope, ref_rope)


def test_latent_dequant_decodes_codes_times_block_scale():
    rng = np.random.default_rng(52)
    x = rng.standard_normal((16, 576)).astype(np.float32)
    rows = oracle.latent_quant(x, 512)
    y = oracle.latent_dequant(rows, 512, 64)
    dec = torch.from_numpy(rows[:, :512].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    sc = np.repeat(rows[:, 512:528].copy().view(np.float32), 128, axis=1).astype(np.float64)
    assert np.array_equal(y[:, :512], (dec * sc).astype(np.float32))
    # bf16-representable rotary values come back exactly
    xb = torch.from_numpy(x[:, 512:]).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y[:, 512:], xb)
    # the quantisation error stays within half an e4m3 step of each value / scale
    q = x[:, :512].astype(np.float64) / sc
    a = np.abs(q)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    half_ulp = np.exp2(e - 3) / 2
    assert np.all(np.abs(y[:, :512] - x[:, :512]) <= half_ulp * sc * (1 + 2.0 ** -20))


def test_latent_blocks_are_independent():
    rng = np.random.default_rng(53)
    x = rng.standard_normal((4, 576)).astype(np.float32)
    r0 = oracle.latent_quant(x, 512)
    x2 = x.copy()
    x2[:, 128:256] *= np.float32(8.0)                  # block 1 only, by a power of two
    r1 = oracle.latent_quant(x2, 512)
    assert np.array_equal(r1[:, :512], r0[:, :512])     # same codes everywhere
    s0, s1 = r0[:, 512:528].copy().view(np.float32), r1[:, 512:528].copy().view(np.float32)
    assert np.array_equal(s1[:, [0, 2, 3]], s0[:, [0, 2, 3]])
    assert np.array_equal(s1[:, 1], s0[:, 1] * np.float32(8.0))


def test_sparse_attention_over_fp8_rows_is_attention_over_decoded_bf16_rows():
    rng = np.random.default_rng(54)
    q = rng.standard_normal((1, 2, 8, 576)).astype(np.float32)
    kv = rng.standard_normal((1, 300, 576)).astype(np.float32)
    idx = np.sort(rng.permutation(300)[:40]).astype(np.int32).reshape(1, 1, 40).repeat(2, axis=1)
    rows = oracle.latent_quant(kv, 512)
    o8, l8 = oracle.sparse_mla_fp8(q, rows, idx, 299, 576 ** -0.5, 512, 64)
    # the decoded rows enter the bf16 attention as bf16 operands (torch's rounding)
    dec = torch.from_numpy(oracle.latent_dequant(rows, 512, 64)).to(torch.bfloat16).float().numpy()
    od, ld = oracle.sparse_mla(q, dec, idx, 299, 576 ** -0.5, 512)
    assert np.array_equal(o8, od) and np.array_equal(l8, ld)
    # and it tracks the unquantised attention to within the FP8 error
    o, _ = oracle.sparse_mla(q, kv, idx, 299, 576 ** -0.5, 512)
    assert np.abs(o8 - o).max() < 0.1
