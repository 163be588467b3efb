"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against a closed form, a library routine
(torch's float8_e4m3fn cast, scipy's Hadamard matrix, numpy sorts/einsums,
scipy's softmax), an invariant, or brute force on tiny inputs, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, a
wrong rounding mode) fails at least one of them.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- #
# e4m3fn (OCP FP8: 1-4-3, bias 7, max 448, no inf)
# --------------------------------------------------------------------------- #
def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_closed_form_and_library():
    table = oracle.e4m3_decode(np.arange(256))
    ref = _torch_e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(table), nan)
    assert np.array_equal(table[~nan], ref[~nan])
    assert nan.sum() == 2 and np.isnan(table[0x7F]) and np.isnan(table[0xFF])
    assert table[0x7E] == 448.0 and table[0xFE] == -448.0
    assert table[0x01] == 2.0 ** -9 and table[0x08] == 2.0 ** -6 and table[0x38] == 1.0


def _boundary_points():
    vals = np.unique(np.abs(_torch_e4m3_values()[~np.isnan(_torch_e4m3_values())]))
    vals = vals.astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1].astype(np.float64) + vals[1:]) / 2)
    pts = np.concatenate([vals, mids])
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(-np.inf))
    pts = np.concatenate([pts, up, dn, [np.float32(464.0) - np.float32(2 ** -16)]])
    pts = pts[np.abs(pts) < 464.0]
    return np.concatenate([pts, -pts]).astype(np.float32)


def test_e4m3_encode_matches_torch_at_rounding_boundaries():
    x = _boundary_points()
    got = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_matches_torch_random():
    rng = np.random.default_rng(1)
    mag = np.exp2(rng.uniform(-16, np.log2(463.99), size=2_000_000))
    sign = rng.choice([-1.0, 1.0], size=mag.size)
    x = (sign * mag).astype(np.float32)
    x = np.concatenate([x, rng.uniform(-463.9, 463.9, size=500_000).astype(np.float32)])
    got = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates_and_nan():
    big = np.array([448.0, 463.9, 464.0, 480.0, 1e4, 3.0e38, np.inf], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    assert oracle.e4m3_encode(np.array([np.nan], dtype=np.float32))[0] & 0x7F == 0x7F


def test_e4m3_roundtrip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


# --------------------------------------------------------------------------- #
# rotate_activation: Walsh-Hadamard, orthonormal
# --------------------------------------------------------------------------- #
def test_hadamard_scale_is_nearest_fp32():
    getcontext().prec = 60
    for D in (2, 4, 8, 16, 32, 64, 128, 256):
        s = oracle.hadamard_scale(D)
        exact = Decimal(1) / Decimal(D).sqrt()
        err = abs(Decimal(float(s)) - exact)
        half_ulp = Decimal(float(np.spacing(s))) / 2
        assert err <= half_ulp


def test_fwht_d2_closed_form():
    x = np.array([[3.0, 1.0], [1.5, -2.25]], dtype=np.float32)
    y = oracle.fwht(x)
    r = 1 / math.sqrt(2)
    ref = np.array([[4 * r, 2 * r], [-0.75 * r, 3.75 * r]])
    assert np.allclose(y, ref, rtol=2e-7, atol=0)


@pytest.mark.parametrize("D", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_equals_sylvester_matrix(D):
    Hm = scipy.linalg.hadamard(D).astype(np.float64) / math.sqrt(D)
    eye = oracle.fwht(np.eye(D, dtype=np.float32))
    assert np.allclose(eye, Hm.T, atol=1e-7, rtol=0)
    rng = np.random.default_rng(D)
    x = rng.standard_normal((16, D)).astype(np.float32)
    y = oracle.fwht(x).astype(np.float64)
    ref = x.astype(np.float64) @ Hm.T
    assert np.allclose(y, ref, atol=1e-5 * np.abs(x).max(), rtol=0)


def test_fwht_orthonormal_involution_and_dot_invariance():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((32, 128)).astype(np.float32)
    k = rng.standard_normal((32, 128)).astype(np.float32)
    hx, hk = oracle.fwht(x), oracle.fwht(k)
    assert np.allclose(oracle.fwht(hx), x, atol=2e-6)
    assert np.allclose(np.linalg.norm(hx, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)
    dots = np.einsum("rd,rd->r", x.astype(np.float64), k.astype(np.float64))
    hdots = np.einsum("rd,rd->r", hx.astype(np.float64), hk.astype(np.float64))
    assert np.allclose(hdots, dots, atol=1e-4)


# --------------------------------------------------------------------------- #
# act_quant: blockwise e4m3 with s = amax / 448
# --------------------------------------------------------------------------- #
def _e4m3_half_ulp(v):
    a = np.abs(v).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3) / 2


def test_act_quant_error_within_half_ulp():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((256, 128)) * np.exp2(rng.integers(-6, 6, (256, 1)))).astype(np.float32)
    y, s = oracle.act_quant(x, 128)
    q = x / s                                 # the fp32 quotient the quantiser rounds
    dec = oracle.e4m3_decode(y)
    assert np.all(np.abs(dec - q.astype(np.float64)) <= _e4m3_half_ulp(q))


def test_act_quant_max_element_maps_to_448():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    y, s = oracle.act_quant(x, 128)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s[:, 0], (amax / np.float32(448.0)).astype(np.float32))
    i = np.abs(x).argmax(axis=1)
    picked = y[np.arange(64), i]
    assert np.all((picked == 0x7E) | (picked == 0xFE))
    assert np.all((picked == 0xFE) == (x[np.arange(64), i] < 0))


def test_act_quant_power_of_two_equivariance():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    y0, s0 = oracle.act_quant(x, 128)
    for k in (-5, -1, 1, 3, 7):
        y, s = oracle.act_quant(x * np.float32(2.0 ** k), 128)
        assert np.array_equal(y, y0)
        assert np.array_equal(s, s0 * np.float32(2.0 ** k))


def test_act_quant_zero_block_and_independent_blocks():
    y, s = oracle.act_quant(np.zeros((1, 128), np.float32), 128)
    assert np.all(y == 0) and s[0, 0] == np.float32(np.float32(1e-4) / np.float32(448.0))
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    yb, sb = oracle.act_quant(x, 32)
    for j in range(4):
        yj, sj = oracle.act_quant(x[:, 32 * j:32 * (j + 1)], 32)
        assert np.array_equal(yb[:, 32 * j:32 * (j + 1)], yj)
        assert np.array_equal(sb[:, j], sj[:, 0])


def test_golden_v32_row_sizes():
    g = json.load(open(os.path.join(GOLDEN, "v32_decode_sizes.json")))
    rng = np.random.default_rng(0)
    k = rng.standard_normal((1, g["indexer_head_dim"])).astype(np.float32)
    codes, scale = oracle.indexer_quant(k)
    # one FP8 byte per dim plus one fp32 scale per token = the 132 B row
    assert codes.nbytes + scale.nbytes == g["indexer_key_bytes_per_token"]
    # the latent row reading: 512 FP8 + four fp32 per-128 scales + 64 bf16 rope
    assert 512 * 1 + (512 // 128) * 4 + g["rope_width_bf16"] * 2 == g["latent_row_bytes"]
    assert 512 + g["rope_width_bf16"] == g["latent_width"]
    assert g["latent_row_bytes"] + g["indexer_key_bytes_per_token"] == g["bytes_per_token_per_layer"]
    assert g["bytes_per_token_per_layer"] * g["layers"] == g["bytes_per_token_all_layers"]
    assert workloads.WORKLOADS[4].H == g["indexer_heads"]
    assert workloads.WORKLOADS[4].D == g["indexer_head_dim"]
    assert workloads.WORKLOADS[4].topk == g["topk"]
    assert workloads.WORKLOADS[4].Hq == g["mla_heads"]
    assert workloads.WORKLOADS[4].dqk == g["latent_width"]


# --------------------------------------------------------------------------- #
# weight fold and fp8_index scoring
# --------------------------------------------------------------------------- #
def test_weight_fold_matches_page_expression_in_torch():
    # the Indexer.forward weight step, evaluated by torch in fp32: the projected
    # weights times H^-1/2, then times each head's query scale and the softmax scale
    rng = np.random.default_rng(8)
    for H in (4, 64, 3):
        w = torch.from_numpy(rng.standard_normal(H).astype(np.float32))
        qs = torch.from_numpy((rng.random(H) * 0.02 + 1e-3).astype(np.float32))
        sm = 128 ** -0.5
        ref = (w * H ** -0.5).unsqueeze(-1) * qs.unsqueeze(-1) * sm
        got = [oracle.weight_fold(float(w[h]), H, float(qs[h]), sm) for h in range(H)]
        assert np.array_equal(np.array(got, np.float32), ref[:, 0].numpy())


def _rand_codes(rng, shape, positive=None):
    codes = rng.integers(0, 0x7E, size=shape, dtype=np.uint8)    # finite, non-negative
    if positive is None:
        codes |= (rng.integers(0, 2, size=shape, dtype=np.uint8) << 7)
    elif not positive:
        codes |= 0x80
    return codes


def _brute_scores(q_fp8, q_scale, w, k_cache, k_scale, start_pos, T, sm):
    B, S, H, D = q_fp8.shape
    qd = oracle.e4m3_decode(q_fp8)
    kd = oracle.e4m3_decode(k_cache[:, :T])
    dots = np.einsum("bshd,btd->bsht", qd, kd)
    wt = torch.from_numpy(w) * H ** -0.5
    wt = (wt.unsqueeze(-1) * torch.from_numpy(q_scale).unsqueeze(-1) * sm)[..., 0].numpy()
    sc = np.einsum("bsh,bsht->bst", wt.astype(np.float64), np.maximum(dots, 0.0))
    sc = sc * k_scale[:, None, :T].astype(np.float64)
    s_idx = np.arange(S)[None, :, None]
    t_idx = np.arange(T)[None, None, :]
    return np.where(t_idx > start_pos + s_idx, -np.inf, sc).astype(np.float32)


def test_scores_brute_force_tiny():
    rng = np.random.default_rng(9)
    B, S, H, D, t_max, T, sp = 2, 3, 4, 64, 12, 10, 7
    q = _rand_codes(rng, (B, S, H, D))
    qs = (rng.random((B, S, H)) * 0.01 + 1e-3).astype(np.float32)
    w = rng.standard_normal((B, S, H)).astype(np.float32)
    k = _rand_codes(rng, (B, t_max, D))
    ks = (rng.random((B, t_max)) * 0.01 + 1e-3).astype(np.float32)
    got = oracle.index_scores(q, qs, w, k, ks, sp, T, 0.125)
    ref = _brute_scores(q, qs, w, k, ks, sp, T, 0.125)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(got[~fin] == -np.inf)
    assert np.allclose(got[fin], ref[fin], rtol=1e-6, atol=0)
    # the mask is exactly triu(1) offset by start_pos
    for s in range(S):
        assert np.all(np.isfinite(got[:, s, :sp + s + 1]))
        assert np.all(got[:, s, sp + s + 1:] == -np.inf)


def test_scores_single_head_closed_form():
    rng = np.random.default_rng(10)
    q = _rand_codes(rng, (1, 1, 1, 128))
    k = _rand_codes(rng, (1, 50, 128))
    ks = (rng.random((1, 50)) + 0.5).astype(np.float32)
    qs = np.array([[[0.01]]], np.float32)
    got = oracle.index_scores(q, qs, np.ones((1, 1, 1), np.float32), k, ks, 49, 50, 1.0)
    dots = oracle.e4m3_decode(k[0]) @ oracle.e4m3_decode(q[0, 0, 0])
    ref = (np.float64(np.float32(0.01)) * np.maximum(dots, 0) * ks[0]).astype(np.float32)
    assert np.array_equal(got[0, 0], ref)


def test_scores_homogeneous_in_key_scale_and_zero_for_negative_dots():
    rng = np.random.default_rng(11)
    q = _rand_codes(rng, (1, 1, 8, 64))
    k = _rand_codes(rng, (1, 40, 64))
    ks = (rng.random((1, 40)) * 0.01 + 1e-3).astype(np.float32)
    qs = (rng.random((1, 1, 8)) * 0.01 + 1e-3).astype(np.float32)
    w = rng.standard_normal((1, 1, 8)).astype(np.float32)
    a = oracle.index_scores(q, qs, w, k, ks, 39, 40, 0.125)
    b = oracle.index_scores(q, qs, w, k, ks * 2, 39, 40, 0.125)
    assert np.array_equal(b, a * 2)
    qp = _rand_codes(rng, (1, 1, 8, 64), positive=True)
    kn = _rand_codes(rng, (1, 40, 64), positive=False)
    z = oracle.index_scores(qp, qs, w, kn, ks, 39, 40, 0.125)
    assert np.all(z == 0.0)


def test_scores_head_permutation_invariance():
    rng = np.random.default_rng(12)
    q = _rand_codes(rng, (1, 2, 16, 64))
    k = _rand_codes(rng, (1, 30, 64))
    ks = (rng.random((1, 30)) * 0.01 + 1e-3).astype(np.float32)
    qs = (rng.random((1, 2, 16)) * 0.01 + 1e-3).astype(np.float32)
    w = rng.standard_normal((1, 2, 16)).astype(np.float32)
    p = rng.permutation(16)
    a = oracle.index_scores(q, qs, w, k, ks, 28, 30, 0.125)
    b = oracle.index_scores(q[:, :, p], qs[:, :, p], w[:, :, p], k, ks, 28, 30, 0.125)
    fin = np.isfinite(a)
    assert np.allclose(a[fin], b[fin], rtol=1e-6, atol=1e-30)


def test_scores_track_unquantised_definition_within_fp8_bound():
    """I ~= sum_h w_h H^-1/2 sm ReLU(q_h . k): the rotation preserves dot products,
    FP8 only perturbs each rotated element by at most half an e4m3 ulp."""
    rng = np.random.default_rng(13)
    H, D, T = 16, 128, 64
    q = rng.standard_normal((H, D)).astype(np.float32)
    keys = rng.standard_normal((T, D)).astype(np.float32)
    w = rng.standard_normal(H).astype(np.float32)
    sm = D ** -0.5
    kf, ks = oracle.indexer_quant(keys)
    qf, qs = oracle.indexer_quant(q)
    got = oracle.index_scores(qf[None, None], qs[None, None], w[None, None], kf[None],
                              ks[None], T - 1, T, sm)[0, 0].astype(np.float64)
    q64, k64 = q.astype(np.float64), keys.astype(np.float64)
    exact = (np.maximum(k64 @ q64.T, 0) * (w.astype(np.float64) * H ** -0.5 * sm)).sum(1)
    Hm = scipy.linalg.hadamard(D) / math.sqrt(D)
    u, v = q64 @ Hm.T, k64 @ Hm.T                        # rotated, unquantised
    du = np.abs(u) * 2.0 ** -4 + qs[:, None].astype(np.float64) * 2.0 ** -10 + 1e-6 * np.abs(u)
    dv = np.abs(v) * 2.0 ** -4 + ks[:, None].astype(np.float64) * 2.0 ** -10 + 1e-6 * np.abs(v)
    dot_err = np.abs(v) @ du.T + dv @ np.abs(u).T + dv @ du.T   # [T,H]
    bound = (dot_err * np.abs(w.astype(np.float64) * H ** -0.5 * sm)).sum(1)
    assert np.all(np.abs(got - exact) <= bound + 1e-6)
    # FP8 errors are unbiased, so the observed error sits far inside the worst
    # case: a dropped head, a sign slip or a wrong scale would be O(spread)
    err = np.abs(got - exact)
    assert np.sqrt((err ** 2).mean()) < 0.03 * np.sqrt((exact ** 2).mean())


# --------------------------------------------------------------------------- #
# top-k selection
# --------------------------------------------------------------------------- #
def _lexsort_select(row_scores, n_valid, K):
    t = np.arange(n_valid)
    order = np.lexsort((t, -row_scores[:n_valid].astype(np.float64)))
    return np.sort(order[:min(K, n_valid)])


def test_topk_matches_lexsort_on_tie_free_rows():
    s = workloads.score_rows(6, 300, seed=1).numpy()[None]       # [1,6,300]
    for sp, k in ((299, 16), (100, 50), (0, 7), (294, 400)):
        S = 6 if sp + 5 < 300 else 1
        sc = s[:, :S]
        idx = oracle.topk_select(sc, sp, k)
        K = min(k, 300)
        assert idx.shape == (1, S, K)
        for r in range(S):
            n_valid = min(300, sp + r + 1)
            sel = _lexsort_select(sc[0, r], n_valid, K)
            assert np.array_equal(idx[0, r, :len(sel)], sel)
            assert np.all(idx[0, r, len(sel):] == -1)


def test_topk_ties_take_lower_position_and_zero_signs_tie():
    sc = np.full((1, 1, 20), 1.5, np.float32)
    assert np.array_equal(oracle.topk_select(sc, 19, 5)[0, 0], np.arange(5))
    sc = np.zeros((1, 1, 6), np.float32)
    sc[0, 0, [0, 2, 4]] = -0.0
    assert np.array_equal(oracle.topk_select(sc, 5, 3)[0, 0], [0, 1, 2])
    s2 = workloads.score_rows(4, 500, seed=2, tie_frac=0.3).numpy()[None]
    idx = oracle.topk_select(s2, 499, 64)
    for r in range(4):
        assert np.array_equal(idx[0, r], _lexsort_select(s2[0, r], 500, 64))


def test_topk_causal_prefill_never_future_and_all_when_short():
    T, k = 64, 16
    sc = workloads.score_rows(T, T, seed=3).numpy()[None]       # prefill: S = T
    idx = oracle.topk_select(sc, 0, k)
    for s in range(T):
        row = idx[0, s]
        valid = row[row >= 0]
        assert np.all(valid <= s)
        if s + 1 <= k:
            assert np.array_equal(valid, np.arange(s + 1))
            assert np.all(row[s + 1:] == -1)
        else:
            assert len(valid) == k


def test_topk_k_larger_than_T():
    sc = workloads.score_rows(1, 10, seed=4).numpy()[None]
    idx = oracle.topk_select(sc, 9, 2048)
    assert idx.shape == (1, 1, 10) and np.array_equal(idx[0, 0], np.arange(10))


# --------------------------------------------------------------------------- #
# sparse latent attention
# --------------------------------------------------------------------------- #
def _dense_latent_attention(q, kv, s_pos, sm, dc):
    """Softmax over every causal position (scipy), latent row as key and value."""
    qh = q.astype(np.float64)                              # [Hq, dqk]
    keys = kv[:s_pos + 1].astype(np.float64)               # [n, dqk]
    z = sm * (qh @ keys.T)
    p = scipy.special.softmax(z, axis=-1)
    return p @ keys[:, :dc], scipy.special.logsumexp(z, axis=-1)


def test_sparse_equals_dense_causal_when_k_ge_T():
    wl = workloads.WORKLOADS[0]
    rng = np.random.default_rng(14)
    T, Hq, dc, dr = 40, wl.Hq, wl.dc, wl.dr
    q = rng.standard_normal((1, T, Hq, dc + dr)).astype(np.float32)
    kv = rng.standard_normal((1, T, dc + dr)).astype(np.float32)
    sc = rng.standard_normal((1, T, T)).astype(np.float32)
    idx = oracle.topk_select(sc, 0, 2048)                  # k >= T: all causal
    out, lse = oracle.sparse_mla(q, kv, idx, 0, wl.sm_scale, dc)
    for s in (0, 1, 17, T - 1):
        ref, rl = _dense_latent_attention(q[0, s], kv[0], s, wl.sm_scale, dc)
        assert np.allclose(out[0, s], ref, rtol=1e-5, atol=1e-6)
        assert np.allclose(lse[0, s], rl, rtol=1e-6)


def test_sparse_equals_index_mask_formulation():
    """The MLA prefill excerpt's formulation: an index mask, -inf except at the
    selected positions, plus the causal mask, added to the scaled scores;
    softmax; mix (latent row as key and value)."""
    rng = np.random.default_rng(15)
    T, Hq, dc, dr, k = 30, 4, 32, 8, 6
    q = torch.from_numpy(rng.standard_normal((1, T, Hq, dc + dr)))
    kv = torch.from_numpy(rng.standard_normal((1, T, dc + dr)))
    sc = workloads.score_rows(T, T, seed=5).numpy()[None]
    idx = oracle.topk_select(sc, 0, k)
    sm = (dc + dr) ** -0.5
    scores = torch.einsum("bshd,btd->bsht", q, kv) * sm
    topk = torch.from_numpy(idx.astype(np.int64))
    index_mask = torch.full((1, T, T), float("-inf"), dtype=torch.float64)
    for s in range(T):
        sel = topk[0, s][topk[0, s] >= 0]
        index_mask[0, s].scatter_(-1, sel, 0.0)
    mask = torch.full((T, T), float("-inf"), dtype=torch.float64).triu_(1)
    index_mask += mask
    scores = scores + index_mask.unsqueeze(2)
    ref = torch.einsum("bsht,btd->bshd", scores.softmax(dim=-1), kv[..., :dc]).numpy()
    out, _ = oracle.sparse_mla(q.numpy(), kv.numpy(), idx, 0, sm, dc)
    assert np.allclose(out, ref, rtol=1e-5, atol=1e-6)


def test_sparse_single_row_zero_query_sentinels_and_empty():
    rng = np.random.default_rng(16)
    T, Hq, dc, dr = 20, 3, 16, 4
    q = rng.standard_normal((1, 1, Hq, dc + dr)).astype(np.float32)
    kv = rng.standard_normal((1, T, dc + dr)).astype(np.float32)
    idx = np.array([[[-1, 7, -1, -1]]], np.int32)
    out, lse = oracle.sparse_mla(q, kv, idx, 19, 0.3, dc)
    assert np.array_equal(out[0, 0], np.broadcast_to(kv[0, 7, :dc], (Hq, dc)))
    z = 0.3 * (q[0, 0].astype(np.float64) @ kv[0, 7].astype(np.float64))
    assert np.allclose(lse[0, 0], z, rtol=1e-6)
    sel = [2, 5, 11, 19]
    out0, _ = oracle.sparse_mla(np.zeros_like(q), kv, np.array([[sel]], np.int32), 19, 0.3, dc)
    assert np.allclose(out0[0, 0], np.broadcast_to(kv[0, sel, :dc].mean(0), (Hq, dc)), atol=1e-6)
    # -1 slots and positions past the causal limit contribute nothing
    a, _ = oracle.sparse_mla(q, kv, np.array([[[2, 5, -1, 11, 15]]], np.int32), 12, 0.3, dc)
    b, _ = oracle.sparse_mla(q, kv, np.array([[[2, 5, 11]]], np.int32), 12, 0.3, dc)
    assert np.array_equal(a, b)
    e, le = oracle.sparse_mla(q, kv, np.full((1, 1, 4), -1, np.int32), 19, 0.3, dc)
    assert np.all(e == 0) and np.all(le == -np.inf)


def test_sparse_latent_mode_equals_up_projected_heads():
    """MQA (absorbed) mode equals the MHA prefill form with per-head up-projections:
    q_nope.(W_UK c) = (W_UK^T q_nope).c and sum p (W_UV c) = W_UV (sum p c)."""
    rng = np.random.default_rng(17)
    T, Hq, dc, dr, dn, dv = 25, 3, 16, 4, 8, 12
    Wuk = rng.standard_normal((Hq, dc, dn))
    Wuv = rng.standard_normal((Hq, dc, dv))
    q_nope = rng.standard_normal((Hq, dn))
    q_pe = rng.standard_normal((Hq, dr))
    c = rng.standard_normal((T, dc))
    k_pe = rng.standard_normal((T, dr))
    sm = 0.2
    s = T - 1
    sel = np.array([0, 3, 4, 9, 16, 24], np.int32)
    # MHA form: k = [W_UK c | k_pe], v = W_UV c, per head
    ref = np.empty((Hq, dv))
    for h in range(Hq):
        kn = c[sel] @ Wuk[h]
        z = sm * (kn @ q_nope[h] + k_pe[sel] @ q_pe[h])
        p = scipy.special.softmax(z)
        ref[h] = p @ (c[sel] @ Wuv[h])
    q_lat = np.einsum("hcn,hn->hc", Wuk, q_nope)
    q = np.concatenate([q_lat, q_pe], axis=1).astype(np.float32)[None, None]
    kv = np.concatenate([c, k_pe], axis=1).astype(np.float32)[None]
    o_lat, _ = oracle.sparse_mla(q, kv, sel[None, None], s, sm, dc)
    got = np.einsum("hc,hcv->hv", o_lat[0, 0].astype(np.float64), Wuv)
    assert np.allclose(got, ref, rtol=1e-4, atol=1e-4)


# --------------------------------------------------------------------------- #
# composed passes
# --------------------------------------------------------------------------- #
def test_decode_short_context_selects_everything_and_is_deterministic():
    wl = workloads.WORKLOADS[1]
    inp = workloads.decode_sequence(wl, 0, T=300)
    kw = dict(topk=wl.topk, softmax_scale_idx=wl.softmax_scale_idx, sm_scale=wl.sm_scale,
              dc=wl.dc)
    args = (inp["q_idx"].numpy(), inp["w"].numpy(), inp["keys"].numpy(),
            inp["q_mla"].float().numpy(), inp["kv"].float().numpy())
    r1 = oracle.decode_step(*args, **kw)
    r2 = oracle.decode_step(*args, **kw)
    assert r1["idx"].shape == (300,) and np.array_equal(r1["idx"], np.arange(300))
    for key in r1:
        assert np.array_equal(r1[key], r2[key])


def _planted_check(T):
    wl = workloads.WORKLOADS[4]
    inp = workloads.decode_sequence(wl, 0, T=T)
    r = oracle.decode_step(inp["q_idx"].numpy(), inp["w"].numpy(), inp["keys"].numpy(),
                           inp["q_mla"].float().numpy(), inp["kv"].float().numpy(),
                           topk=wl.topk, softmax_scale_idx=wl.softmax_scale_idx,
                           sm_scale=wl.sm_scale, dc=wl.dc)
    planted = inp["planted"].numpy()
    assert len(planted) == int(0.01 * T)
    assert np.isin(planted, r["idx"]).all()
    assert np.all(r["idx"] >= 0) and len(np.unique(r["idx"])) == wl.topk


def test_decode_planted_positions_selected_16k():
    _planted_check(16384)


@pytest.mark.slow
def test_decode_planted_positions_selected_full_128k():
    _planted_check(131072)


def test_prefill_rows_agree_with_full_matrix():
    wl = workloads.WORKLOADS[0]
    inp = workloads.prefill_inputs(wl)
    T = wl.T
    rows = [0, 5, 15, 16, 63, 127]
    r = oracle.prefill_rows(inp["q_idx"][0].numpy(), inp["w"][0].numpy(),
                            inp["keys"][0].numpy(), inp["q_mla"][0].float().numpy(),
                            inp["kv"][0].float().numpy(), rows, topk=wl.topk,
                            softmax_scale_idx=wl.softmax_scale_idx, sm_scale=wl.sm_scale,
                            dc=wl.dc)
    kf, ks = oracle.indexer_quant(inp["keys"].numpy())
    qf, qs = oracle.indexer_quant(inp["q_idx"].numpy())
    full = oracle.index_scores(qf, qs, inp["w"].numpy(), kf, ks, 0, T, wl.softmax_scale_idx)
    assert np.array_equal(r["scores"], full[0, rows])
    idx = oracle.topk_select(full, 0, wl.topk)
    assert np.array_equal(r["idx"], idx[0, rows])
    for j, s in enumerate(rows):
        if s + 1 <= wl.K:
            assert np.array_equal(r["idx"][j][:s + 1], np.arange(s + 1))
