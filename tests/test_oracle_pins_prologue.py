"""Pins of the oracle's indexer prologue: non-interleaved RoPE, the ue8m0 scale
format and their composition with rotate_activation and act_quant.

The page ("DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward) gives the
first rope_head_dim elements the rotary embedding (not interleaved), then
rotates and quantises with the configured scale format; it does not print the
rotary function or the scale format.  These tests check the oracle
against numpy complex arithmetic, scipy's Hadamard matrix, torch's e4m3 cast,
exact special angles and invariants, so that a swapped pairing (interleaved
instead of split halves), a sign slip or a wrong rounding of the scale fails.
"""
import numpy as np
import scipy.linalg
import torch

import oracle


def _angles(rng, shape):
    th = rng.uniform(-np.pi, np.pi, shape)
    return np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32), th


def test_rope_half_matches_complex_multiplication():
    rng = np.random.default_rng(40)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    cs, _ = _angles(rng, (64, 32))
    out = oracle.rope_half(x, cs)
    z = (x[:, :32].astype(np.float64) + 1j * x[:, 32:64].astype(np.float64)) * \
        (cs[..., 0].astype(np.float64) + 1j * cs[..., 1].astype(np.float64))
    a = np.abs(x[:, :32] * cs[..., 0]).astype(np.float64)
    b = np.abs(x[:, 32:64] * cs[..., 1]).astype(np.float64)
    c = np.abs(x[:, :32] * cs[..., 1]).astype(np.float64)
    d = np.abs(x[:, 32:64] * cs[..., 0]).astype(np.float64)
    # two products and one sum, each rounded to fp32
    assert np.all(np.abs(out[:, :32] - z.real) <= (a + b) * 2.0 ** -23 + 1e-30)
    assert np.all(np.abs(out[:, 32:64] - z.imag) <= (c + d) * 2.0 ** -23 + 1e-30)
    assert np.array_equal(out[:, 64:], x[:, 64:])      # the non-rotary part is untouched


def test_rope_half_special_angles_are_exact():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    one = np.tile(np.array([1.0, 0.0], np.float32), (16, 1))
    assert np.array_equal(oracle.rope_half(x, one), x)
    quarter = np.tile(np.array([0.0, 1.0], np.float32), (16, 1))   # multiply by i
    out = oracle.rope_half(x, quarter)
    assert np.array_equal(out[:, :16], -x[:, 16:32])
    assert np.array_equal(out[:, 16:32], x[:, :16])
    assert np.array_equal(out[:, 32:], x[:, 32:])
    half = np.tile(np.array([-1.0, 0.0], np.float32), (16, 1))     # multiply by -1
    assert np.array_equal(oracle.rope_half(x, half)[:, :32], -x[:, :32])


def test_rope_half_preserves_pair_norms_and_composes():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((32, 128)).astype(np.float32)
    cs1, t1 = _angles(rng, (32, 32))
    cs2, t2 = _angles(rng, (32, 32))
    y = oracle.rope_half(x, cs1)
    n0 = x[:, :32].astype(np.float64) ** 2 + x[:, 32:64].astype(np.float64) ** 2
    n1 = y[:, :32].astype(np.float64) ** 2 + y[:, 32:64].astype(np.float64) ** 2
    assert np.allclose(n1, n0, rtol=1e-5, atol=1e-6)
    both = oracle.rope_half(y, cs2)
    th = t1 + t2
    cs12 = np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32)
    once = oracle.rope_half(x, cs12)
    assert np.allclose(both, once, rtol=0, atol=2e-5)


def test_scale_ue8m0_is_the_smallest_power_of_two_not_below():
    rng = np.random.default_rng(43)
    s = (2.0 ** rng.uniform(-30, 10, 4000)).astype(np.float32)
    for v in s:
        r = oracle.scale_ue8m0(float(v))
        m, _ = np.frexp(np.float64(r))
        assert m == 0.5 and r >= v and r / 2 < v
    for k in (-22, -3, 0, 5):
        assert oracle.scale_ue8m0(2.0 ** k) == np.float32(2.0 ** k)


def test_act_quant_ue8m0_matches_torch_cast_of_exact_quotients():
    rng = np.random.default_rng(44)
    x = (rng.standard_normal((128, 128)) * np.exp2(rng.integers(-8, 8, (128, 1)))).astype(np.float32)
    y, s = oracle.act_quant_fmt(x, 128, 1)
    amax = np.abs(x).max(axis=1)
    s_fp32 = (np.maximum(amax, np.float32(1e-4)) / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(s[:, 0], np.array([oracle.scale_ue8m0(float(v)) for v in s_fp32], np.float32))
    q = x / s                                  # exact: s is a power of two
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(y, ref)
    assert np.all(np.abs(q) <= 448.0)
    # fp32 format: the same library cast of the correctly rounded quotient
    y0, s0 = oracle.act_quant_fmt(x, 128, 0)
    y1, s1 = oracle.act_quant(x, 128)
    assert np.array_equal(y0, y1) and np.array_equal(s0, s1)


def _half_ulp_e4m3(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3) / 2


def test_prologue_composition_tracks_fp64_pipeline():
    """dec(codes) * scale against RoPE (numpy complex) -> Hadamard (scipy) in fp64."""
    rng = np.random.default_rng(45)
    B, S, H, D, R = 2, 3, 4, 128, 64
    q = rng.standard_normal((B, S, H, D)).astype(np.float32)
    k = rng.standard_normal((B, S, D)).astype(np.float32)
    cs, _ = _angles(rng, (S, R // 2))
    Hd = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)

    def ref(v, csr):
        v = v.astype(np.float64).copy()
        z = (v[:R // 2] + 1j * v[R // 2:R]) * (csr[:, 0].astype(np.float64) + 1j * csr[:, 1])
        v[:R // 2], v[R // 2:R] = z.real, z.imag
        return Hd @ v

    for fmt in (0, 1):
        qf, qs, kf, ks = oracle.indexer_prologue(q, k, cs, fmt)
        for b in range(B):
            for s in range(S):
                for h in range(H + 1):
                    codes, sc = (qf[b, s, h], qs[b, s, h]) if h < H else (kf[b, s], ks[b, s])
                    r = ref(q[b, s, h] if h < H else k[b, s], cs[s])
                    dec = oracle.e4m3_decode(codes) * np.float64(sc)
                    # e4m3 rounding of r / scale, plus the fp32 arithmetic before it
                    bound = _half_ulp_e4m3(r / sc) * sc + 1e-5 * np.abs(r).max()
                    assert np.all(np.abs(dec - r) <= bound)


def test_prologue_without_rope_is_indexer_quant():
    rng = np.random.default_rng(46)
    q = rng.standard_normal((1, 2, 3, 64)).astype(np.float32)
    k = rng.standard_normal((1, 2, 64)).astype(np.float32)
    qf, qs, kf, ks = oracle.indexer_prologue(q, k, None, 0)
    rq, rqs = oracle.indexer_quant(q)
    rk, rks = oracle.indexer_quant(k)
    assert np.array_equal(qf, rq) and np.array_equal(qs, rqs)
    assert np.array_equal(kf, rk) and np.array_equal(ks, rks)
