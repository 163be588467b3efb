"""CPU oracle for the DeepSeek Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check and
by the benchmark's CPU-baseline leg, never by the product path.  The arithmetic
lives in plain C (``dsa_oracle.c``), single-threaded, compiled with gcc without
fast-math and without floating-point contraction.  This module only compiles
that file, marshals numpy arrays, and chains the steps in the order the pages'
Indexer.forward and MLA excerpts run them.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms, library routines (torch's e4m3 cast, numpy sorts and einsums),
invariants and brute force on tiny inputs.  Two values are readings, not pinned
facts: the indexer softmax scale and the attention scale (both arguments).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-frounding-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [f32]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode_array.argtypes = [P, i64, P]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_hadamard_scale.argtypes = [i32]
    lib.oracle_hadamard_scale.restype = f32
    lib.oracle_fwht_f32.argtypes = [P, i32]
    lib.oracle_fwht_f32.restype = None
    lib.oracle_act_quant.argtypes = [P, i32, i32, P, P]
    lib.oracle_act_quant.restype = None
    lib.oracle_indexer_quant.argtypes = [P, i64, i32, P, P]
    lib.oracle_indexer_quant.restype = None
    lib.oracle_rope_half.argtypes = [P, i32, P]
    lib.oracle_rope_half.restype = None
    lib.oracle_scale_ue8m0.argtypes = [f32]
    lib.oracle_scale_ue8m0.restype = f32
    lib.oracle_act_quant_fmt.argtypes = [P, i32, i32, i32, P, P]
    lib.oracle_act_quant_fmt.restype = None
    lib.oracle_indexer_prologue.argtypes = [P, P, i32, i32, i32, i32, i32, P, i32, P, P, P, P]
    lib.oracle_indexer_prologue.restype = None
    lib.oracle_latent_row_bytes.argtypes = [i32, i32]
    lib.oracle_latent_row_bytes.restype = i64
    lib.oracle_latent_quant.argtypes = [P, i32, i32, P]
    lib.oracle_latent_quant.restype = None
    lib.oracle_latent_dequant.argtypes = [P, i32, i32, P]
    lib.oracle_latent_dequant.restype = None
    lib.oracle_weight_fold.argtypes = [f32, i32, f32, f32]
    lib.oracle_weight_fold.restype = f32
    lib.oracle_index_scores.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i32, i64, i64,
                                        f32, P]
    lib.oracle_index_scores.restype = None
    lib.oracle_topk_select.argtypes = [P, i32, i32, i64, i64, i32, P]
    lib.oracle_topk_select.restype = None
    lib.oracle_csa_available.argtypes = [i64, i32]
    lib.oracle_csa_available.restype = i64
    lib.oracle_index_scores_csa.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i32, i64, i64,
                                            i32, f32, P]
    lib.oracle_index_scores_csa.restype = None
    lib.oracle_topk_select_csa.argtypes = [P, i32, i32, i64, i64, i32, i32, P]
    lib.oracle_topk_select_csa.restype = None
    lib.oracle_sparse_mla.argtypes = [P, P, i64, P, i32, i32, i32, i32, i32, i32, i64, f32,
                                      P, P]
    lib.oracle_sparse_mla.restype = None
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- #
# Scalar / per-vector primitives
# --------------------------------------------------------------------------- #
def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3fn code (closed form), as float64."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def e4m3_encode(x) -> np.ndarray:
    """Round fp32 values to e4m3fn codes: nearest-even, saturating at +-448."""
    lib = _load()
    x = _c(x, np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib.oracle_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def hadamard_scale(D: int) -> np.float32:
    return np.float32(_load().oracle_hadamard_scale(D))


def fwht(x: np.ndarray) -> np.ndarray:
    """rotate_activation of each trailing D-vector (fp32 in, fp32 out)."""
    lib = _load()
    x = _c(x, np.float32).copy()
    D = x.shape[-1]
    flat = x.reshape(-1, D)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib.oracle_fwht_f32(_p(row), D)
        flat[r] = row
    return flat.reshape(x.shape)


def act_quant(x: np.ndarray, block: int):
    """Blockwise e4m3 quantisation of the trailing dim: returns (codes, scales)."""
    lib = _load()
    x = _c(x, np.float32)
    n = x.shape[-1]
    flat = x.reshape(-1, n)
    y = np.empty(flat.shape, dtype=np.uint8)
    s = np.empty((flat.shape[0], n // block), dtype=np.float32)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        yr = np.empty(n, dtype=np.uint8)
        sr = np.empty(n // block, dtype=np.float32)
        lib.oracle_act_quant(_p(row), n, block, _p(yr), _p(sr))
        y[r], s[r] = yr, sr
    return y.reshape(x.shape), s.reshape(x.shape[:-1] + (n // block,))


def indexer_quant(x: np.ndarray):
    """rotate_activation + act_quant (block = D) of each trailing D-vector.

    Returns (codes uint8 [..., D], scale fp32 [...]).
    """
    lib = _load()
    x = _c(x, np.float32)
    D = x.shape[-1]
    n_vec = x.size // D
    out = np.empty(x.shape, dtype=np.uint8)
    sc = np.empty(x.shape[:-1], dtype=np.float32)
    lib.oracle_indexer_quant(_p(x), n_vec, D, _p(out), _p(sc))
    return out, sc


def rope_half(x: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """Non-interleaved rotary embedding of the first R = 2 * cs.shape[-2] elements
    of each trailing vector of x, with the angles cs [..., R/2, 2] (cos, sin)
    broadcast over the leading dims of x except the last."""
    lib = _load()
    x = _c(x, np.float32).copy()
    R = 2 * cs.shape[-2]
    D = x.shape[-1]
    flat = x.reshape(-1, D)
    csb = np.broadcast_to(_c(cs, np.float32), x.shape[:-1] + (R // 2, 2)).reshape(-1, R // 2, 2)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        c = np.ascontiguousarray(csb[r])
        lib.oracle_rope_half(_p(row), R, _p(c))
        flat[r] = row
    return flat.reshape(x.shape)


def scale_ue8m0(s: float) -> np.float32:
    return np.float32(_load().oracle_scale_ue8m0(s))


def act_quant_fmt(x: np.ndarray, block: int, fmt: int):
    """act_quant with scale format fmt (0 fp32, 1 ue8m0): returns (codes, scales)."""
    lib = _load()
    x = _c(x, np.float32)
    n = x.shape[-1]
    flat = x.reshape(-1, n)
    y = np.empty(flat.shape, dtype=np.uint8)
    s = np.empty((flat.shape[0], n // block), dtype=np.float32)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        yr = np.empty(n, dtype=np.uint8)
        sr = np.empty(n // block, dtype=np.float32)
        lib.oracle_act_quant_fmt(_p(row), n, block, fmt, _p(yr), _p(sr))
        y[r], s[r] = yr, sr
    return y.reshape(x.shape), s.reshape(x.shape[:-1] + (n // block,))


def indexer_prologue(q: np.ndarray, k: np.ndarray, cs: np.ndarray, fmt: int = 0):
    """RoPE (first R dims, not interleaved) + rotate_activation + act_quant of the
    indexer's queries q [B,S,H,D] and keys k [B,S,D]; cs [S, R/2, 2] (cos, sin),
    R = 0 when cs has no columns.  Returns (q_fp8, q_scale, k_fp8, k_scale)."""
    lib = _load()
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    B, S, H, D = q.shape
    cs = _c(cs, np.float32).reshape(S, -1, 2) if cs is not None else np.zeros((S, 0, 2), np.float32)
    R = 2 * cs.shape[1]
    qf = np.empty(q.shape, dtype=np.uint8)
    qs = np.empty((B, S, H), dtype=np.float32)
    kf = np.empty(k.shape, dtype=np.uint8)
    ks = np.empty((B, S), dtype=np.float32)
    cs_buf = np.ascontiguousarray(cs if R else np.zeros((S, 1, 2), np.float32))
    lib.oracle_indexer_prologue(_p(q), _p(k), B, S, H, D, R, _p(cs_buf), fmt, _p(qf), _p(qs),
                                _p(kf), _p(ks))
    return qf, qs, kf, ks


def latent_row_bytes(dc: int, dr: int) -> int:
    return int(_load().oracle_latent_row_bytes(dc, dr))


def latent_quant(kv: np.ndarray, dc: int) -> np.ndarray:
    """FP8 latent rows: kv [..., dc + dr] -> uint8 [..., latent_row_bytes(dc, dr)]."""
    lib = _load()
    kv = _c(kv, np.float32)
    dr = kv.shape[-1] - dc
    nbytes = latent_row_bytes(dc, dr)
    flat = kv.reshape(-1, dc + dr)
    out = np.empty((flat.shape[0], nbytes), dtype=np.uint8)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        o = np.empty(nbytes, dtype=np.uint8)
        lib.oracle_latent_quant(_p(row), dc, dr, _p(o))
        out[r] = o
    return out.reshape(kv.shape[:-1] + (nbytes,))


def latent_dequant(rows: np.ndarray, dc: int, dr: int) -> np.ndarray:
    """Decoded FP8 latent rows: uint8 [..., bytes] -> fp32 [..., dc + dr]."""
    lib = _load()
    rows = _c(rows, np.uint8)
    flat = rows.reshape(-1, rows.shape[-1])
    out = np.empty((flat.shape[0], dc + dr), dtype=np.float32)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        o = np.empty(dc + dr, dtype=np.float32)
        lib.oracle_latent_dequant(_p(row), dc, dr, _p(o))
        out[r] = o
    return out.reshape(rows.shape[:-1] + (dc + dr,))


def sparse_mla_fp8(q, kv_rows, idx, start_pos: int, sm_scale: float, dc: int, dr: int):
    """Sparse attention over an FP8 latent cache.  The attention computes in bf16
    (bf16 operands, fp32-or-wider softmax and accumulation), so each decoded row
    enters it as a bf16 operand: decode, round to bf16 (nearest even), then the
    same fp64 attention as sparse_mla."""
    dec = latent_dequant(kv_rows, dc, dr)
    b = dec.view(np.uint32).astype(np.uint64)
    rounded = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16    # bf16, nearest even (finite values)
    dec_bf16 = rounded.astype(np.uint32).view(np.float32)
    return sparse_mla(q, dec_bf16, idx, start_pos, sm_scale, dc)


def weight_fold(w: float, H: int, q_scale: float, softmax_scale: float) -> np.float32:
    return np.float32(_load().oracle_weight_fold(w, H, q_scale, softmax_scale))


# --------------------------------------------------------------------------- #
# Hot-path steps
# --------------------------------------------------------------------------- #
def index_scores(q_fp8, q_scale, w, k_cache, k_scale, start_pos: int, T: int,
                 softmax_scale: float) -> np.ndarray:
    """fp8_index + causal mask.  q_fp8 [B,S,H,D], k_cache [B,t_max,D] -> [B,S,T]."""
    lib = _load()
    q_fp8 = _c(q_fp8, np.uint8)
    B, S, H, D = q_fp8.shape
    k_cache = _c(k_cache, np.uint8)
    t_max = k_cache.shape[1]
    q_scale = _c(q_scale, np.float32)
    w = _c(w, np.float32)
    k_scale = _c(k_scale, np.float32)
    assert q_scale.shape == (B, S, H) and w.shape == (B, S, H)
    assert k_cache.shape == (B, t_max, D) and k_scale.shape == (B, t_max) and T <= t_max
    out = np.empty((B, S, T), dtype=np.float32)
    lib.oracle_index_scores(_p(q_fp8), _p(q_scale), _p(w), _p(k_cache), _p(k_scale), t_max,
                            B, S, H, D, start_pos, T, softmax_scale, _p(out))
    return out


def topk_select(scores, start_pos: int, k: int) -> np.ndarray:
    """scores [B,S,T] -> idx [B,S,min(k,T)] int32, ascending, -1 padded."""
    lib = _load()
    scores = _c(scores, np.float32)
    B, S, T = scores.shape
    K = min(k, T)
    idx = np.empty((B, S, K), dtype=np.int32)
    lib.oracle_topk_select(_p(scores), B, S, T, start_pos, k, _p(idx))
    return idx


def csa_available(i: int, m: int) -> int:
    """Compressed entries (m tokens each) available to the query at position i."""
    return int(_load().oracle_csa_available(i, m))


def index_scores_csa(q_fp8, q_scale, w, k_cache, k_scale, start_pos: int, T: int, m: int,
                     softmax_scale: float) -> np.ndarray:
    """fp8_index over compressed entries with the CSA availability mask.
    q_fp8 [B,S,H,D], k_cache [B,t_max,D] (entry keys) -> [B,S,T] over entries."""
    lib = _load()
    q_fp8 = _c(q_fp8, np.uint8)
    B, S, H, D = q_fp8.shape
    k_cache = _c(k_cache, np.uint8)
    t_max = k_cache.shape[1]
    q_scale = _c(q_scale, np.float32)
    w = _c(w, np.float32)
    k_scale = _c(k_scale, np.float32)
    assert q_scale.shape == (B, S, H) and w.shape == (B, S, H)
    assert k_cache.shape == (B, t_max, D) and k_scale.shape == (B, t_max) and T <= t_max
    out = np.empty((B, S, T), dtype=np.float32)
    lib.oracle_index_scores_csa(_p(q_fp8), _p(q_scale), _p(w), _p(k_cache), _p(k_scale), t_max,
                                B, S, H, D, start_pos, T, m, softmax_scale, _p(out))
    return out


def topk_select_csa(scores, start_pos: int, m: int, k: int) -> np.ndarray:
    """scores [B,S,T] over entries -> idx [B,S,min(k,T)] int32 entry ids, ascending, -1 padded."""
    lib = _load()
    scores = _c(scores, np.float32)
    B, S, T = scores.shape
    K = min(k, T)
    idx = np.empty((B, S, K), dtype=np.int32)
    lib.oracle_topk_select_csa(_p(scores), B, S, T, start_pos, m, k, _p(idx))
    return idx


def sparse_mla(q, kv, idx, start_pos: int, sm_scale: float, dc: int):
    """q [B,S,Hq,dc+dr], kv [B,t_max,dc+dr], idx [B,S,k] -> (out [B,S,Hq,dc], lse [B,S,Hq])."""
    lib = _load()
    q = _c(q, np.float32)
    kv = _c(kv, np.float32)
    idx = _c(idx, np.int32)
    B, S, Hq, dqk = q.shape
    dr = dqk - dc
    t_max = kv.shape[1]
    k = idx.shape[2]
    assert kv.shape == (B, t_max, dqk) and idx.shape[:2] == (B, S)
    out = np.empty((B, S, Hq, dc), dtype=np.float32)
    lse = np.empty((B, S, Hq), dtype=np.float32)
    lib.oracle_sparse_mla(_p(q), _p(kv), t_max, _p(idx), B, S, Hq, dc, dr, k, start_pos,
                          sm_scale, _p(out), _p(lse))
    return out, lse


# --------------------------------------------------------------------------- #
# Whole passes, in the order of Indexer.forward and the MLA excerpt
# --------------------------------------------------------------------------- #
def decode_step(q_idx, w, keys, q_mla, kv, topk: int, softmax_scale_idx: float,
                sm_scale: float, dc: int) -> dict:
    """One decode step for ONE sequence with T = len(keys) visible tokens.

    keys [T, D] are the raw keys of every position (position T-1 is the new
    token's); each is rotated and quantised into the cache, as the cache write
    of Indexer.forward does position by position.
    """
    T, D = keys.shape
    H = q_idx.shape[0]
    k_fp8, k_sc = indexer_quant(keys)                       # [T,D], [T]
    q_fp8, q_sc = indexer_quant(q_idx)                      # [H,D], [H]
    sc = index_scores(q_fp8[None, None], q_sc[None, None], np.asarray(w)[None, None],
                      k_fp8[None], k_sc[None], start_pos=T - 1, T=T,
                      softmax_scale=softmax_scale_idx)      # [1,1,T]
    idx = topk_select(sc, start_pos=T - 1, k=topk)          # [1,1,K]
    out, lse = sparse_mla(np.asarray(q_mla, dtype=np.float32)[None, None],
                          np.asarray(kv, dtype=np.float32)[None], idx, start_pos=T - 1,
                          sm_scale=sm_scale, dc=dc)
    return dict(k_fp8=k_fp8, k_scale=k_sc, q_fp8=q_fp8, q_scale=q_sc, scores=sc[0, 0],
                idx=idx[0, 0], out=out[0, 0], lse=lse[0, 0])


def prefill_rows(q_idx, w, keys, q_mla, kv, rows, topk: int, softmax_scale_idx: float,
                 sm_scale: float, dc: int) -> dict:
    """Prefill (start_pos = 0, S = T) of ONE sequence, evaluated at query rows ``rows``.

    q_idx [T,H,D], w [T,H], keys [T,D], q_mla [T,Hq,dc+dr], kv [T,dc+dr].
    Each row is computed exactly as the full pass would compute it.
    """
    T, D = keys.shape
    rows = np.asarray(rows, dtype=np.int64)
    k_fp8, k_sc = indexer_quant(keys)
    q_fp8, q_sc = indexer_quant(np.asarray(q_idx)[rows])    # [R,H,D]
    w = np.asarray(w)[rows]
    scores = np.empty((len(rows), T), dtype=np.float32)
    idx = np.empty((len(rows), min(topk, T)), dtype=np.int32)
    outs, lses = [], []
    qm = np.asarray(q_mla, dtype=np.float32)
    kvf = np.asarray(kv, dtype=np.float32)[None]
    for r, s in enumerate(rows.tolist()):
        # query s of a prefill sees positions 0..s: same as start_pos = s, S = 1
        sc = index_scores(q_fp8[r][None, None], q_sc[r][None, None], w[r][None, None],
                          k_fp8[None], k_sc[None], start_pos=s, T=T,
                          softmax_scale=softmax_scale_idx)
        scores[r] = sc[0, 0]
        ix = topk_select(sc, start_pos=s, k=topk)
        idx[r] = ix[0, 0]
        o, l = sparse_mla(qm[s][None, None], kvf, ix, start_pos=s, sm_scale=sm_scale, dc=dc)
        outs.append(o[0, 0])
        lses.append(l[0, 0])
    return dict(k_fp8=k_fp8, k_scale=k_sc, q_fp8=q_fp8, q_scale=q_sc, scores=scores,
                idx=idx, out=np.stack(outs), lse=np.stack(lses))
