"""Python binding of libdsa, the B200 (sm_100a) DeepSeek Sparse Attention hot path.

Each function here has the name of the C entry point it calls (include/dsa.h)
and only marshals arguments: torch tensors become device pointers, shapes
become the integer arguments, the current torch stream becomes the stream
argument.  Every computation runs in libdsa's CUDA kernels; there is no CPU or
PyTorch fallback.  Importing the package fails if libdsa.so has not been built
(``python top_kv_selection_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libdsa.so is not built at {LIB_PATH}; run "
                      "`python top_kv_selection_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA = 0, 1, 2, 3
DSA_ERR_TIMEOUT, DSA_ERR_DEVICE, DSA_ERR_WORKSPACE = 4, 5, 6
DSA_F32, DSA_BF16, DSA_FP8_LATENT = 0, 1, 2
DSA_SCALE_F32, DSA_SCALE_UE8M0 = 0, 1
DSA_NOALLOC_SCRATCH_BYTES = 32 << 20

_P, _i32, _i64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)

_SIGNATURES = {
    "dsa_status_string": ([_i32], ctypes.c_char_p),
    "dsa_version": ([], _i32),
    "dsa_get_device_error": ([_P, _P], _i32),
    "dsa_wait_selftest": ([_i64, _i32, _P], _i32),
    "dsa_indexer_quant": ([_P, _i32, _i64, _i64, _i32, _P, _i64, _P, _i64, _P], _i32),
    "dsa_indexer_prologue": ([_P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _P, _i32, _i64, _i64,
                              _P, _P, _P, _P, _P], _i32),
    "dsa_latent_row_bytes": ([_i32, _i32], _i64),
    "dsa_latent_quant": ([_P, _i32, _i64, _i64, _i32, _i32, _P, _i64, _P], _i32),
    "dsa_sparse_mla_attn_fp8_workspace_size": ([_i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "dsa_sparse_mla_attn_fp8": ([_P, _P, _i64, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i64,
                                 _f32, _P, _P, _P, _sz, _P], _i32),
    "dsa_index_scores": ([_P, _P, _P, _P, _P, _i64, _i32, _i32, _i32, _i32, _i64, _i64, _f32,
                          _P, _P], _i32),
    "dsa_decode_index_scores": ([_P, _P, _P, _P, _P, _i64, _i32, _i32, _i32, _i64, _f32, _P, _P],
                                _i32),
    "dsa_topk_select_workspace_size": ([_i32, _i32, _i64, _i32], _sz),
    "dsa_index_scores_csa": ([_P, _P, _P, _P, _P, _i64, _i32, _i32, _i32, _i32, _i64, _i64, _i32,
                              _f32, _P, _P], _i32),
    "dsa_topk_select_csa": ([_P, _i32, _i32, _i64, _i64, _i32, _i32, _P, _P, _sz, _P], _i32),
    "dsa_topk_select": ([_P, _i32, _i32, _i64, _i64, _i32, _P, _P, _sz, _P], _i32),
    "dsa_sparse_mla_attn_workspace_size": ([_i32, _i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "dsa_sparse_mla_attn": ([_P, _P, _i64, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i64, _f32,
                             _i32, _P, _P, _P, _sz, _P], _i32),
    "dsa_decode_step_workspace_size": ([_i32, _i32, _i32, _i64, _i32, _i32, _i32, _i32, _i32],
                                       _sz),
    "dsa_decode_step": ([_P, _P, _P, _P, _P, _i64, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32,
                         _i64, _i32, _f32, _f32, _i32, _P, _P, _P, _P, _sz, _P], _i32),
    "dsa_decode_step_noalloc": ([_P, _P, _P, _P, _P, _i64, _P, _P, _i32, _i32, _i32, _i32, _i32,
                                 _i32, _i64, _i32, _f32, _f32, _i32, _P, _P, _P, _P], _i32),
}

for _name, (_args, _res) in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGNATURES)


class DSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status}: {status_string(status)}")
        self.status = status


def status_string(status: int) -> str:
    return _lib.dsa_status_string(status).decode()


def version() -> int:
    return _lib.dsa_version()


def _check(fn: str, status: int) -> None:
    if status != DSA_OK:
        raise DSAError(fn, status)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdsa takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _kv_dtype(kv_cache: torch.Tensor, q_mla: torch.Tensor) -> int:
    """The decode step's cache type: uint8 rows are the FP8 latent cache."""
    return DSA_FP8_LATENT if kv_cache.dtype == torch.uint8 else _dtype(q_mla)


def dsa_get_device_error(stream=None) -> int:
    """Wait for the stream, return and clear the sticky device error code."""
    code = ctypes.c_int32(0)
    _check("dsa_get_device_error", _lib.dsa_get_device_error(_stream(stream), ctypes.byref(code)))
    return code.value


def dsa_wait_selftest(budget_cycles: int, complete: bool = False, stream=None) -> None:
    """Run one bounded device wait of budget_cycles SM cycles: with complete=False
    nobody arrives, so it expires and records DSA_ERR_TIMEOUT (read it with
    dsa_get_device_error); with complete=True it succeeds at once."""
    _check("dsa_wait_selftest", _lib.dsa_wait_selftest(int(budget_cycles), 1 if complete else 0,
                                                       _stream(stream)))


def dsa_indexer_quant(x: torch.Tensor, out_fp8: torch.Tensor, out_scale: torch.Tensor,
                      n_rows: int = 1, out_row_stride: int = 0, scale_row_stride: int = 0,
                      stream=None) -> None:
    """rotate_activation + act_quant of the d-vectors of x ([n_rows, n_vec, d] as laid out).

    For a cache append pass views that start at the cache row and the cache
    strides (see include/dsa.h); otherwise out_fp8 / out_scale are contiguous.
    """
    d = x.shape[-1]
    n_vec = x.numel() // d // n_rows
    _check("dsa_indexer_quant", _lib.dsa_indexer_quant(
        _ptr(x), _dtype(x), n_rows, n_vec, d, ctypes.c_void_p(out_fp8.data_ptr()),
        out_row_stride, ctypes.c_void_p(out_scale.data_ptr()), scale_row_stride,
        _stream(stream)))


def dsa_indexer_prologue(q: torch.Tensor | None, k: torch.Tensor, rope_cs: torch.Tensor | None,
                         start_pos: int, q_fp8: torch.Tensor | None, q_scale: torch.Tensor | None,
                         k_cache: torch.Tensor, k_scale: torch.Tensor,
                         scale_fmt: int = DSA_SCALE_F32, stream=None) -> None:
    """RoPE (first rope_dim elements, not interleaved) + rotate_activation + act_quant of
    q [B,S,H,d] and k [B,S,d]; keys appended to k_cache [B,t_max,d] / k_scale [B,t_max]
    at start_pos.  rope_cs [S, rope_dim/2, 2] fp32 (cos, sin), or None for no rotary part."""
    B, S, d = k.shape
    H = q.shape[2] if q is not None else 0
    rope_dim = 2 * rope_cs.shape[1] if rope_cs is not None else 0
    t_max = k_cache.shape[1]
    _check("dsa_indexer_prologue", _lib.dsa_indexer_prologue(
        _ptr(q), _ptr(k), _dtype(k), B, S, H, d, rope_dim, _ptr(rope_cs), scale_fmt, start_pos,
        t_max, _ptr(q_fp8), _ptr(q_scale), _ptr(k_cache), _ptr(k_scale), _stream(stream)))


def dsa_latent_row_bytes(dc: int, dr: int) -> int:
    return int(_lib.dsa_latent_row_bytes(dc, dr))


def dsa_latent_quant(kv: torch.Tensor, out: torch.Tensor, dc: int, n_rows: int = 1,
                     out_row_stride: int = 0, stream=None) -> None:
    """FP8 latent rows of kv ([n_rows, n_vec, dc + dr] as laid out) into out (uint8 rows of
    dsa_latent_row_bytes bytes; a cache append passes a view at the cache row and the cache
    row stride in bytes)."""
    dqk = kv.shape[-1]
    n_vec = kv.numel() // dqk // n_rows
    _check("dsa_latent_quant", _lib.dsa_latent_quant(
        _ptr(kv), _dtype(kv), n_rows, n_vec, dc, dqk - dc, ctypes.c_void_p(out.data_ptr()),
        out_row_stride, _stream(stream)))


def dsa_sparse_mla_attn_fp8_workspace_size(B: int, S: int, Hq: int, dc: int, dr: int,
                                           k: int) -> int:
    return int(_lib.dsa_sparse_mla_attn_fp8_workspace_size(B, S, Hq, dc, dr, k))


def dsa_sparse_mla_attn_fp8(q: torch.Tensor, kv_fp8: torch.Tensor, idx: torch.Tensor,
                            start_pos: int, sm_scale: float, dc: int, out: torch.Tensor,
                            lse: torch.Tensor | None, workspace: torch.Tensor,
                            stream=None) -> None:
    """q [B,S,Hq,dc+dr] bf16, kv_fp8 [B,t_max,row_bytes] uint8, idx [B,S,k] int32 ->
    out [B,S,Hq,dc] bf16, lse [B,S,Hq] fp32."""
    B, S, Hq, dqk = q.shape
    t_max = kv_fp8.shape[1]
    k = idx.shape[-1]
    _check("dsa_sparse_mla_attn_fp8", _lib.dsa_sparse_mla_attn_fp8(
        _ptr(q), _ptr(kv_fp8), t_max, _ptr(idx), B, S, Hq, dc, dqk - dc, k, start_pos,
        sm_scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def dsa_index_scores(q_fp8: torch.Tensor, q_scale: torch.Tensor, w: torch.Tensor,
                     k_cache: torch.Tensor, k_scale: torch.Tensor, start_pos: int, T: int,
                     softmax_scale: float, scores: torch.Tensor, stream=None) -> None:
    """q_fp8 [B,S,H,D] uint8, k_cache [B,t_max,D] uint8 -> scores [B,S,T] fp32."""
    B, S, H, D = q_fp8.shape
    t_max = k_cache.shape[1]
    _check("dsa_index_scores", _lib.dsa_index_scores(
        _ptr(q_fp8), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale), t_max, B, S, H, D,
        start_pos, T, softmax_scale, _ptr(scores), _stream(stream)))


def dsa_decode_index_scores(q_idx: torch.Tensor, w: torch.Tensor, k_new: torch.Tensor,
                            k_cache: torch.Tensor, k_scale: torch.Tensor, T: int,
                            softmax_scale: float, scores: torch.Tensor, stream=None) -> None:
    """Indexer half of a decode step: q_idx [B,H,D], w [B,H], k_new [B,D] fp32; appends the
    key at T-1 of k_cache [B,t_max,D] / k_scale [B,t_max]; scores [B,T] fp32."""
    B, H, D = q_idx.shape
    t_max = k_cache.shape[1]
    _check("dsa_decode_index_scores", _lib.dsa_decode_index_scores(
        _ptr(q_idx), _ptr(w), _ptr(k_new), _ptr(k_cache), _ptr(k_scale), t_max, B, H, D, T,
        softmax_scale, _ptr(scores), _stream(stream)))


def dsa_topk_select_workspace_size(B: int, S: int, T: int, k: int) -> int:
    return _lib.dsa_topk_select_workspace_size(B, S, T, k)


def dsa_topk_select(scores: torch.Tensor, start_pos: int, k: int, idx: torch.Tensor,
                    workspace: torch.Tensor | None = None, stream=None) -> None:
    """scores [B,S,T] fp32 -> idx [B,S,min(k,T)] int32 (ascending positions, -1 padded)."""
    B, S, T = scores.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("dsa_topk_select", _lib.dsa_topk_select(
        _ptr(scores), B, S, T, start_pos, k, _ptr(idx), _ptr(workspace), ws_bytes,
        _stream(stream)))


def dsa_index_scores_csa(q_fp8: torch.Tensor, q_scale: torch.Tensor, w: torch.Tensor,
                         k_cache: torch.Tensor, k_scale: torch.Tensor, start_pos: int, T: int,
                         compress: int, softmax_scale: float, scores: torch.Tensor,
                         stream=None) -> None:
    """fp8_index over compressed entries (m = compress tokens each): scores [B,S,T] over
    the T entries of k_cache [B,t_max,D], entry e of query s masked unless
    e < (start_pos + s + 1) // m."""
    B, S, H, D = q_fp8.shape
    t_max = k_cache.shape[1]
    _check("dsa_index_scores_csa", _lib.dsa_index_scores_csa(
        _ptr(q_fp8), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale), t_max, B, S, H, D,
        start_pos, T, compress, softmax_scale, _ptr(scores), _stream(stream)))


def dsa_topk_select_csa(scores: torch.Tensor, start_pos: int, compress: int, k: int,
                        idx: torch.Tensor, workspace: torch.Tensor | None = None,
                        stream=None) -> None:
    """scores [B,S,T] over entries -> idx [B,S,min(k,T)] entry ids (ascending, -1 padded)
    among the (start_pos + s + 1) // compress available entries of each row."""
    B, S, T = scores.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("dsa_topk_select_csa", _lib.dsa_topk_select_csa(
        _ptr(scores), B, S, T, start_pos, compress, k, _ptr(idx), _ptr(workspace), ws_bytes,
        _stream(stream)))


def dsa_sparse_mla_attn_workspace_size(B: int, S: int, Hq: int, dc: int, dr: int, k: int,
                                       dt: int) -> int:
    return _lib.dsa_sparse_mla_attn_workspace_size(B, S, Hq, dc, dr, k, dt)


def dsa_sparse_mla_attn(q: torch.Tensor, kv_cache: torch.Tensor, idx: torch.Tensor,
                        start_pos: int, sm_scale: float, out: torch.Tensor,
                        lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        stream=None) -> None:
    """q [B,S,Hq,dc+dr], kv_cache [B,t_max,dc+dr], idx [B,S,k] -> out [B,S,Hq,dc]."""
    B, S, Hq, dqk = q.shape
    dc = out.shape[-1]
    t_max = kv_cache.shape[1]
    k = idx.shape[-1]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("dsa_sparse_mla_attn", _lib.dsa_sparse_mla_attn(
        _ptr(q), _ptr(kv_cache), t_max, _ptr(idx), B, S, Hq, dc, dqk - dc, k, start_pos,
        sm_scale, _dtype(q), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))


def dsa_decode_step_workspace_size(B: int, H: int, D: int, T: int, index_topk: int, Hq: int,
                                   dc: int, dr: int, dt: int) -> int:
    return _lib.dsa_decode_step_workspace_size(B, H, D, T, index_topk, Hq, dc, dr, dt)


def dsa_decode_step(q_idx: torch.Tensor, w: torch.Tensor, k_new: torch.Tensor,
                    k_cache: torch.Tensor, k_scale: torch.Tensor, kv_cache: torch.Tensor,
                    q_mla: torch.Tensor, T: int, index_topk: int, softmax_scale: float,
                    sm_scale: float, idx: torch.Tensor, out: torch.Tensor,
                    lse: torch.Tensor | None, workspace: torch.Tensor, stream=None) -> None:
    """One decode step (see include/dsa.h): q_idx [B,H,D], w [B,H], k_new [B,D] fp32;
    k_cache [B,t_max,D] uint8, k_scale [B,t_max]; kv_cache [B,t_max,dc+dr] (or uint8
    [B,t_max,row_bytes]: the FP8 latent cache, q_mla bf16); q_mla [B,Hq,dc+dr];
    idx [B,K]; out [B,Hq,dc]."""
    B, H, D = q_idx.shape
    Hq, dqk = q_mla.shape[1], q_mla.shape[2]
    dc = out.shape[-1]
    t_max = k_cache.shape[1]
    _check("dsa_decode_step", _lib.dsa_decode_step(
        _ptr(q_idx), _ptr(w), _ptr(k_new), _ptr(k_cache), _ptr(k_scale), t_max, _ptr(kv_cache),
        _ptr(q_mla), B, H, D, Hq, dc, dqk - dc, T, index_topk, softmax_scale, sm_scale,
        _kv_dtype(kv_cache, q_mla), _ptr(idx), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def dsa_decode_step_noalloc(q_idx: torch.Tensor, w: torch.Tensor, k_new: torch.Tensor,
                            k_cache: torch.Tensor, k_scale: torch.Tensor, kv_cache: torch.Tensor,
                            q_mla: torch.Tensor, T: int, index_topk: int, softmax_scale: float,
                            sm_scale: float, idx: torch.Tensor, out: torch.Tensor,
                            lse: torch.Tensor | None, stream=None) -> None:
    """dsa_decode_step without a workspace: for callers that cannot allocate device
    memory, scratch comes from a fixed DSA_NOALLOC_SCRATCH_BYTES array inside libdsa
    (shared by all calls on a device; calls overlapping on the GPU race)."""
    B, H, D = q_idx.shape
    Hq, dqk = q_mla.shape[1], q_mla.shape[2]
    dc = out.shape[-1]
    t_max = k_cache.shape[1]
    _check("dsa_decode_step_noalloc", _lib.dsa_decode_step_noalloc(
        _ptr(q_idx), _ptr(w), _ptr(k_new), _ptr(k_cache), _ptr(k_scale), t_max, _ptr(kv_cache),
        _ptr(q_mla), B, H, D, Hq, dc, dqk - dc, T, index_topk, softmax_scale, sm_scale,
        _kv_dtype(kv_cache, q_mla), _ptr(idx), _ptr(out), _ptr(lse), _stream(stream)))
