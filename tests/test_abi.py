"""The C ABI loads and exports what include/dsa.h declares; host-side argument
checks reject bad calls before anything is launched (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def dsa():
    import __graft_entry__
    __graft_entry__._builder().build()
    import top_kv_selection_b200 as m
    return m


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_entry_points():
    names = header_functions()
    for n in ("dsa_indexer_quant", "dsa_index_scores", "dsa_topk_select",
              "dsa_sparse_mla_attn", "dsa_decode_step", "dsa_decode_step_noalloc",
              "dsa_indexer_prologue", "dsa_latent_quant", "dsa_sparse_mla_attn_fp8"):
        assert n in names


def test_library_exports_every_declared_symbol(dsa):
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dsa_\w+)", out))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    assert set(header_functions()) == set(dsa.EXPORTED)


def test_status_strings_and_version(dsa):
    assert dsa.version() >= 100
    for code in range(7):
        assert dsa.status_string(code) and dsa.status_string(code) != "unknown status"
    assert dsa.status_string(99) == "unknown status"


NULL = None
FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced: checks fail first
ODD = ctypes.c_void_p((1 << 20) + 4)   # misaligned


def test_indexer_quant_argument_checks(dsa):
    L = dsa._lib
    assert L.dsa_indexer_quant(FAKE, 0, 1, 8, 96, FAKE, 0, FAKE, 0, NULL) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_indexer_quant(FAKE, 7, 1, 8, 128, FAKE, 0, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_indexer_quant(NULL, 0, 1, 8, 128, FAKE, 0, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_indexer_quant(ODD, 0, 1, 8, 128, FAKE, 0, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_indexer_quant(FAKE, 0, -1, 8, 128, FAKE, 0, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    # cache append with a row stride shorter than a row
    assert L.dsa_indexer_quant(FAKE, 0, 2, 8, 128, FAKE, 512, FAKE, 8, NULL) == dsa.DSA_ERR_INVALID_ARG
    # empty problems succeed without a launch (no GPU here)
    assert L.dsa_indexer_quant(NULL, 0, 1, 0, 128, NULL, 0, NULL, 0, NULL) == dsa.DSA_OK


def test_indexer_prologue_argument_checks(dsa):
    L = dsa._lib
    F, U = dsa.DSA_SCALE_F32, dsa.DSA_SCALE_UE8M0

    def call(q=FAKE, k=FAKE, dt=0, B=1, S=2, H=4, d=128, R=64, cs=FAKE, fmt=F, sp=0, t_max=8,
             qf=FAKE, qs=FAKE, kc=FAKE, ks=FAKE):
        return L.dsa_indexer_prologue(q, k, dt, B, S, H, d, R, cs, fmt, sp, t_max, qf, qs, kc, ks,
                                      NULL)

    assert call(d=96) == dsa.DSA_ERR_UNSUPPORTED
    for R in (24, 4, 256):                      # not a power of two / below d/16 / above d
        assert call(R=R) == dsa.DSA_ERR_UNSUPPORTED
    assert call(dt=7) == dsa.DSA_ERR_INVALID_ARG
    assert call(fmt=2) == dsa.DSA_ERR_INVALID_ARG
    assert call(sp=7, S=2, t_max=8) == dsa.DSA_ERR_INVALID_ARG   # rows 7, 8 past the cache
    assert call(cs=NULL) == dsa.DSA_ERR_INVALID_ARG
    assert call(k=NULL) == dsa.DSA_ERR_INVALID_ARG
    assert call(q=ODD) == dsa.DSA_ERR_INVALID_ARG
    assert call(kc=ODD) == dsa.DSA_ERR_INVALID_ARG
    assert call(B=-1) == dsa.DSA_ERR_INVALID_ARG
    # empty problems succeed without a launch (no GPU here)
    assert call(B=0, q=NULL, k=NULL, cs=NULL, fmt=U) == dsa.DSA_OK
    assert call(S=0) == dsa.DSA_OK


def test_latent_fp8_argument_checks(dsa):
    L = dsa._lib
    assert L.dsa_latent_row_bytes(512, 64) == 656
    assert L.dsa_latent_quant(FAKE, 1, 1, 8, 500, 64, FAKE, 0, NULL) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_latent_quant(FAKE, 1, 1, 8, 512, 72, FAKE, 0, NULL) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_latent_quant(FAKE, 9, 1, 8, 512, 64, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_latent_quant(NULL, 1, 1, 8, 512, 64, FAKE, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    # cache append with a row stride shorter than the rows it must hold
    assert L.dsa_latent_quant(FAKE, 1, 2, 8, 512, 64, FAKE, 656, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_latent_quant(NULL, 1, 1, 0, 512, 64, NULL, 0, NULL) == dsa.DSA_OK
    assert L.dsa_sparse_mla_attn_fp8_workspace_size(1, 1, 128, 500, 64, 16) == 0
    # V3.2 shapes decode in the gather: a workspace only for split partials
    # (none when one unit covers the row), never for decoded rows
    assert L.dsa_sparse_mla_attn_fp8_workspace_size(1, 1, 128, 512, 64, 16) == 0
    need = L.dsa_sparse_mla_attn_fp8_workspace_size(1, 1, 128, 512, 64, 2048)
    assert need > 0
    # other shapes decode into the workspace first
    assert (L.dsa_sparse_mla_attn_fp8_workspace_size(1, 1, 16, 256, 32, 16) >=
            16 * 288 * 2 + 16 * 4)

    def attn(q=FAKE, kv=FAKE, t_max=3000, idx=FAKE, B=1, S=1, k=2048, sp=99, out=FAKE, ws=FAKE,
             wsb=None):
        return L.dsa_sparse_mla_attn_fp8(q, kv, t_max, idx, B, S, 128, 512, 64, k, sp, 0.04, out,
                                         NULL, ws, need if wsb is None else wsb, NULL)

    assert attn(sp=3000) == dsa.DSA_ERR_INVALID_ARG         # start_pos + S > t_max
    assert attn(q=ODD) == dsa.DSA_ERR_INVALID_ARG
    assert attn(kv=ODD) == dsa.DSA_ERR_INVALID_ARG          # 16-byte rows for the V3.2 shapes
    assert attn(idx=NULL) == dsa.DSA_ERR_INVALID_ARG
    assert attn(k=0) == dsa.DSA_ERR_INVALID_ARG
    assert attn(wsb=need - 1) == dsa.DSA_ERR_WORKSPACE
    assert attn(ws=NULL) == dsa.DSA_ERR_WORKSPACE
    assert attn(B=0) == dsa.DSA_OK


def test_index_scores_argument_checks(dsa):
    L = dsa._lib
    args = lambda **kw: [kw.get("q", FAKE), FAKE, FAKE, kw.get("k", FAKE), FAKE,
                         kw.get("t_max", 64), kw.get("B", 1), kw.get("S", 1), kw.get("H", 64),
                         kw.get("D", 128), kw.get("sp", 63), kw.get("T", 64), 0.1, FAKE, NULL]
    assert L.dsa_index_scores(*args(D=32)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_index_scores(*args(H=300)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_index_scores(*args(T=65)) == dsa.DSA_ERR_INVALID_ARG       # T > t_max
    assert L.dsa_index_scores(*args(sp=64)) == dsa.DSA_ERR_INVALID_ARG      # start_pos + S > T
    assert L.dsa_index_scores(*args(q=NULL)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_index_scores(*args(k=ODD)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_index_scores(*args(B=0)) == dsa.DSA_OK


def test_topk_argument_checks(dsa):
    L = dsa._lib
    assert L.dsa_topk_select(FAKE, 1, 1, 100, 99, 0, FAKE, NULL, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_topk_select(FAKE, 1, 2, 100, 99, 8, FAKE, NULL, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_topk_select(NULL, 1, 1, 100, 99, 8, FAKE, NULL, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_topk_select(NULL, 0, 1, 100, 99, 8, NULL, NULL, 0, NULL) == dsa.DSA_OK
    need = L.dsa_topk_select_workspace_size(8, 1, 131072, 2048)
    if need:
        assert L.dsa_topk_select(FAKE, 8, 1, 131072, 131071, 2048, FAKE, FAKE, need - 1,
                                 NULL) == dsa.DSA_ERR_WORKSPACE


def test_sparse_mla_argument_checks(dsa):
    L = dsa._lib
    base = lambda **kw: [FAKE, FAKE, kw.get("t_max", 4096), FAKE, 1, 1, 128, kw.get("dc", 512),
                         kw.get("dr", 64), 2048, kw.get("sp", 4095), 0.04, kw.get("dt", 1),
                         kw.get("out", FAKE), NULL, FAKE, 1 << 30, NULL]
    assert L.dsa_sparse_mla_attn(*base(dc=500)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_sparse_mla_attn(*base(dc=512, dr=128)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.dsa_sparse_mla_attn(*base(dt=5)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_sparse_mla_attn(*base(sp=4096)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_sparse_mla_attn(*base(out=ODD)) == dsa.DSA_ERR_INVALID_ARG


def test_decode_step_argument_checks(dsa):
    L = dsa._lib
    need = L.dsa_decode_step_workspace_size(8, 64, 128, 131072, 2048, 128, 512, 64, 1)
    assert need >= 8 * 131072 * 4          # the score rows
    def call(**kw):
        return L.dsa_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("t_max", 131072), FAKE,
                                 FAKE, 8, 64, kw.get("D", 128), 128, 512, 64, kw.get("T", 131072),
                                 2048, 0.088, 0.041, 1, FAKE, FAKE, NULL, kw.get("ws", FAKE),
                                 kw.get("ws_bytes", need), NULL)
    assert call(D=96) == dsa.DSA_ERR_UNSUPPORTED
    assert call(T=131073) == dsa.DSA_ERR_INVALID_ARG
    assert call(T=0) == dsa.DSA_ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == dsa.DSA_ERR_WORKSPACE
    assert call(ws=NULL) == dsa.DSA_ERR_WORKSPACE


def test_wait_selftest_argument_checks(dsa):
    L = dsa._lib
    # a budget outside 1 .. 2e9 cycles is refused before anything is launched
    assert L.dsa_wait_selftest(0, 0, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_wait_selftest(-5, 1, NULL) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_wait_selftest(2_000_000_001, 0, NULL) == dsa.DSA_ERR_INVALID_ARG


def test_csa_argument_checks(dsa):
    L = dsa._lib
    def scores(**kw):
        return L.dsa_index_scores_csa(FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("t_max", 1000), 1,
                                      kw.get("S", 1), 64, 128, kw.get("sp", 3999),
                                      kw.get("T", 1000), kw.get("m", 4), 0.088, FAKE, NULL)
    assert scores(m=0) == dsa.DSA_ERR_INVALID_ARG
    assert scores(sp=4003) == dsa.DSA_ERR_INVALID_ARG           # entry 1000 would be visible
    assert scores(T=1001) == dsa.DSA_ERR_INVALID_ARG            # more entries than the cache holds
    def topk(**kw):
        return L.dsa_topk_select_csa(FAKE, 1, 1, kw.get("T", 1000), kw.get("sp", 3999),
                                     kw.get("m", 4), 2048, FAKE, NULL, 0, NULL)
    assert topk(m=0) == dsa.DSA_ERR_INVALID_ARG
    assert topk(sp=4003) == dsa.DSA_ERR_INVALID_ARG
