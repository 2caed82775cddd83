"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol the header declares, sizes workspaces, and rejects bad arguments on
the host before anything is launched (no compute call is made here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from sparse_attention_pool_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def header_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"sizeof"})


def test_exports_every_header_symbol(L):
    names = header_functions()
    assert set(names) == set(_lib.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    assert L.sa_abi_version() == 1


def test_workspace_sizes(L):
    ws = L.sa_workspace_size
    assert ws(_lib.SA_OP_HYBRID_DECODE, 4, 1, 64, 262144, 8192, 2048) > 4 * 262144 * 12
    assert ws(_lib.SA_OP_HYBRID_DECODE, 4, 2, 64, 262144, 8192, 2048) == 0   # decode is one query per sequence
    assert ws(_lib.SA_OP_INDEX_TOPK, 1, 1, 8, 1024, 0, 0) == 0               # k = 0 is invalid
    assert ws(99, 1, 1, 8, 1024, 0, 64) == 0
    assert ws(_lib.SA_OP_SPARSE_ATTN, 1, 1, 129, 1024, 0, 64) == 0           # H > 128
    # batch scales the decode workspace linearly, per sequence independent of the batch
    a = ws(_lib.SA_OP_INDEX_TOPK, 1, 1, 64, 16384, 0, 512)
    b = ws(_lib.SA_OP_INDEX_TOPK, 8, 1, 64, 16384, 0, 512)
    assert a > 0 and b > 7 * (a - 1024)
    assert ws(_lib.SA_OP_HYBRID_PREFILL, 1, 131072, 64, 32768, 1024, 2048) >= 1024 * 32768 * 4


FAKE = 0x10000          # aligned, never dereferenced: every call below fails validation first


def _cache(**kw):
    c = _lib.SaCache(FAKE, FAKE, None, None, FAKE, FAKE, 1, 1024, 128, 64, 4, _lib.SA_BF16)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _raw(**kw):
    r = _lib.SaRaw(FAKE, FAKE, FAKE, FAKE, 1, 4096, 128, 64)
    for k, v in kw.items():
        setattr(r, k, v)
    return r


@pytest.mark.parametrize("raw_kw,cache_kw,frag", [
    ({}, {"d": 64}, "head dim"),
    ({}, {"m": 3}, "power of two"),
    ({}, {"m": 2048}, "power of two"),
    ({}, {"dtype": 7}, "dtype"),
    ({}, {"kidx": None}, "kidx"),
    ({}, {"k": FAKE + 4}, "aligned"),
    ({}, {"dtype": _lib.SA_FP8_E4M3}, "k_scale"),
    ({}, {"dtype": _lib.SA_KV_MIXED}, "k_scale"),
    ({}, {"dtype": 3}, "dtype"),
    ({"kidx": None}, {}, "kidx"),
    ({"B": 2}, {}, "B=2"),
    ({"Lcap": 8192}, {}, "Ncap"),
    ({"d": 256}, {}, "raw d"),
])
def test_compress_rejects_bad_arguments(L, raw_kw, cache_kw, frag):
    r, c = _raw(**raw_kw), _cache(**cache_kw)
    st = L.csa_compress(ctypes.byref(r), ctypes.byref(c), None)
    assert st == _lib.SA_ERR_INVALID_ARG
    assert frag in L.sa_last_error().decode()


@pytest.mark.parametrize("raw_kw,cache_kw,frag", [
    ({}, {"m": 3}, "power of two"),
    ({"Lcap": 8192}, {}, "Ncap"),
    ({"kidx": None}, {}, "kidx"),
])
def test_append_rejects_bad_arguments(L, raw_kw, cache_kw, frag):
    r, c = _raw(**raw_kw), _cache(**cache_kw)
    assert L.csa_append(ctypes.byref(r), ctypes.byref(c), 1, None) == _lib.SA_ERR_INVALID_ARG
    assert frag in L.sa_last_error().decode()
    r, c = _raw(), _cache()
    assert L.csa_append(ctypes.byref(r), ctypes.byref(c), -1, None) == _lib.SA_ERR_INVALID_ARG
    assert "max_new_tokens" in L.sa_last_error().decode()
    h = _cache(m=128, kidx=None)
    assert L.hca_append(ctypes.byref(r), ctypes.byref(h), -5, None) == _lib.SA_ERR_INVALID_ARG
    assert "hca_append" in L.sa_last_error().decode()


def test_window_and_merge_reject_bad_arguments(L):
    P = ctypes.c_void_p
    r = _raw()
    assert L.swa_attn(P(FAKE), 1, 8, None, ctypes.byref(r), 0, 0.0, P(FAKE), None, P(FAKE), 1 << 30, None) == 1
    assert "window" in L.sa_last_error().decode()
    assert L.swa_attn(P(FAKE), 4, 8, None, ctypes.byref(r), 64, 0.0, P(FAKE), None, P(FAKE), 1 << 30, None) == 1
    assert "q_pos" in L.sa_last_error().decode()
    assert L.swa_attn(P(FAKE), 1, 8, None, None, 64, 0.0, P(FAKE), None, P(FAKE), 1 << 30, None) == 1
    assert L.swa_attn(P(FAKE), 1, 8, None, ctypes.byref(r), 64, 0.0, P(FAKE), None, P(FAKE), 16, None) == 3
    assert L.attn_lse_merge(P(FAKE), P(FAKE), P(FAKE), P(FAKE), -1, P(FAKE), None, None) == 1
    assert L.attn_lse_merge(P(FAKE), P(FAKE), P(FAKE + 4), P(FAKE), 8, P(FAKE), None, None) == 1
    assert "aligned" in L.sa_last_error().decode()
    assert L.attn_lse_merge(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 0, P(FAKE), None, None) == 0  # nothing to do
    assert L.sa_workspace_size(6, 2, 1, 64, 0, 0, 128) > 256
    assert L.sa_workspace_size(6, 2, 1, 64, 0, 0, 0) == 0


def test_null_descriptors(L):
    assert L.csa_compress(None, None, None) == _lib.SA_ERR_INVALID_ARG
    c = _cache()
    assert L.hca_compress(None, ctypes.byref(c), None) == _lib.SA_ERR_INVALID_ARG
    assert "raw descriptor" in L.sa_last_error().decode()


def test_topk_and_attention_reject_bad_arguments(L):
    c = _cache()
    P = ctypes.c_void_p
    # k out of range
    assert L.csa_index_topk(P(FAKE), 1, None, ctypes.byref(c), 0, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    # decode with Tq > 1
    assert L.csa_index_topk(P(FAKE), 2, None, ctypes.byref(c), 8, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    # workspace too small
    st = L.csa_index_topk(P(FAKE), 1, None, ctypes.byref(c), 8, P(FAKE), P(FAKE), P(FAKE), 16, None)
    assert st == _lib.SA_ERR_WORKSPACE and "workspace" in L.sa_last_error().decode()
    # misaligned workspace
    st = L.csa_index_topk(P(FAKE), 1, None, ctypes.byref(c), 8, P(FAKE), P(FAKE), P(FAKE + 16), 1 << 30, None)
    assert st == _lib.SA_ERR_WORKSPACE
    # H out of range, negative scale, NaN scale
    assert L.csa_sparse_attn(P(FAKE), 1, 0, ctypes.byref(c), P(FAKE), P(FAKE), 8, 0.0, P(FAKE), None, P(FAKE),
                             1 << 30, None) == 1
    assert L.hca_dense_attn(P(FAKE), 1, 8, None, ctypes.byref(c), -1.0, P(FAKE), None, P(FAKE), 1 << 30, None) == 1
    assert L.hca_dense_attn(P(FAKE), 1, 8, None, ctypes.byref(c), float("nan"), P(FAKE), None, P(FAKE), 1 << 30,
                            None) == 1
    # prefill needs idx_out / cnt_out
    h = _cache(m=128, kidx=None)
    assert L.hybrid_attn_prefill(P(FAKE), P(FAKE), 16, 8, ctypes.byref(c), ctypes.byref(h), 8, 0.0, P(FAKE),
                                 P(FAKE), None, None, None, None, P(FAKE), 1 << 30, None) == 1
    assert "idx_out" in L.sa_last_error().decode()
    # mismatched batches
    h2 = _cache(m=128, kidx=None, B=2)
    assert L.hybrid_attn_decode(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h2), 8, 0.0, P(FAKE), P(FAKE),
                                None, None, None, None, P(FAKE), 1 << 30, None) == 1
    assert "B=" in L.sa_last_error().decode()


def test_mxfp4_entry_points_reject_bad_arguments(L):
    c = _cache()
    P = ctypes.c_void_p
    q = L.csa_index_quantize_mxfp4
    assert q(ctypes.byref(c), 0, None, P(FAKE), None) == 1
    assert q(ctypes.byref(c), 0, P(FAKE), P(FAKE + 2), None) == 1
    assert "aligned" in L.sa_last_error().decode()
    assert q(ctypes.byref(c), -1, P(FAKE), P(FAKE), None) == 1
    assert "row_from" in L.sa_last_error().decode()
    assert q(ctypes.byref(_cache(kidx=None)), 0, P(FAKE), P(FAKE), None) == 1
    assert q(ctypes.byref(c), c.Ncap, P(FAKE), P(FAKE), None) == 0  # no entry to write: nothing launched
    t = L.csa_index_topk_mxfp4
    assert t(P(FAKE), 1, None, ctypes.byref(c), P(FAKE), P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    assert t(P(FAKE), 1, None, ctypes.byref(c), P(FAKE + 8), P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    assert t(P(FAKE), 1, None, ctypes.byref(c), None, P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    st = t(P(FAKE), 1, None, ctypes.byref(c), P(FAKE), P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 16, None)
    assert st == _lib.SA_ERR_WORKSPACE
    # decode needs Tq == 1; prefill needs an aligned q_pos and the prefill workspace
    assert t(P(FAKE), 2, None, ctypes.byref(c), P(FAKE), P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    assert "Tq == 1" in L.sa_last_error().decode()
    assert t(P(FAKE), 2, P(FAKE + 4), ctypes.byref(c), P(FAKE), P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 1 << 30,
             None) == 1
    st = t(P(FAKE), 64, P(FAKE), ctypes.byref(c), P(FAKE), P(FAKE), 8, P(FAKE), P(FAKE), P(FAKE), 256, None)
    assert st == _lib.SA_ERR_WORKSPACE


def test_hybrid_decode_mxfp4_rejects_bad_arguments(L):
    c, h = _cache(kidx=None), _cache(m=128, kidx=None)
    P = ctypes.c_void_p
    f = L.hybrid_attn_decode_mxfp4
    args = [P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h)]
    rest = [8, 0.0, P(FAKE), P(FAKE), None, None, None, None, P(FAKE), 1 << 30, None]
    assert f(*args, None, P(FAKE), *rest) == 1
    assert "codes" in L.sa_last_error().decode()
    assert f(*args, P(FAKE + 4), P(FAKE), *rest) == 1
    assert "aligned" in L.sa_last_error().decode()
    h2 = _cache(m=128, kidx=None, B=2)
    assert f(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h2), P(FAKE), P(FAKE), *rest) == 1
    assert "B=" in L.sa_last_error().decode()
    small = [8, 0.0, P(FAKE), P(FAKE), None, None, None, None, P(FAKE), 16, None]
    assert f(*args, P(FAKE), P(FAKE), *small) == _lib.SA_ERR_WORKSPACE
    # the bf16 entry point still needs the bf16 indexer keys
    assert L.hybrid_attn_decode(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h), *rest) == 1
    assert "kidx" in L.sa_last_error().decode()


def test_context_parallel_entry_points_reject_bad_arguments(L):
    c = _cache()
    P = ctypes.c_void_p
    cand = L.cp_decode_candidates
    assert cand(P(FAKE), ctypes.byref(c), 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    assert cand(P(FAKE), ctypes.byref(c), 8, None, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 30, None) == 1
    assert cand(P(FAKE), ctypes.byref(_cache(kidx=None)), 8, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1 << 30,
                None) == 1
    assert cand(P(FAKE), ctypes.byref(c), 8, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, None) == \
        _lib.SA_ERR_WORKSPACE
    ms = L.cp_decode_merge_select
    ok = [P(FAKE)] * 3
    outs = [P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None]
    assert ms(*ok, 8, 1, 0, 1, 8, 0, *outs) == 1                        # W = 0
    assert ms(*ok, 8, 1, 2, 1, 8, 2, *outs) == 1                        # rank outside 0..W-1
    assert "rank" in L.sa_last_error().decode()
    assert ms(*ok, 4096, 1, 8, 1, 4096, 0, *outs) == _lib.SA_ERR_UNSUPPORTED  # 32768 candidates
    assert ms(*ok, 8, 1, 2, 1, 8, 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None) == 1  # sel_idx without sel_cnt
    assert "sel_idx" in L.sa_last_error().decode()
    assert ms(P(FAKE + 2), P(FAKE), P(FAKE), 8, 1, 2, 1, 8, 0, P(FAKE), P(FAKE), P(FAKE), None, None, None) == 1
    assert "aligned" in L.sa_last_error().decode()
    assert ms(*ok, 7, 1, 2, 1, 8, 0, *outs) == 1                        # stride_list < B*k
    assert "stride" in L.sa_last_error().decode()
    mn = L.attn_lse_merge_n
    assert mn(P(FAKE), P(FAKE), 0, 8, 1024, 8, P(FAKE), None, None) == 1
    assert mn(P(FAKE), P(FAKE), 2, -1, 1024, 8, P(FAKE), None, None) == 1
    assert mn(P(FAKE), P(FAKE + 2), 2, 8, 1024, 8, P(FAKE), None, None) == 1
    assert mn(P(FAKE), P(FAKE), 2, 8, 1020, 8, P(FAKE), None, None) == 1   # stride_out < rows * 128
    assert mn(P(FAKE), P(FAKE), 2, 8, 1028, 8, P(FAKE), None, None) == 1   # not a multiple of 8
    assert mn(P(FAKE), P(FAKE), 2, 0, 0, 0, P(FAKE), None, None) == 0      # nothing to do
    assert L.sa_workspace_size(7, 2, 1, 64, 262144, 0, 2048) > 0
    assert L.sa_workspace_size(7, 2, 2, 64, 262144, 0, 2048) == 0  # decode only


def test_hybrid_decode_swa_rejects_bad_arguments(L):
    c, h, r = _cache(), _cache(m=128, kidx=None), _raw()
    P = ctypes.c_void_p
    f = L.hybrid_attn_decode_swa
    tail = [P(FAKE), P(FAKE), None, None, None, None, P(FAKE), 1 << 30, None]
    assert f(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h), None, 64, 8, 0.0, *tail) == 1
    assert "raw" in L.sa_last_error().decode()
    assert f(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h), ctypes.byref(r), 0, 8, 0.0, *tail) == 1
    assert "window" in L.sa_last_error().decode()
    r2 = _raw(B=2)
    assert f(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h), ctypes.byref(r2), 64, 8, 0.0, *tail) == 1
    assert "B=" in L.sa_last_error().decode()
    small = [P(FAKE), P(FAKE), None, None, None, None, P(FAKE), 16, None]
    assert f(P(FAKE), P(FAKE), 8, ctypes.byref(c), ctypes.byref(h), ctypes.byref(r), 64, 8, 0.0, *small) == \
        _lib.SA_ERR_WORKSPACE
    ws = L.sa_workspace_size
    # the window-inclusive step needs more than the plain one, whatever the window
    assert ws(8, 4, 1, 64, 262144, 8192, 2048) > ws(4, 4, 1, 64, 262144, 8192, 2048) > 0
    assert ws(8, 4, 2, 64, 262144, 8192, 2048) == 0


def test_selftest_rejects_bad_arguments(L):
    assert L.sa_selftest_wait_timeout(0, None) == _lib.SA_ERR_INVALID_ARG
    assert L.sa_selftest_wait_timeout((1 << 22) + 1, None) == _lib.SA_ERR_INVALID_ARG
    assert "wait_tries" in L.sa_last_error().decode()


def test_options_on_the_host(L):
    import sparse_attention_pool_b200 as S
    v = ctypes.c_int64(-1)
    assert L.sa_get_option(_lib.SA_OPT_PREFILL_SELECT, ctypes.byref(v)) == _lib.SA_OK and v.value == 4  # default
    try:
        S.set_option(S.SA_OPT_PREFILL_SELECT, 2)
        assert S.get_option(S.SA_OPT_PREFILL_SELECT) == 2
        assert L.sa_set_option(_lib.SA_OPT_PREFILL_SELECT, 5) == _lib.SA_ERR_INVALID_ARG
        assert "SA_OPT_PREFILL_SELECT" in L.sa_last_error().decode()
        assert S.get_option(S.SA_OPT_PREFILL_SELECT) == 2  # a refused value changes nothing
        assert L.sa_set_option(99, 1) == _lib.SA_ERR_INVALID_ARG
        assert L.sa_get_option(99, ctypes.byref(v)) == _lib.SA_ERR_INVALID_ARG
        assert L.sa_get_option(_lib.SA_OPT_PREFILL_SELECT, None) == _lib.SA_ERR_INVALID_ARG
        with pytest.raises(S.SparseAttnError):
            S.set_option(S.SA_OPT_PREFILL_SELECT, 0)
    finally:
        S.set_option(S.SA_OPT_PREFILL_SELECT, 4)
    assert L.sa_get_option(_lib.SA_OPT_DECODE_FAST, ctypes.byref(v)) == _lib.SA_OK and v.value == 0  # default
    try:
        for val in (1, 2, 0):
            S.set_option(S.SA_OPT_DECODE_FAST, val)
            assert S.get_option(S.SA_OPT_DECODE_FAST) == val
        assert L.sa_set_option(_lib.SA_OPT_DECODE_FAST, 3) == _lib.SA_ERR_INVALID_ARG
        assert "SA_OPT_DECODE_FAST" in L.sa_last_error().decode()
        assert L.sa_set_option(_lib.SA_OPT_DECODE_FAST, -1) == _lib.SA_ERR_INVALID_ARG
        assert S.get_option(S.SA_OPT_DECODE_FAST) == 0
    finally:
        S.set_option(S.SA_OPT_DECODE_FAST, 0)
    assert L.sa_get_option(_lib.SA_OPT_HCA_PREFILL, ctypes.byref(v)) == _lib.SA_OK and v.value == 0  # default
    try:
        S.set_option(S.SA_OPT_HCA_PREFILL, 1)
        assert S.get_option(S.SA_OPT_HCA_PREFILL) == 1
        S.set_option(S.SA_OPT_HCA_PREFILL, 2)
        assert S.get_option(S.SA_OPT_HCA_PREFILL) == 2
        S.set_option(S.SA_OPT_HCA_PREFILL, 1)
        assert L.sa_set_option(_lib.SA_OPT_HCA_PREFILL, 3) == _lib.SA_ERR_INVALID_ARG
        assert "SA_OPT_HCA_PREFILL" in L.sa_last_error().decode()
        assert S.get_option(S.SA_OPT_HCA_PREFILL) == 1
    finally:
        S.set_option(S.SA_OPT_HCA_PREFILL, 0)


def test_trace_calls_need_the_profiling_build(L):
    n = ctypes.c_uint32(7)
    assert L.sa_trace_install(None, 0, None) == _lib.SA_ERR_UNSUPPORTED
    assert "SA_TRACE" in L.sa_last_error().decode()
    assert L.sa_trace_count(ctypes.byref(n), None) == _lib.SA_ERR_UNSUPPORTED and n.value == 0
    assert L.sa_trace_count(None, None) == _lib.SA_ERR_INVALID_ARG


def test_profiling_build_exports_every_header_symbol():
    build.build(trace=True)
    T = ctypes.CDLL(_lib.TRACE_LIB_PATH)
    for n in header_functions():
        assert hasattr(T, n), n
    T.sa_trace_install.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    T.sa_trace_install.restype = ctypes.c_int32
    T.sa_last_error.restype = ctypes.c_char_p
    # argument checks run before any CUDA call
    assert T.sa_trace_install(ctypes.c_void_p(0x10004), 8, None) == _lib.SA_ERR_INVALID_ARG


def test_hybrid_prefill_mxfp4_rejects_bad_arguments(L):
    c, h = _cache(kidx=None), _cache(m=128, kidx=None)
    P = ctypes.c_void_p
    f = L.hybrid_attn_prefill_mxfp4
    rest = [8, 0.0, P(FAKE), P(FAKE), None, None, P(FAKE), P(FAKE), P(FAKE), 1 << 30, None]
    assert f(P(FAKE), P(FAKE), 16, 8, ctypes.byref(c), ctypes.byref(h), None, P(FAKE), *rest) == 1
    assert "codes" in L.sa_last_error().decode()
    nocnt = [8, 0.0, P(FAKE), P(FAKE), None, None, P(FAKE), None, P(FAKE), 1 << 30, None]
    assert f(P(FAKE), P(FAKE), 16, 8, ctypes.byref(c), ctypes.byref(h), P(FAKE), P(FAKE), *nocnt) == 1
    assert "idx_out" in L.sa_last_error().decode()
    # the bf16 prefill still needs the bf16 indexer keys
    assert L.hybrid_attn_prefill(P(FAKE), P(FAKE), 16, 8, ctypes.byref(c), ctypes.byref(h), *rest) == 1
    assert "kidx" in L.sa_last_error().decode()


def test_header_is_plain_c_and_cpp():
    """The boundary is a C ABI: the header compiles as strict C99 and as C++17,
    and a C caller links against the library's exports."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    for std, lang in (("c99", "c"), ("c++17", "c++")):
        subprocess.check_call([gcc, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                               "-x", lang, HEADER])
    caller = ("#include \"sparse_attn.h\"\n"
              "int main(void) {\n"
              "    size_t n = sa_workspace_size(SA_OP_HYBRID_DECODE, 4, 1, 64, 262144, 8192, 2048);\n"
              "    return (sa_abi_version() == SA_ABI_VERSION && n > 0) ? 0 : 1;\n"
              "}\n")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), "-x", "c", "-", "-o",
                    os.devnull, "-L", lib_dir, "-l:libsparse_attn.so"], input=caller.encode(), check=True)


@pytest.mark.parametrize("op", [1, 2, 3, 4, 5, 6, 7, 8])
def test_workspace_sizes_are_monotone(L, op):
    """Every op's scratch never shrinks as the batch, the capacities or k grow."""
    ws = L.sa_workspace_size
    Tq = 4096 if op in (5,) else 1
    base = dict(B=2, Tq=Tq, H=64, Nc=65536, Nh=2048, k=512)

    def size(**kw):
        a = dict(base, **kw)
        return ws(op, a["B"], a["Tq"], a["H"], a["Nc"], a["Nh"], a["k"])
    s0 = size()
    assert s0 >= 0
    for key, bigger in (("B", 4), ("Nc", 262144), ("Nh", 8192), ("k", 2048), ("H", 128)):
        assert size(**{key: bigger}) >= s0, key
    assert ws(8, 4, 1, 64, 262144, 8192, 2048) >= ws(4, 4, 1, 64, 262144, 8192, 2048)


def test_decode_io_layout_on_the_host(L):
    io = _lib.SaDecodeIO()
    assert L.sa_decode_io_layout(4, 64, ctypes.byref(io)) == _lib.SA_OK
    rows = 4 * 64
    # q_idx then q; out_hca, lse_hca, out_csa, lse_csa: every region 256-byte aligned and large enough
    assert io.q_idx_off == 0 and io.q_off == 512 and io.in_bytes == 512 + rows * 256
    assert io.out_hca_off == 0 and io.lse_hca_off == rows * 256
    assert io.out_csa_off == io.lse_hca_off + rows * 4 and io.lse_csa_off == io.out_csa_off + rows * 256
    assert io.out_bytes == io.lse_csa_off + rows * 4
    assert L.sa_decode_io_layout(3, 5, ctypes.byref(io)) == _lib.SA_OK
    offs = [io.q_idx_off, io.q_off, io.out_hca_off, io.lse_hca_off, io.out_csa_off, io.lse_csa_off]
    assert all(o % 256 == 0 for o in offs)
    assert io.q_off >= 3 * 64 * 2 and io.in_bytes - io.q_off >= 15 * 256
    assert io.lse_hca_off >= 15 * 256 and io.out_csa_off - io.lse_hca_off >= 15 * 4
    assert io.out_bytes - io.lse_csa_off >= 15 * 4
    for B, H in ((0, 64), (4, 0), (4, 129)):
        assert L.sa_decode_io_layout(B, H, ctypes.byref(io)) == _lib.SA_ERR_INVALID_ARG
    assert L.sa_decode_io_layout(4, 64, None) == _lib.SA_ERR_INVALID_ARG


def test_decode_graph_rejects_bad_arguments(L):
    g = ctypes.c_void_p()
    c = _lib.SaCache()
    args = [ctypes.byref(c), ctypes.byref(c), 64, 512, 0.0, None, None, None, None, None, None, None, None, None, 0,
            0]
    assert L.sa_decode_graph_create(*args, None) == _lib.SA_ERR_INVALID_ARG
    assert "graph" in L.sa_last_error().decode()
    args2 = list(args)
    args2[0] = None
    assert L.sa_decode_graph_create(*args2, ctypes.byref(g)) == _lib.SA_ERR_INVALID_ARG and not g.value
    args3 = list(args)
    args3[5] = ctypes.c_void_p(16)  # codes without scales
    assert L.sa_decode_graph_create(*args3, ctypes.byref(g)) == _lib.SA_ERR_INVALID_ARG
    assert "codes" in L.sa_last_error().decode()
    args4 = list(args)
    args4[15] = 8  # an unknown flag
    assert L.sa_decode_graph_create(*args4, ctypes.byref(g)) == _lib.SA_ERR_INVALID_ARG
    assert "flags" in L.sa_last_error().decode()
    c.B = 2
    assert L.sa_decode_graph_create(*args, ctypes.byref(g)) == _lib.SA_ERR_INVALID_ARG  # NULL buffers
    assert "I/O buffers" in L.sa_last_error().decode()
    assert L.sa_decode_graph_step(None, None) == _lib.SA_ERR_INVALID_ARG
    assert L.sa_decode_graph_destroy(None) == _lib.SA_OK
