"""ctypes front end of the fp64 C oracle (``sa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` import this module; the library itself never
does.  The oracle shares no code with the CUDA path.  The method it follows
is the CSA / HCA hybrid attention of "DeepSeek-V4: Towards Highly Efficient
Million-Token Context Intelligence Review", section 3-2 (2) "Hybrid attention
with CSA and HCA" (component table); the readings of what that section leaves
open are listed in the header of ``sa_oracle.c``.

All bf16 tensors are passed as numpy ``uint16`` bit patterns, e4m3 tensors as
``uint8`` codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no CUDA involved)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.or_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_double.restype = dbl
        L.or_bf16_from_double.argtypes = [dbl]
        L.or_bf16_from_double.restype = ctypes.c_uint16
        L.or_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.or_e4m3_to_double.restype = dbl
        L.or_e4m3_from_double_satfinite.argtypes = [dbl]
        L.or_e4m3_from_double_satfinite.restype = ctypes.c_uint8
        L.or_compress.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P]
        L.or_compress.restype = i64
        L.or_fp8_quantize.argtypes = [P, i64, ctypes.c_int, P, P]
        L.or_fp8_quantize.restype = None
        L.or_index_scores.argtypes = [P, P, i64, ctypes.c_int, P]
        L.or_index_scores.restype = None
        L.or_topk.argtypes = [P, i64, i32, P]
        L.or_topk.restype = i32
        L.or_attention.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P, ctypes.c_int, P, i64, dbl, P, P, P]
        L.or_attention.restype = None
        L.or_hybrid_query.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, i64,
                                      ctypes.c_int, P, P, P, P, P, i64,
                                      ctypes.c_int, P, P, P, P, i64, ctypes.c_int, i32, dbl,
                                      P, P, P, P, P, P]
        L.or_hybrid_query.restype = None
        L.or_e2m1_to_double.argtypes = [ctypes.c_uint8]
        L.or_e2m1_to_double.restype = dbl
        L.or_e2m1_from_double_satfinite.argtypes = [dbl]
        L.or_e2m1_from_double_satfinite.restype = ctypes.c_uint8
        L.or_e8m0_to_double.argtypes = [ctypes.c_uint8]
        L.or_e8m0_to_double.restype = dbl
        L.or_mxfp4_quantize.argtypes = [P, i64, ctypes.c_int, P, P]
        L.or_mxfp4_quantize.restype = None
        L.or_mxfp4_index_scores.argtypes = [P, P, P, P, i64, ctypes.c_int, P]
        L.or_mxfp4_index_scores.restype = None
        L.or_mixed_quantize.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P, P]
        L.or_mixed_quantize.restype = None
        L.or_attention_kv.argtypes = [P, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, P, P, P, ctypes.c_int, P, P, P, ctypes.c_int,
                                      P, i64, dbl, P, P]
        L.or_attention_kv.restype = None
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# -- number formats ---------------------------------------------------------

def bf16_to_double(bits: int) -> float:
    return lib().or_bf16_to_double(int(bits))


def bf16_from_double(x: float) -> int:
    return int(lib().or_bf16_from_double(float(x)))


def e4m3_to_double(code: int) -> float:
    return lib().or_e4m3_to_double(int(code))


def e4m3_from_double(x: float) -> int:
    return int(lib().or_e4m3_from_double_satfinite(float(x)))


def bf16_array_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode an array of bf16 bit patterns through the oracle's codec."""
    table = np.array([lib().or_bf16_to_double(i) for i in range(65536)], dtype=np.float64)
    return table[np.asarray(bits, dtype=np.uint16)]


def e4m3_array_to_f64(codes: np.ndarray) -> np.ndarray:
    table = np.array([lib().or_e4m3_to_double(i) for i in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


# -- the method ---------------------------------------------------------------

def compress(x: np.ndarray, m: int) -> np.ndarray:
    """O1: x [L][d] uint16 -> [L // m][d] uint16 (mean of each complete block)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    L, d = x.shape
    out = np.zeros((L // m, d), dtype=np.uint16)
    n = lib().or_compress(_p(x), L, d, m, _p(out))
    assert n == L // m
    return out


def fp8_quantize(xc: np.ndarray):
    """O2: xc [n][d] uint16 -> (codes [n][d] uint8, scales [ceil(n/64)] float32)."""
    xc = np.ascontiguousarray(xc, dtype=np.uint16)
    n, d = xc.shape
    codes = np.zeros((n, d), dtype=np.uint8)
    scales = np.zeros(((n + 63) // 64,), dtype=np.float32)
    lib().or_fp8_quantize(_p(xc), n, d, _p(codes), _p(scales))
    return codes, scales


def index_scores(qI: np.ndarray, Ic: np.ndarray) -> np.ndarray:
    """O3: qI [dI] uint16, Ic [n][dI] uint16 -> fp32 scores [n]."""
    qI = np.ascontiguousarray(qI, dtype=np.uint16)
    Ic = np.ascontiguousarray(Ic, dtype=np.uint16)
    n, dI = Ic.shape
    s = np.zeros((n,), dtype=np.float32)
    lib().or_index_scores(_p(qI), _p(Ic), n, dI, _p(s))
    return s


def topk(s: np.ndarray, k: int, n_visible: int | None = None):
    """O4: returns (idx [k] int32 ascending, -1 padded; count)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    nv = s.shape[0] if n_visible is None else n_visible
    idx = np.zeros((k,), dtype=np.int32)
    cnt = lib().or_topk(_p(s), nv, k, _p(idx))
    return idx, int(cnt)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, rows, scale: float,
              k_scales: np.ndarray | None = None, v_scales: np.ndarray | None = None,
              return_p: bool = False):
    """O5: q [H][d] uint16; K, V [N][d] uint16 (bf16) or uint8 (e4m3 + scales).

    Returns (out [H][d] f64, lse [H] f64[, p [H][nrows] f64]).
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    H, d = q.shape
    fp8 = K.dtype == np.uint8
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    out = np.zeros((H, d), dtype=np.float64)
    lse = np.zeros((H,), dtype=np.float64)
    p = np.zeros((H, max(rows.shape[0], 1)), dtype=np.float64) if return_p else None
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    ks = None if k_scales is None else np.ascontiguousarray(k_scales, dtype=np.float32)
    vs = None if v_scales is None else np.ascontiguousarray(v_scales, dtype=np.float32)
    lib().or_attention(_p(q), H, d, _p(K), _p(ks), _p(V), _p(vs), int(fp8), _p(rows), rows.shape[0],
                       float(scale), _p(out), _p(lse), _p(p))
    if return_p:
        return out, lse, p[:, :rows.shape[0]]
    return out, lse


class CompressedSeq:
    """One sequence's compressed caches as the oracle builds them (O1 + O2)."""

    def __init__(self, K, V, KI, m_csa=4, m_hca=128, fp8=False):
        self.fp8 = fp8
        self.m_csa, self.m_hca = m_csa, m_hca
        ck, cv = compress(K, m_csa), compress(V, m_csa)
        hk, hv = compress(K, m_hca), compress(V, m_hca)
        self.cidx = compress(KI, m_csa)
        self.n_csa, self.n_hca = ck.shape[0], hk.shape[0]
        self.ck_bf16, self.cv_bf16, self.hk_bf16, self.hv_bf16 = ck, cv, hk, hv
        if fp8:
            self.ck, self.cks = fp8_quantize(ck)
            self.cv, self.cvs = fp8_quantize(cv)
            self.hk, self.hks = fp8_quantize(hk)
            self.hv, self.hvs = fp8_quantize(hv)
        else:
            self.ck, self.cv, self.hk, self.hv = ck, cv, hk, hv
            self.cks = self.cvs = self.hks = self.hvs = None


def hybrid_query(cs: CompressedSeq, q: np.ndarray, qI: np.ndarray, t: int, k: int, scale: float):
    """O6 for one query at token position t.  Returns a dict of results."""
    L = lib()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    qI = np.ascontiguousarray(qI, dtype=np.uint16)
    H, d = q.shape
    dI = qI.shape[0]
    idx = np.zeros((k,), dtype=np.int32)
    cnt = np.zeros((1,), dtype=np.int32)
    oc = np.zeros((H, d)); lc = np.zeros((H,))
    oh = np.zeros((H, d)); lh = np.zeros((H,))

    def c(a):
        return None if a is None else np.ascontiguousarray(a)
    ck, cks, cv, cvs = c(cs.ck), c(cs.cks), c(cs.cv), c(cs.cvs)
    hk, hks, hv, hvs = c(cs.hk), c(cs.hks), c(cs.hv), c(cs.hvs)
    cidx = c(cs.cidx)
    # keep 1-element dummies so that empty caches still pass valid pointers
    dummy16 = np.zeros((1,), dtype=np.uint16)
    L.or_hybrid_query(_p(q), _p(qI), H, d, dI, int(t),
                      cs.m_csa, _p(ck if ck.size else dummy16), _p(cks), _p(cv if cv.size else dummy16), _p(cvs),
                      _p(cidx if cidx.size else dummy16), cs.n_csa,
                      cs.m_hca, _p(hk if hk.size else dummy16), _p(hks), _p(hv if hv.size else dummy16), _p(hvs),
                      cs.n_hca, int(cs.fp8), int(k), float(scale),
                      _p(idx), _p(cnt), _p(oc), _p(lc), _p(oh), _p(lh))
    return {"idx": idx, "cnt": int(cnt[0]), "out_csa": oc, "lse_csa": lc, "out_hca": oh, "lse_hca": lh}


def window_rows(t: int, n_raw: int, window: int):
    """Raw tokens a query at position t sees in the sliding-window branch:
    the last `window` of the tokens before t (reading in the design notes)."""
    T = min(int(n_raw), int(t))
    return np.arange(max(0, T - int(window)), T, dtype=np.int32)


def union_attention(q: np.ndarray, parts, scale: float):
    """Softmax attention over the union of several key sets, each given as
    (K [N][d] uint16 bf16, V [N][d] uint16 bf16, rows); one softmax over all
    of them (the sliding-window branch joined with a compressed branch,
    "DeepSeek-V4 ... Review" section 3-2 (2)).  Returns (out [H][d], lse [H])."""
    Ks, Vs = [], []
    for K, V, rows in parts:
        rows = np.asarray(rows, dtype=np.int64)
        Ks.append(np.asarray(K, dtype=np.uint16)[rows])
        Vs.append(np.asarray(V, dtype=np.uint16)[rows])
    d = np.asarray(q).shape[1]
    Ku = np.concatenate(Ks, axis=0) if Ks else np.zeros((0, d), np.uint16)
    Vu = np.concatenate(Vs, axis=0) if Vs else np.zeros((0, d), np.uint16)
    if Ku.shape[0] == 0:
        H = np.asarray(q).shape[0]
        return np.zeros((H, d)), np.full((H,), -np.inf)
    return attention(q, Ku, Vu, np.arange(Ku.shape[0], dtype=np.int32), scale)


# -- low-precision storage on the CSA path ------------------------------------
# "DeepSeek-V4 ... Review", section 3-2 (2) ("Mixed KV storage": rotary dims in
# BF16, the rest in FP8) and section 3-2 (4) (FP4 on the CSA indexer QK path).
# The readings (MXFP4 for the indexer, the last d_rope dims of K as the rotary
# dims, V all e4m3) are stated in the header of sa_oracle.c.

def e2m1_to_double(code: int) -> float:
    return lib().or_e2m1_to_double(int(code))


def e2m1_from_double(x: float) -> int:
    return int(lib().or_e2m1_from_double_satfinite(float(x)))


def e8m0_to_double(code: int) -> float:
    return lib().or_e8m0_to_double(int(code))


def mxfp4_quantize(x: np.ndarray):
    """x [n][d] uint16 (bf16), d a multiple of 32 -> (codes [n][d/2] uint8,
    element 2i in the low nibble; scales [n][d/32] uint8 E8M0 codes)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    n, d = x.shape
    assert d % 32 == 0
    codes = np.zeros((n, d // 2), dtype=np.uint8)
    scales = np.zeros((n, d // 32), dtype=np.uint8)
    lib().or_mxfp4_quantize(_p(x), n, d, _p(codes), _p(scales))
    return codes, scales


def mxfp4_to_f64(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantize MXFP4 rows: [n][d/2] codes, [n][d/32] scales -> [n][d] f64."""
    codes = np.asarray(codes, dtype=np.uint8)
    n, half = codes.shape
    table = np.array([lib().or_e2m1_to_double(c) for c in range(16)], dtype=np.float64)
    el = np.empty((n, 2 * half), dtype=np.float64)
    el[:, 0::2] = table[codes & 0xF]
    el[:, 1::2] = table[codes >> 4]
    sc = np.array([lib().or_e8m0_to_double(c) for c in range(256)], dtype=np.float64)[np.asarray(scales, np.uint8)]
    return el * np.repeat(sc, 32, axis=1)


def mxfp4_index_scores(q_codes, q_scales, k_codes, k_scales) -> np.ndarray:
    """FP4 index scores of one MXFP4 query against n MXFP4 key rows (fp32)."""
    qc = np.ascontiguousarray(np.asarray(q_codes, np.uint8).reshape(-1))
    qs = np.ascontiguousarray(np.asarray(q_scales, np.uint8).reshape(-1))
    kc = np.ascontiguousarray(k_codes, dtype=np.uint8)
    ks = np.ascontiguousarray(k_scales, dtype=np.uint8)
    n = kc.shape[0]
    d = 2 * qc.shape[0]
    assert kc.shape[1] * 2 == d and ks.shape == (n, d // 32) and qs.shape[0] == d // 32
    s = np.zeros((n,), dtype=np.float32)
    lib().or_mxfp4_index_scores(_p(qc), _p(qs), _p(kc), _p(ks), n, d, _p(s))
    return s


def mixed_quantize(xc: np.ndarray, d_rope: int = 64):
    """Mixed storage of a compressed K: (codes [n][d - d_rope] e4m3 for the
    leading dims, scales [ceil(n/64)] fp32 over those dims, rope [n][d_rope]
    bf16 bits = the trailing dims unchanged)."""
    xc = np.ascontiguousarray(xc, dtype=np.uint16)
    n, d = xc.shape
    codes = np.zeros((n, d - d_rope), dtype=np.uint8)
    scales = np.zeros(((n + 63) // 64,), dtype=np.float32)
    rope = np.zeros((n, d_rope), dtype=np.uint16)
    lib().or_mixed_quantize(_p(xc), n, d, d_rope, _p(codes), _p(scales), _p(rope))
    return codes, scales, rope


_KV_MODES = {"bf16": 0, "fp8": 1, "mixed": 2}


def attention_kv(q: np.ndarray, k: dict, v: dict, rows, scale: float, d_rope: int = 64):
    """O5 with K and V in any storage: each of k, v is a dict with "mode"
    ("bf16", "fp8" or "mixed"), "data" (bf16 bits / e4m3 codes), "scales"
    (fp8 and mixed) and "rope" (mixed).  Returns (out [H][d], lse [H])."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    H, d = q.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    out = np.zeros((H, d), dtype=np.float64)
    lse = np.zeros((H,), dtype=np.float64)

    def parts(t):
        data = np.ascontiguousarray(t["data"])
        sc = t.get("scales")
        sc = None if sc is None else np.ascontiguousarray(sc, dtype=np.float32)
        ro = t.get("rope")
        ro = None if ro is None else np.ascontiguousarray(ro, dtype=np.uint16)
        return _KV_MODES[t["mode"]], data, sc, ro
    km, kd, ksc, kro = parts(k)
    vm, vd, vsc, vro = parts(v)
    lib().or_attention_kv(_p(q), H, d, km, _p(kd), _p(ksc), _p(kro), vm, _p(vd), _p(vsc), _p(vro),
                          int(d_rope), _p(rows), rows.shape[0], float(scale), _p(out), _p(lse))
    return out, lse


def lowp_query(K, V, KI, q, qI, t: int, k: int, scale: float, d_rope: int = 64, m: int = 4):
    """One CSA query with the low-precision storage: compress (O1), MXFP4
    indexer keys and query, FP4 scores, top-k (O4), then attention over the
    selected entries with mixed-storage K and e4m3 V.  Returns a dict."""
    ck, cv, ci = compress(K, m), compress(V, m), compress(KI, m)
    kc, ks = mxfp4_quantize(ci)
    qc, qs = mxfp4_quantize(np.asarray(qI, np.uint16).reshape(1, -1))
    n_vis = min(int(t) // m, ci.shape[0])
    s = mxfp4_index_scores(qc[0], qs[0], kc[:n_vis], ks[:n_vis])
    idx, cnt = topk(s, k)
    codes, sc, rope = mixed_quantize(ck, d_rope)
    vcodes, vsc = fp8_quantize(cv)
    out, lse = attention_kv(q, {"mode": "mixed", "data": codes, "scales": sc, "rope": rope},
                            {"mode": "fp8", "data": vcodes, "scales": vsc}, idx[:cnt], scale, d_rope)
    return {"scores": s, "idx": idx, "cnt": cnt, "out": out, "lse": lse,
            "idx_codes": kc, "idx_scales": ks, "q_codes": qc[0], "q_scales": qs[0]}


def hybrid_query_mxfp4(cs: CompressedSeq, q: np.ndarray, qI: np.ndarray, t: int, k: int, scale: float,
                       idx_codes=None, idx_scales=None):
    """O6 with the CSA selection on FP4 scores: the query and the compressed
    indexer keys in MXFP4 (reading in the header of sa_oracle.c), top-k (O4),
    then both attentions as in O6.  idx_codes / idx_scales: the keys' MXFP4
    form when already built (mxfp4_quantize(cs.cidx)).  Returns a dict like
    hybrid_query."""
    if idx_codes is None:
        idx_codes, idx_scales = mxfp4_quantize(cs.cidx)
    qc, qs = mxfp4_quantize(np.asarray(qI, np.uint16).reshape(1, -1))
    n_vis = min(int(t) // cs.m_csa, cs.n_csa)
    s = mxfp4_index_scores(qc[0], qs[0], idx_codes[:n_vis], idx_scales[:n_vis])
    idx, cnt = topk(s, k)
    oc, lc = attention(q, cs.ck, cs.cv, idx[:cnt], scale, k_scales=cs.cks, v_scales=cs.cvs)
    n_h = min(int(t) // cs.m_hca, cs.n_hca)
    oh, lh = attention(q, cs.hk, cs.hv, np.arange(n_h, dtype=np.int32), scale, k_scales=cs.hks, v_scales=cs.hvs)
    return {"idx": idx, "cnt": cnt, "out_csa": oc, "lse_csa": lc, "out_hca": oh, "lse_hca": lh}
