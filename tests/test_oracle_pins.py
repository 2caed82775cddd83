"""Pins for the fp64 CPU oracle, checked against things other than itself.

Every test here runs on the CPU (no GPU marker).  The independent sources are:
numpy's / torch's own number-format conversions, exact rational arithmetic
(``fractions.Fraction``), brute force on tiny inputs, library softmax in fp64,
closed forms, and the hand-worked fixtures under ``tests/golden/``.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_attention_pool_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def hexf(s):
    return float.fromhex(s) if "0x" in s else float(s)


def bits_of(x):
    """float values -> bf16 bit patterns through torch (exact for bf16 values)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- formats ---

def test_bf16_decode_exhaustive_vs_numpy_view():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        ref = synth.bf16_bits_to_f32(codes).astype(np.float64)
    got = O.bf16_array_to_f64(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_encode_roundtrip_all_finite():
    L = O.lib()
    for c in range(65536):
        if (c & 0x7F80) == 0x7F80:
            continue
        assert L.or_bf16_from_double(L.or_bf16_to_double(c)) == c


def test_bf16_encode_matches_torch_rne_on_float32_inputs():
    rng = np.random.default_rng(7)
    # random patterns plus exact midpoints (low 16 bits = 0x8000) and near-midpoints
    u = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]                       # finite only
    mids = (u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    near = mids + np.uint32(1)
    allu = np.concatenate([u, mids, near])
    allu = allu[((allu >> 23) & 0xFF) < 0xFE]                 # keep away from overflow
    x = allu.view(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.bf16_from_double(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)


def _nearest_bf16_bruteforce(x: Fraction) -> int:
    """Nearest bf16 (ties to even) of a positive rational, by checking neighbours."""
    best = None
    vals = synth.bf16_bits_to_f32(np.arange(0x7F80, dtype=np.uint16))
    for c in range(0x0000, 0x7F80):
        v = Fraction(float(vals[c]))
        d = abs(v - x)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return best[1]


def test_bf16_encode_is_single_rounding_from_double():
    # just above a bf16 midpoint by far less than an fp32 ulp: must round up
    for base in (1.0, 3.0, 0.15625, 2.0**-100):
        lo = float(Fraction(base))
        mid = lo * (1 + 2.0**-8)
        x = mid + lo * 2.0**-40
        want = _nearest_bf16_bruteforce(Fraction(x))
        assert O.bf16_from_double(x) == want
        assert O.bf16_from_double(-x) == want | 0x8000
    # overflow: the midpoint between the largest bf16 and 2^128 rounds to inf
    assert O.bf16_from_double(2.0**128 - 2.0**119) == 0x7F80
    assert O.bf16_from_double(2.0**128 - 2.0**119 - 2.0**100) == 0x7F7F
    # subnormal boundary: 2^-134 is the midpoint of 0 and the smallest subnormal
    assert O.bf16_from_double(2.0**-134) == 0
    assert O.bf16_from_double(2.0**-134 * 1.0001) == 1


def test_e4m3_decode_exhaustive_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_array_to_f64(codes.numpy())
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.isnan(got[nan]).all()
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


def test_e4m3_encode_vs_torch_in_range_and_satfinite():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(50),
        rng.standard_normal(5000).astype(np.float32) * np.float32(1e-2),
        # exact midpoints between neighbouring e4m3 values
        ((torch.arange(0, 126, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
          + torch.arange(1, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()) / 2).numpy(),
    ]).astype(np.float32)
    x = x[np.abs(x) < 464]
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_from_double(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
    for v, c in [(449.0, 0x7E), (464.0, 0x7E), (1e9, 0x7E), (-500.0, 0xFE), (0.0, 0x00), (-0.0, 0x80)]:
        assert O.e4m3_from_double(v) == c
    assert O.e4m3_from_double(float("nan")) == 0x7F
    for c in range(256):
        if (c & 0x7F) != 0x7F:
            assert O.e4m3_from_double(O.e4m3_to_double(c)) == c


# --------------------------------------------------------------- compress ---

def test_compress_golden_mean_and_tail():
    g = golden("compress_mean_m2.txt")
    m = int(g["m"][0])
    x = bits_of([float(v) for v in g["tokens"]]).reshape(-1, 1)
    out = O.compress(x, m)
    assert out.shape == (len(g["entries"]), 1)
    assert np.array_equal(bf16_value(out[:, 0]), np.array([float(v) for v in g["entries"]]))


def test_compress_golden_direct_rounding():
    g = golden("compress_direct_rounding.txt")
    m = int(g["m"][0])
    x = bits_of([hexf(v) for v in g["tokens"]]).reshape(-1, 1)
    assert np.array_equal(bf16_value(x[:, 0]), np.array([hexf(v) for v in g["tokens"]]))
    out = O.compress(x, m)
    assert bf16_value(out[:, 0])[0] == hexf(g["entries"][0])


def _is_nearest_bf16(code: int, exact: Fraction) -> bool:
    """code is a nearest bf16 of exact (ties to even), checked against both neighbours."""
    v = Fraction(float(bf16_value(np.uint16(code))))
    err = abs(v - exact)
    for nb in (code - 1, code + 1):
        if (nb & 0x7FFF) >= 0x7F80 or nb < 0 or ((nb ^ code) & 0x8000):
            continue
        e2 = abs(Fraction(float(bf16_value(np.uint16(nb)))) - exact)
        if e2 < err or (e2 == err and (code & 1)):
            return False
    return True


@pytest.mark.parametrize("m", [1, 2, 3, 4, 128])
def test_compress_equals_exact_rational_mean(m):
    L, d = (m * 5 + (m - 1 if m > 1 else 0)), 16
    x = synth.normal_bf16(123 + m, "k", (1, L * d)).reshape(L, d)
    out = O.compress(x, m)
    assert out.shape == (L // m, d)
    vals = bf16_value(x)
    for c in range(L // m):
        for i in range(0, d, 3):
            # the fp64 sum of these values is exact (their binades span < 40 bits),
            # so the specified result is the nearest bf16 of the exact rational mean
            exact = sum(Fraction(vals[t, i]) for t in range(c * m, c * m + m)) / m
            assert _is_nearest_bf16(int(out[c, i]), exact), (c, i)
    if m == 1:
        assert np.array_equal(out, x)


def test_compress_constant_block_gives_constant():
    x = np.full((12, 8), bits_of([0.7])[0], dtype=np.uint16)
    for m in (1, 3, 4, 12):
        assert np.array_equal(O.compress(x, m), x[: 12 // m])


# ------------------------------------------------------------------- fp8 ----

def test_fp8_golden_group():
    g = golden("fp8_group.txt")
    d = int(g["d"][0])
    x = bits_of([float(v) for v in g["values"]]).reshape(1, d)
    codes, scales = O.fp8_quantize(x)
    assert scales.tolist() == [float(g["scale"][0])]
    assert codes[0].tolist() == [int(c, 16) for c in g["codes"]]
    z = np.zeros((64, 4), dtype=np.uint16)
    codes, scales = O.fp8_quantize(z)
    assert scales.tolist() == [1.0] and not codes.any()


def test_fp8_groups_against_torch_encoder():
    n, d = 150, 32                               # three groups, the last one partial (22 entries)
    x = synth.normal_bf16(5, "k", (1, n * d)).reshape(n, d)
    codes, scales = O.fp8_quantize(x)
    assert scales.shape == (3,)
    vals = bf16_value(x)
    for g in range(3):
        lo, hi = g * 64, min(n, g * 64 + 64)
        amax = np.abs(vals[lo:hi]).max()
        s = np.float32(amax / 448.0)             # one division, rounded once to fp32
        assert scales[g] == s
        y = (torch.tensor(vals[lo:hi], dtype=torch.float64) / float(s)).float()
        ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes[lo:hi], ref)
        # the group's largest magnitude maps to (almost exactly) the largest code
        assert np.abs(O.e4m3_array_to_f64(codes[lo:hi])).max() == 448.0


# ---------------------------------------------------------------- scores ----

def test_score_golden_fp64_order():
    g = golden("score_fp64_order.txt")
    for case in "abc":
        q = [hexf(v) for v in g[f"q_{case}"]] + [0.0] * 61
        k = [hexf(v) for v in g[f"k_{case}"]] + [0.0] * 61
        s = O.index_scores(bits_of(q), bits_of(k).reshape(1, 64))
        assert s[0] == hexf(g[f"score_{case}"][0]), case
        assert not np.signbit(s[0])


def test_scores_equal_exact_sum_rounded_to_fp32():
    n, dI = 300, 64
    qI = synth.normal_bf16(9, "qidx", (1, dI))[0]
    Ic = synth.normal_bf16(9, "kidx", (1, n * dI)).reshape(n, dI)
    s = O.index_scores(qI, Ic)
    q = bf16_value(qI)
    K = bf16_value(Ic)
    for j in range(n):
        exact = sum(Fraction(q[i]) * Fraction(K[j, i]) for i in range(dI))
        # exact fp64 sum here: fp32 of the exact value, i.e. nearest float32
        f = np.float32(float(exact))
        cands = [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
        best = min(cands, key=lambda c: (abs(Fraction(float(c)) - exact),
                                         int(np.array([c], np.float32).view(np.uint32)[0]) & 1))
        assert s[j] == best, j


def test_scores_zero_is_positive():
    qI = bits_of([-1.0] + [0.0] * 63)
    Ic = bits_of([0.0] * 64).reshape(1, 64)
    s = O.index_scores(qI, Ic)
    assert s[0] == 0.0 and not np.signbit(s[0])


# ------------------------------------------------------------------ top-k ---

def test_topk_golden_ties():
    g = golden("topk_ties.txt")
    s = np.array([float(v) for v in g["scores"]], dtype=np.float32)
    for kk, ik in (("k", "indices"), ("k_big", "indices_big"), ("k_two", "indices_two")):
        k = int(g[kk][0])
        idx, cnt = O.topk(s, k)
        assert idx.tolist() == [int(v) for v in g[ik]]
        assert cnt == min(k, len(s))


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 400))
    k = int(rng.integers(1, 60))
    s = rng.integers(-5, 6, size=n).astype(np.float32) * np.float32(0.5)   # many ties
    idx, cnt = O.topk(s, k)
    order = sorted(range(n), key=lambda j: (-float(s[j]), j))[:min(k, n)]
    assert idx[:cnt].tolist() == sorted(order)
    assert (idx[cnt:] == -1).all() and cnt == min(k, n)
    # visibility limit
    nv = n // 2
    idx2, cnt2 = O.topk(s, k, n_visible=nv)
    order2 = sorted(range(nv), key=lambda j: (-float(s[j]), j))[:min(k, nv)]
    assert idx2[:cnt2].tolist() == sorted(order2)


def test_topk_all_equal_and_empty():
    s = np.zeros(100, dtype=np.float32)
    idx, cnt = O.topk(s, 10)
    assert idx.tolist() == list(range(10)) and cnt == 10
    idx, cnt = O.topk(np.zeros(0, dtype=np.float32), 4)
    assert idx.tolist() == [-1] * 4 and cnt == 0


# -------------------------------------------------------------- attention ---

def test_attention_golden_two_entry():
    g = golden("softmax_two_entry.txt")
    # head dim 1 is enough for the closed form
    q = bits_of([float(g["q"][0])]).reshape(1, 1)
    K = bits_of([float(v) for v in g["keys"]]).reshape(2, 1)
    V = bits_of([float(v) for v in g["values"]]).reshape(2, 1)
    out, lse, p = O.attention(q, K, V, [0, 1], math.log(3.0), return_p=True)
    assert np.allclose(p[0], [float(v) for v in g["weights"]], rtol=0, atol=1e-15)
    assert abs(out[0, 0] - float(g["out"][0])) < 1e-12
    assert abs(lse[0] - math.log(4.0)) < 1e-15


def _dense_ref(q, K, V, scale):
    qt = torch.tensor(bf16_value(q))
    Kt = torch.tensor(bf16_value(K))
    Vt = torch.tensor(bf16_value(V))
    z = (qt @ Kt.T) * scale
    return torch.softmax(z, dim=-1) @ Vt, torch.logsumexp(z, dim=-1)


def test_attention_matches_library_softmax_fp64():
    H, d, N = 8, 128, 37
    q = synth.normal_bf16(1, "q", (1, H * d)).reshape(H, d)
    K = synth.normal_bf16(1, "k", (1, N * d)).reshape(N, d)
    V = synth.normal_bf16(1, "v", (1, N * d)).reshape(N, d)
    scale = 1 / math.sqrt(128)
    out, lse, p = O.attention(q, K, V, np.arange(N), scale, return_p=True)
    ref_o, ref_l = _dense_ref(q, K, V, scale)
    assert np.abs(out - ref_o.numpy()).max() < 1e-12
    assert np.abs(lse - ref_l.numpy()).max() < 1e-12
    assert np.abs(p.sum(axis=1) - 1).max() < 1e-12
    # a subset of rows in arbitrary order equals dense attention over that subset
    rows = np.array([30, 2, 17, 5])
    out2, _ = O.attention(q, K, V, rows, scale)
    ref2, _ = _dense_ref(q, K[rows], V[rows], scale)
    assert np.abs(out2 - ref2.numpy()).max() < 1e-12


def test_attention_special_cases():
    H, d = 4, 128
    q = synth.normal_bf16(2, "q", (1, H * d)).reshape(H, d)
    K = synth.normal_bf16(2, "k", (1, 5 * d)).reshape(5, d)
    V = synth.normal_bf16(2, "v", (1, 5 * d)).reshape(5, d)
    out, lse = O.attention(q, K, V, [3], 0.1)
    assert np.array_equal(out, np.tile(bf16_value(V[3]), (H, 1)))
    same = np.tile(K[0], (5, 1))
    out, _ = O.attention(q, same, V, np.arange(5), 0.1)
    assert np.abs(out - bf16_value(V).mean(axis=0)).max() < 1e-12
    out, lse = O.attention(q, K, V, [], 0.1)
    assert not out.any() and np.isneginf(lse).all()


def test_attention_fp8_uses_dequantised_values():
    H, d, N = 2, 128, 70
    q = synth.normal_bf16(3, "q", (1, H * d)).reshape(H, d)
    Kb = synth.normal_bf16(3, "k", (1, N * d)).reshape(N, d)
    Vb = synth.normal_bf16(3, "v", (1, N * d)).reshape(N, d)
    kc, ks = O.fp8_quantize(Kb)
    vc, vs = O.fp8_quantize(Vb)
    out, lse = O.attention(q, kc, vc, np.arange(N), 0.1, ks, vs)
    Kd = O.e4m3_array_to_f64(kc) * np.repeat(ks.astype(np.float64), 64)[:N, None]
    Vd = O.e4m3_array_to_f64(vc) * np.repeat(vs.astype(np.float64), 64)[:N, None]
    z = torch.tensor(bf16_value(q)) @ torch.tensor(Kd).T * 0.1
    ref = torch.softmax(z, -1) @ torch.tensor(Vd)
    assert np.abs(out - ref.numpy()).max() < 1e-12


# ----------------------------------------------------------------- hybrid ---

def _raw(seed, L, d=128, dI=64):
    K = synth.normal_bf16(seed, "k", (1, L * d)).reshape(L, d)
    V = synth.normal_bf16(seed, "v", (1, L * d)).reshape(L, d)
    KI = synth.normal_bf16(seed, "kidx", (1, L * dI)).reshape(L, dI)
    return K, V, KI


def test_hybrid_m1_full_k_is_dense_attention():
    L, H, d = 40, 4, 128
    K, V, KI = _raw(21, L)
    q = synth.normal_bf16(21, "q", (1, H * d)).reshape(H, d)
    qI = synth.normal_bf16(21, "qidx", (1, 64))[0]
    cs = O.CompressedSeq(K, V, KI, m_csa=1, m_hca=1)
    scale = 1 / math.sqrt(128)
    r = O.hybrid_query(cs, q, qI, t=L, k=L + 3, scale=scale)
    ref_o, ref_l = _dense_ref(q, K, V, scale)
    assert r["cnt"] == L and r["idx"][:L].tolist() == list(range(L))
    assert np.abs(r["out_csa"] - ref_o.numpy()).max() < 1e-12
    assert np.abs(r["out_hca"] - ref_o.numpy()).max() < 1e-12
    assert np.abs(r["lse_csa"] - ref_l.numpy()).max() < 1e-12


def test_hybrid_topk_selects_best_indexer_scores():
    L, H, d, k = 64 * 4 + 3, 2, 128, 9
    K, V, KI = _raw(22, L)
    q = synth.normal_bf16(22, "q", (1, H * d)).reshape(H, d)
    qI = synth.normal_bf16(22, "qidx", (1, 64))[0]
    cs = O.CompressedSeq(K, V, KI)
    r = O.hybrid_query(cs, q, qI, t=L, k=k, scale=0.1)
    s = O.index_scores(qI, cs.cidx)
    assert cs.n_csa == 64 and cs.n_hca == 2
    best = sorted(range(64), key=lambda j: (-float(s[j]), j))[:k]
    assert r["idx"].tolist() == sorted(best)
    ref_o, _ = _dense_ref(q, cs.ck[sorted(best)], cs.cv[sorted(best)], 0.1)
    assert np.abs(r["out_csa"] - ref_o.numpy()).max() < 1e-12
    ref_h, _ = _dense_ref(q, cs.hk, cs.hv, 0.1)
    assert np.abs(r["out_hca"] - ref_h.numpy()).max() < 1e-12


def test_prefill_row_equals_decode_at_that_length():
    L, H, d, k = 300, 2, 128, 8
    K, V, KI = _raw(23, L)
    q = synth.normal_bf16(23, "q", (1, H * d)).reshape(H, d)
    qI = synth.normal_bf16(23, "qidx", (1, 64))[0]
    full = O.CompressedSeq(K, V, KI)
    for t in (0, 3, 4, 5, 127, 128, 129, 255, 256, 299):
        causal = O.hybrid_query(full, q, qI, t=t, k=k, scale=0.1)
        part = O.CompressedSeq(K[:t], V[:t], KI[:t])
        dec = O.hybrid_query(part, q, qI, t=t, k=k, scale=0.1)
        assert causal["idx"].tolist() == dec["idx"].tolist()
        assert np.array_equal(causal["out_csa"], dec["out_csa"])
        assert np.array_equal(causal["out_hca"], dec["out_hca"])
        assert causal["cnt"] == min(k, t // 4)
        if t < 4:
            assert not causal["out_csa"].any() and np.isneginf(causal["lse_csa"]).all()


# ------------------------------------------------- sliding-window branch ----

def test_window_rows_are_the_last_tokens_before_the_query():
    assert O.window_rows(10, 100, 4).tolist() == [6, 7, 8, 9]
    assert O.window_rows(3, 100, 8).tolist() == [0, 1, 2]
    assert O.window_rows(50, 20, 8).tolist() == list(range(12, 20))   # only tokens that exist
    assert O.window_rows(0, 100, 8).tolist() == []


def test_union_attention_is_one_softmax_and_the_lse_merge_of_its_parts():
    H, d = 4, 128
    q = synth.normal_bf16(31, "q", (1, H * d)).reshape(H, d)
    Ka, Va = synth.normal_bf16(31, "k", (1, 40 * d)).reshape(40, d), synth.normal_bf16(31, "v", (1, 40 * d)).reshape(40, d)
    Kb, Vb = synth.normal_bf16(32, "k", (1, 25 * d)).reshape(25, d), synth.normal_bf16(32, "v", (1, 25 * d)).reshape(25, d)
    ra, rb = [3, 17, 5, 39], list(range(10, 25))
    scale = 1 / np.sqrt(128.0)
    out, lse = O.union_attention(q, [(Ka, Va, ra), (Kb, Vb, rb)], scale)
    # one softmax over the stacked keys, in numpy fp64
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    Kf = np.concatenate([synth.bf16_bits_to_f32(Ka).astype(np.float64)[ra], synth.bf16_bits_to_f32(Kb).astype(np.float64)[rb]])
    Vf = np.concatenate([synth.bf16_bits_to_f32(Va).astype(np.float64)[ra], synth.bf16_bits_to_f32(Vb).astype(np.float64)[rb]])
    z = qf @ Kf.T * scale
    ref_lse = np.log(np.exp(z - z.max(1, keepdims=True)).sum(1)) + z.max(1)
    p = np.exp(z - ref_lse[:, None])
    np.testing.assert_allclose(out, p @ Vf, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    # the exact merge of the two separate attentions gives the same
    oa, la = O.attention(q, Ka, Va, ra, scale)
    ob, lb = O.attention(q, Kb, Vb, rb, scale)
    m = np.logaddexp(la, lb)
    merged = oa * np.exp(la - m)[:, None] + ob * np.exp(lb - m)[:, None]
    np.testing.assert_allclose(out, merged, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, m, rtol=0, atol=1e-12)


def test_union_attention_of_nothing_is_empty():
    q = np.full((2, 128), 0x3F80, dtype=np.uint16)  # bf16 1.0
    out, lse = O.union_attention(q, [(np.zeros((4, 128), np.uint16), np.zeros((4, 128), np.uint16), [])], 0.1)
    assert not out.any() and np.isneginf(lse).all()
