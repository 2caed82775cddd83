"""Pins of the oracle's low-precision storage on the CSA path: the FP4 indexer
(MXFP4: e2m1 elements, blocks of 32, E8M0 power-of-two scales) and mixed KV
storage (rotary dims of K in bf16, the rest and V in e4m3), "DeepSeek-V4 ...
Review", section 3-2 (2) component table ("Mixed KV storage") and section 3-2
(4) (FP4 on the CSA indexer QK path).

Each check rests on something other than the oracle's own code: the e2m1
value table of the format definition, a brute-force nearest-value search,
exact rational arithmetic (``fractions``) with an exact round-to-fp32, and
reductions to the already pinned bf16 / e4m3 functions.
"""
from __future__ import annotations

from fractions import Fraction
from math import floor

import numpy as np
import pytest

from oracle import oracle as O

# The eight e2m1 magnitudes of the OCP Microscaling FP4 (E2M1) format, by code.
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values that are exact in bf16 -> their bf16 bit patterns."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert not (b & 0xFFFF).any(), "test values must be exact in bf16"
    return (b >> 16).astype(np.uint16)


def _brute_e2m1(y: float) -> int:
    """Nearest e2m1 code by search over all magnitudes; ties to the code with
    an even fraction bit; beyond the largest magnitude, the largest."""
    a = abs(y)
    best = min(range(8), key=lambda c: (abs(E2M1_MAGNITUDES[c] - a), c & 1))
    if a > 6.0:
        best = 7
    return best | (8 if np.signbit(y) else 0)


def _fp32_rne(fr: Fraction) -> float:
    """Round an exact rational to the nearest fp32, ties to even (normal and
    subnormal range), without going through any float arithmetic."""
    if fr == 0:
        return 0.0
    neg = fr < 0
    a = -fr if neg else fr
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    f = floor(n)
    rem = n - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    v = f * quantum
    assert v < Fraction(2) ** 128
    out = float(v)  # v has at most 24 significant bits: exact in fp64
    return -out if neg else out


# -- e2m1 and E8M0 codecs ------------------------------------------------------

def test_e2m1_decode_table():
    for c in range(16):
        want = E2M1_MAGNITUDES[c & 7] * (-1.0 if c & 8 else 1.0)
        got = O.e2m1_to_double(c)
        assert got == want and np.signbit(got) == bool(c & 8), c


def test_e2m1_encode_is_the_nearest_value_ties_to_even():
    mags = sorted(set(E2M1_MAGNITUDES))
    probes = set(mags)
    for a, b in zip(mags, mags[1:]):
        mid = (a + b) / 2
        probes |= {mid, np.nextafter(mid, 0), np.nextafter(mid, 10), (a + mid) / 2, (mid + b) / 2}
    probes |= {6.5, 7.0, 7.99, 8.0, 1e3, 1e-30, 0.2499, 0.2501}
    for a in sorted(probes):
        for x in (a, -a):
            assert O.e2m1_from_double(x) == _brute_e2m1(x), x
    # named ties: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4, 7 -> 6
    for x, want in [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (7.0, 7)]:
        assert O.e2m1_from_double(x) == want, x
    assert O.e2m1_from_double(float("inf")) == 7 and O.e2m1_from_double(float("-inf")) == 15
    rng = np.random.default_rng(5)
    for x in rng.uniform(-9, 9, 2000):
        assert O.e2m1_from_double(float(x)) == _brute_e2m1(float(x)), x


def test_e8m0_decode():
    for c in (0, 1, 100, 126, 127, 128, 200, 254):
        assert O.e8m0_to_double(c) == 2.0 ** (c - 127)
    assert np.isnan(O.e8m0_to_double(255))


# -- MXFP4 quantization ----------------------------------------------------------

def test_mxfp4_quantize_hand_cases():
    # a block of ones: amax 1 -> X = 2^(0 - 2) = 1/4, every element 4 (code 6)
    x = np.zeros((3, 64), np.float32)
    x[0, :32] = 1.0
    # second block: amax 6 -> X = 1, 6 -> code 7, 3 -> 5, -0.5 -> 9
    x[0, 32], x[0, 33], x[0, 34] = 6.0, 3.0, -0.5
    # row 1: amax 7 -> X = 1 (floor(log2 7) = 2), 7 saturates to 6 (code 7)
    x[1, 0], x[1, 1] = 7.0, -7.0
    # row 2 stays all zero: scale code 0, codes 0
    codes, scales = O.mxfp4_quantize(_bf16_bits(x))
    assert scales[0].tolist() == [125, 127] and scales[1].tolist() == [127, 0] and scales[2].tolist() == [0, 0]
    assert (codes[0, :16] == 0x66).all()
    assert codes[0, 16] == (7 | (5 << 4))          # element 32 low nibble, 33 high nibble
    assert codes[0, 17] == 9                        # element 34 = -0.5, element 35 = +0
    assert codes[1, 0] == (7 | (15 << 4))
    assert not codes[2].any()


def test_mxfp4_quantize_scale_rule_and_elements_by_brute_force():
    rng = np.random.default_rng(11)
    xf = rng.standard_normal((200, 64)).astype(np.float32)
    xf[17] *= 1e-20                   # tiny magnitudes
    xf[18] *= 3e4                     # large magnitudes
    xf[19, :32] = 0.0                 # one empty block
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = O.mxfp4_quantize(xb)
    xd = O.bf16_array_to_f64(xb)
    for j in range(xd.shape[0]):
        for b in range(2):
            blk = xd[j, 32 * b:32 * b + 32]
            amax = np.abs(blk).max()
            X = 2.0 ** (int(scales[j, b]) - 127)
            if amax == 0:
                assert scales[j, b] == 0
            else:
                assert 4.0 <= amax / X < 8.0, (j, b)
            for i in range(32):
                e = 32 * b + i
                c = (codes[j, e // 2] >> (4 * (e % 2))) & 0xF
                assert c == _brute_e2m1(blk[i] / X), (j, e)


def test_mxfp4_dequantization_error_bound():
    rng = np.random.default_rng(12)
    xf = rng.standard_normal((300, 64)).astype(np.float32)
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = O.mxfp4_quantize(xb)
    xd = O.bf16_array_to_f64(xb)
    xq = O.mxfp4_to_f64(codes, scales)
    X = np.repeat(2.0 ** (scales.astype(np.int64) - 127), 32, axis=1)
    y = np.abs(xd) / X
    err = np.abs(xd - xq) / X
    # half the spacing of each binade: 0.25 below 2, 0.5 in [2, 4), 1 in [4, 6];
    # above 6 the clamp loses less than 2
    bound = np.where(y < 2, 0.25, np.where(y < 4, 0.5, np.where(y <= 6, 1.0, 2.0)))
    assert (err <= bound + 1e-15).all()


# -- FP4 index scores ------------------------------------------------------------

def _exact_score(qc, qs, kc, ks):
    total = Fraction(0)
    for b in range(len(qs)):
        blk = Fraction(0)
        for i in range(32 * b, 32 * b + 32):
            qv = Fraction(O.e2m1_to_double((int(qc[i // 2]) >> (4 * (i % 2))) & 0xF))
            kv = Fraction(O.e2m1_to_double((int(kc[i // 2]) >> (4 * (i % 2))) & 0xF))
            blk += qv * kv
        total += blk * Fraction(2) ** (int(qs[b]) - 127) * Fraction(2) ** (int(ks[b]) - 127)
    return total


def test_mxfp4_scores_are_the_correctly_rounded_exact_sum():
    rng = np.random.default_rng(21)
    n = 60
    kc = rng.integers(0, 256, (n, 32), dtype=np.uint8)
    ks = rng.integers(110, 140, (n, 2), dtype=np.uint8)
    # scale spreads well past fp32's 24 bits (so rounding happens) and past
    # 40 bits (the dominant-term case), in both directions
    ks[0] = [127, 127 - 30]
    ks[1] = [127 - 45, 127]
    ks[2] = [127, 127 - 60]
    ks[3] = [127 - 20, 127]
    qc = rng.integers(0, 256, 32, dtype=np.uint8)
    qs = np.array([127, 126], dtype=np.uint8)
    s = O.mxfp4_index_scores(qc, qs, kc, ks)
    rounded = 0
    for j in range(n):
        ex = _exact_score(qc, qs, kc[j], ks[j])
        want = _fp32_rne(ex)
        assert s[j] == np.float32(want), (j, float(ex), s[j], want)
        rounded += Fraction(float(np.float32(want))) != ex
    assert rounded >= 2  # some cases really needed rounding


def test_mxfp4_score_invariants():
    rng = np.random.default_rng(22)
    xb = (rng.standard_normal((500, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kc, ks = O.mxfp4_quantize(xb)
    qb = (rng.standard_normal((1, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qc, qs = O.mxfp4_quantize(qb)
    s = O.mxfp4_index_scores(qc[0], qs[0], kc, ks)
    # flipping every sign bit of the query negates every score
    neg = O.mxfp4_index_scores(qc[0] ^ 0x88, qs[0], kc, ks)
    assert np.array_equal(neg, np.where(s == 0, s, -s))
    # doubling both query scales doubles every score exactly
    dbl = O.mxfp4_index_scores(qc[0], qs[0] + 1, kc, ks)
    assert np.array_equal(dbl, 2 * s)
    # against the dequantized values in plain fp64 (exact here: small spreads)
    ref = (O.mxfp4_to_f64(kc, ks) @ O.mxfp4_to_f64(qc, qs)[0]).astype(np.float32)
    assert np.array_equal(s, ref + 0)


def test_fp4_topk_composition():
    rng = np.random.default_rng(23)
    L, k = 4000, 100
    K = (rng.standard_normal((L, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    V = (rng.standard_normal((L, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    KI = (rng.standard_normal((L, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q = (rng.standard_normal((8, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qI = (rng.standard_normal(64).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    r = O.lowp_query(K, V, KI, q, qI, t=L - 2, k=k, scale=128 ** -0.5)
    n_vis = (L - 2) // 4
    assert r["scores"].shape == (n_vis,) and r["cnt"] == k
    # the selection is the k largest (score, -index), ascending, by plain sorting
    order = sorted(range(n_vis), key=lambda j: (-float(r["scores"][j]), j))[:k]
    assert r["idx"][:k].tolist() == sorted(order)
    # FP4 scores tie often: ties at the threshold must go to the lower index
    thr = min(float(r["scores"][j]) for j in order)
    tied = [j for j in range(n_vis) if float(r["scores"][j]) == thr]
    chosen = [j for j in tied if j in set(order)]
    assert chosen == tied[:len(chosen)]


# -- mixed KV storage ------------------------------------------------------------

def test_mixed_quantize_reduces_to_bf16_and_e4m3_parts():
    rng = np.random.default_rng(31)
    xc = (rng.standard_normal((150, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    codes, scales, rope = O.mixed_quantize(xc, 64)
    assert np.array_equal(rope, xc[:, 64:])
    c8, s8 = O.fp8_quantize(np.ascontiguousarray(xc[:, :64]))
    assert np.array_equal(codes, c8) and np.array_equal(scales, s8)
    # the scale covers the stored-e4m3 dims only
    xd = O.bf16_array_to_f64(xc[:, :64])
    for g in range(3):
        assert scales[g] == np.float32(np.abs(xd[64 * g:64 * g + 64]).max() / 448.0)


def test_attention_kv_reductions_and_brute_force():
    rng = np.random.default_rng(32)
    N, H, d = 300, 4, 128
    K = (rng.standard_normal((N, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    V = (rng.standard_normal((N, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q = (rng.standard_normal((H, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    rows = rng.choice(N, 77, replace=False).astype(np.int32)
    sc = 128 ** -0.5
    # all-bf16 and all-e4m3 storage give the pinned attention exactly
    o0, l0 = O.attention(q, K, V, rows, sc)
    o1, l1 = O.attention_kv(q, {"mode": "bf16", "data": K}, {"mode": "bf16", "data": V}, rows, sc)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    kc8, ks8 = O.fp8_quantize(K)
    vc8, vs8 = O.fp8_quantize(V)
    o0, l0 = O.attention(q, kc8, vc8, rows, sc, k_scales=ks8, v_scales=vs8)
    o1, l1 = O.attention_kv(q, {"mode": "fp8", "data": kc8, "scales": ks8},
                            {"mode": "fp8", "data": vc8, "scales": vs8}, rows, sc)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    # mixed with no rotary dims is e4m3 storage; with all dims rotary, bf16
    c, s, r = O.mixed_quantize(K, 0)
    o2, _ = O.attention_kv(q, {"mode": "mixed", "data": c, "scales": s, "rope": r},
                           {"mode": "fp8", "data": vc8, "scales": vs8}, rows, sc, d_rope=0)
    assert np.array_equal(o2, o0)
    c, s, r = O.mixed_quantize(K, 128)
    o3, _ = O.attention_kv(q, {"mode": "mixed", "data": c, "scales": s, "rope": r},
                           {"mode": "bf16", "data": V}, rows, sc, d_rope=128)
    o4, _ = O.attention(q, K, V, rows, sc)
    assert np.array_equal(o3, o4)
    # the 64/64 split against a numpy softmax over hand-dequantized rows
    c, s, r = O.mixed_quantize(K, 64)
    om, lm = O.attention_kv(q, {"mode": "mixed", "data": c, "scales": s, "rope": r},
                            {"mode": "fp8", "data": vc8, "scales": vs8}, rows, sc, d_rope=64)
    Kd = np.concatenate([O.e4m3_array_to_f64(c) * np.repeat(s, 64)[:N, None], O.bf16_array_to_f64(r)], axis=1)
    Vd = O.e4m3_array_to_f64(vc8) * np.repeat(vs8, 64)[:N, None]
    z = O.bf16_array_to_f64(q) @ Kd[rows].T * sc
    zm = z.max(axis=1, keepdims=True)
    p = np.exp(z - zm)
    ref = (p / p.sum(axis=1, keepdims=True)) @ Vd[rows]
    assert np.abs(om - ref).max() < 1e-12
    assert np.abs(lm - (zm[:, 0] + np.log(p.sum(axis=1)))).max() < 1e-12


def test_empty_selection_in_mixed_storage():
    q = np.zeros((2, 128), np.uint16)
    c, s, r = O.mixed_quantize(np.zeros((0, 128), np.uint16), 64)
    o, l = O.attention_kv(q, {"mode": "mixed", "data": np.zeros((1, 64), np.uint8), "scales": np.ones(1, np.float32),
                              "rope": np.zeros((1, 64), np.uint16)},
                          {"mode": "fp8", "data": np.zeros((1, 128), np.uint8), "scales": np.ones(1, np.float32)},
                          [], 0.1)
    assert not o.any() and np.isneginf(l).all()


@pytest.mark.parametrize("mistake", ["high_nibble_first", "scale_off_by_one"])
def test_planted_mistakes_are_caught(mistake):
    """A plausible slip in the MXFP4 layout or scale rule breaks the pins: the
    same checks, applied to a deliberately wrong copy of the oracle's output."""
    rng = np.random.default_rng(41)
    xb = (rng.standard_normal((20, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = O.mxfp4_quantize(xb)
    if mistake == "high_nibble_first":
        codes = ((codes >> 4) | (codes << 4)).astype(np.uint8)
    else:
        scales = (scales + 1).astype(np.uint8)
    xd = O.bf16_array_to_f64(xb)
    bad = 0
    for j in range(20):
        for e in range(64):
            X = 2.0 ** (int(scales[j, e // 32]) - 127)
            c = (codes[j, e // 2] >> (4 * (e % 2))) & 0xF
            bad += c != _brute_e2m1(xd[j, e] / X)
    assert bad > 0


def test_hybrid_query_mxfp4_composition():
    """The FP4 hybrid query is the pinned pieces composed: its HCA half is the
    bf16 hybrid query's (HCA has no indexer), its CSA half the attention over
    the top-k of the FP4 scores."""
    rng = np.random.default_rng(51)
    L, k, H = 3000, 64, 4

    def bits(shape):
        return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    K, V, KI, q, qI = bits((L, 128)), bits((L, 128)), bits((L, 64)), bits((H, 128)), bits(64)
    cs = O.CompressedSeq(K, V, KI)
    sc = 128 ** -0.5
    r4 = O.hybrid_query_mxfp4(cs, q, qI, t=L - 1, k=k, scale=sc)
    r16 = O.hybrid_query(cs, q, qI, t=L - 1, k=k, scale=sc)
    assert np.array_equal(r4["out_hca"], r16["out_hca"]) and np.array_equal(r4["lse_hca"], r16["lse_hca"])
    kc, ks = O.mxfp4_quantize(cs.cidx)
    qc, qs = O.mxfp4_quantize(qI.reshape(1, -1))
    n_vis = (L - 1) // 4
    idx, cnt = O.topk(O.mxfp4_index_scores(qc[0], qs[0], kc[:n_vis], ks[:n_vis]), k)
    assert cnt == r4["cnt"] == k and np.array_equal(idx, r4["idx"])
    o, lse = O.attention(q, cs.ck, cs.cv, idx, sc)
    assert np.array_equal(o, r4["out_csa"]) and np.array_equal(lse, r4["lse_csa"])
    assert len(set(idx.tolist()) & set(r16["idx"].tolist())) > k // 2  # FP4 keeps most of the bf16 selection


def test_hybrid_query_mxfp4_without_visible_entries():
    """A query before the first complete block sees nothing: count 0, -1
    padding, zero outputs and lse -inf in both branches (as the bf16 path)."""
    rng = np.random.default_rng(52)

    def bits(shape):
        return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    cs = O.CompressedSeq(bits((600, 128)), bits((600, 128)), bits((600, 64)))
    q, qI = bits((4, 128)), bits(64)
    for t in (0, 1, 3):
        r = O.hybrid_query_mxfp4(cs, q, qI, t=t, k=16, scale=0.1)
        assert r["cnt"] == 0 and (r["idx"] == -1).all()
        assert not r["out_csa"].any() and np.isneginf(r["lse_csa"]).all()
        assert not r["out_hca"].any() and np.isneginf(r["lse_hca"]).all()
    r = O.hybrid_query_mxfp4(cs, q, qI, t=4, k=16, scale=0.1)  # the first entry becomes visible
    assert r["cnt"] == 1 and r["idx"][0] == 0
