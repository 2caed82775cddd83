"""Models, on the CPU, of the integer and bit-level schemes two kernels rely
on, checked against the oracle and against plain sorting:

* the FP4 indexer (mxfp4_quantize_kernel, score_decode_mxfp4_kernel and the
  prefill kernel's int8 words, score_prefill_mxfp4_kernel): the
  e2m1 encoder by threshold compares, the E8M0 exponent from the fp32 bit
  pattern, the doubled-magnitude byte table picked by a byte permute, the
  sign applied by selecting +q or -q bytes, dp4a accumulation and the
  per-block exponent offsets, each block term exact in fp64 and one
  rounding of their sum to fp32 -- the model's codes, scales and scores must
  equal the oracle's bit for bit, also for blocks so small that fp32 terms
  would round on their own;
* the context-parallel merge (cp_merge_select_kernel): rank-major candidate
  offsets, the cut "key > T or (key == T and index <= jmax)" at the k-th
  largest, and ordered output by warps over contiguous runs of the list,
  each writing from its exclusive prefix -- the model's global selection and
  per-rank shares must equal sorting.

* the second and third forms of the prefill selection
  (select_prefill_v2_kernel with 32 or 16 warps): the
  first radix digit over all keys, the second and third over the threshold
  bin's keys only (or over all keys when that bin overflows its list), then
  per-warp runs counted and written with the ties at the threshold taken in
  index order -- the model's indices must equal the oracle's top-k.

* the query pairs of the dense prefill kernel (attn_prefill_pair_kernel):
  with m even, positions 2p and 2p + 1 see the same entries under the causal
  rule (c + 1) m <= t, so one tile of rows serves both; and the fourth
  selection form's run split (per-thread contiguous runs, ties taken in
  index order from the runs' exclusive prefixes) equals plain sorting.

The models restate the kernels' schemes in Python; the CUDA kernels
themselves are checked against the oracle by the GPU tests.
"""
from __future__ import annotations

import math
import struct

import numpy as np

from oracle import oracle as O


# -- FP4 indexer ----------------------------------------------------------------

def _f2u(x) -> int:
    return struct.unpack("<I", struct.pack("<f", float(np.float32(x))))[0]


def _u2f(u: int):
    return np.float32(struct.unpack("<f", struct.pack("<I", u & 0xFFFFFFFF))[0])


def _byte_perm(x: int, y: int, s: int) -> int:
    """CUDA __byte_perm: bytes 0-3 from x, 4-7 from y; selector nibble j's
    low three bits pick output byte j."""
    b = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(b[(s >> (4 * j)) & 7] << (8 * j) for j in range(4))


def _dp4a(a: int, b: int, c: int) -> int:
    def s8(v):
        return v - 256 if v >= 128 else v
    return c + sum(s8((a >> (8 * i)) & 0xFF) * s8((b >> (8 * i)) & 0xFF) for i in range(4))


def _e2m1_code(y) -> int:
    y = np.float32(y)
    a = abs(y)
    c = sum(int(v) for v in (a > 0.25, a >= 0.75, a > 1.25, a >= 1.75, a > 2.5, a >= 3.5, a > 5))
    if a != a:
        c = 7
    return c | ((_f2u(y) >> 28) & 8)


def _scale_exp(amax) -> int:
    if not amax > 0:
        return -127
    u = _f2u(amax)
    e = (u >> 23) & 0xFF
    fl = e - 127 if e else ((u & 0x7FFFFF).bit_length() - 1) - 149
    return min(127, max(-127, fl - 2))


def _inv_scale(se: int):
    return _u2f((127 - se) << 23) if 127 - se <= 254 else _u2f(0x00400000)


LUT_LO, LUT_HI = 0x03020100, 0x0C080604  # doubled e2m1 magnitudes 0 1 2 3 | 4 6 8 12


def _bf16(bits) -> np.float32:
    return _u2f(int(bits) << 16)


def _model_quantize_row(row):
    codes, scales = bytearray(32), []
    for blk in range(2):
        w = row[32 * blk:32 * blk + 32]
        amax = max((abs(_bf16(v)) for v in w), default=np.float32(0))
        se = _scale_exp(np.float32(amax))
        inv = _inv_scale(se)
        for i in range(16):
            lo = _e2m1_code(np.float32(_bf16(w[2 * i]) * inv))
            hi = _e2m1_code(np.float32(_bf16(w[2 * i + 1]) * inv))
            codes[16 * blk + i] = lo | (hi << 4)
        scales.append(se + 127)
    return bytes(codes), scales


def _model_query(qbits):
    qp, qn, qe = [0] * 16, [0] * 16, [0, 0]
    vals = [_bf16(b) for b in qbits]
    for blk in range(2):
        se = _scale_exp(np.float32(max(abs(v) for v in vals[32 * blk:32 * blk + 32])))
        inv = _inv_scale(se)
        qe[blk] = se + 127
        for e in range(32 * blk, 32 * blk + 32):
            c = _e2m1_code(np.float32(vals[e] * inv))
            v = (_byte_perm(LUT_LO, LUT_HI, c & 7) & 0xFF) * (-1 if c & 8 else 1)
            qp[e // 4] |= (v & 0xFF) << (8 * (e % 4))
            qn[e // 4] |= ((-v) & 0xFF) << (8 * (e % 4))
    return qp, qn, qe


def _block_dots(codes: bytes, qp, qn):
    """The two exact integer block sums (doubled e2m1 values) of one entry."""
    w = struct.unpack("<8I", codes)

    def dot8(x, a, b, c, d, acc):
        m0 = _byte_perm(LUT_LO, LUT_HI, x & 0x7777)
        s0 = _byte_perm(a, b, 0x3210 | ((x >> 1) & 0x4444))
        m1 = _byte_perm(LUT_LO, LUT_HI, (x >> 16) & 0x7777)
        s1 = _byte_perm(c, d, 0x3210 | ((x >> 17) & 0x4444))
        return _dp4a(m1, s1, _dp4a(m0, s0, acc))
    A = [0, 0]
    for blk in range(2):
        for i in range(4):
            m = 8 * blk + 2 * i
            A[blk] = dot8(w[4 * blk + i], qp[m], qn[m], qp[m + 1], qn[m + 1], A[blk])
    return A


def _model_score(codes: bytes, sc, qp, qn, qe):
    A = _block_dots(codes, qp, qn)
    return _mx_sum(A[0], int(sc[0]) + int(qe[0]) - 254 - 2, A[1], int(sc[1]) + int(qe[1]) - 254 - 2)


def _mx_sum(A0, e0, A1, e1):
    """The kernels' score of two exact block terms, -0 as +0: with both
    exponents in [-149, 114] the terms in fp32 and one fp32 addition;
    otherwise each term in fp64, one fp64 addition, one rounding to fp32."""
    with np.errstate(over="ignore"):
        if min(e0, e1) >= -149 and max(e0, e1) <= 114:
            s = np.float32(np.float32(math.ldexp(A0, e0)) + np.float32(math.ldexp(A1, e1)))
        else:
            s = np.float32(math.ldexp(A0, e0) + math.ldexp(A1, e1))
    return np.float32(0) if s == 0 else s


def _mx_sum_fp32_terms(A0, e0, A1, e1):
    """A plausible mistake: each term rounded to fp32 first, whatever e (inexact
    once e < -149)."""
    with np.errstate(over="ignore"):
        s = np.float32(np.float32(math.ldexp(A0, e0)) + np.float32(math.ldexp(A1, e1)))
    return np.float32(0) if s == 0 else s


def test_fp4_kernel_scheme_matches_the_oracle_bit_for_bit():
    rng = np.random.default_rng(3)
    n = 300
    x = rng.standard_normal((n, 64)).astype(np.float32)
    x[5] *= 1e-30
    x[6] *= 1e30
    x[7, :32] = 0
    x[8, 3] = -0.0
    x[9, :8] = [4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -0.25]
    x[10, :4] = [6.0, 5.0, -5.0, 7.0]
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    oc, osc = O.mxfp4_quantize(xb)
    for j in range(n):
        c, s = _model_quantize_row(xb[j])
        assert c == bytes(oc[j]) and s == [int(v) for v in osc[j]], j
    qb = (rng.standard_normal(64).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qp, qn, qe = _model_query(qb)
    qc, qs = O.mxfp4_quantize(qb.reshape(1, -1))
    assert qe == [int(v) for v in qs[0]]
    ref = O.mxfp4_index_scores(qc[0], qs[0], oc, osc)
    for j in range(n):
        got = _model_score(bytes(oc[j]), [int(v) for v in osc[j]], qp, qn, qe)
        assert _f2u(got) == _f2u(ref[j]), j


# -- context-parallel merge -----------------------------------------------------

def _select_rank(keys, idx, R):
    """The cut's contract: exactly R entries satisfy key > T or (key == T and
    idx <= jmax)."""
    order = sorted(range(len(keys)), key=lambda p: (-int(keys[p]), int(idx[p])))
    T = int(keys[order[R - 1]])
    ties = sorted(int(idx[q]) for q in range(len(keys)) if keys[q] == T)
    rem = R - sum(1 for q in range(len(keys)) if keys[q] > T)
    return T, (0x7FFFFFFF if rem >= len(ties) else ties[rem - 1])


def _model_merge(keys, gidx, gcnt, W, k, rank, base, nw=32):
    off = [0]
    for w in range(W):
        off.append(off[-1] + gcnt[w])
    C = off[W]
    lk, li = [], []
    for p in range(C):
        w = 0
        while off[w + 1] <= p:
            w += 1
        lk.append(keys[w][p - off[w]])
        li.append(gidx[w][p - off[w]])
    R = min(C, k)
    every = C <= k
    T, jmax = (0, 0x7FFFFFFF) if every else _select_rank(lk, li, R)
    win = [every or lk[p] > T or (lk[p] == T and li[p] <= jmax) for p in range(C)]
    mine = [win[p] and off[rank] <= p < off[rank + 1] for p in range(C)]
    # every warp: one contiguous run of whole 32-entry groups, counted, then
    # written from its exclusive prefix
    run = ((C + 31) // 32 + 31) & ~31
    runs = [(w * run, min(C, w * run + run)) for w in range(nw)]
    nwin = [sum(win[lo:hi]) for lo, hi in runs]
    nmine = [sum(mine[lo:hi]) for lo, hi in runs]
    sel, loc = [-1] * k, [-1] * k
    gpos = lpos = 0
    for w, (lo, hi) in enumerate(runs):
        gpos, lpos = sum(nwin[:w]), sum(nmine[:w])
        for p0 in range(lo, hi, 32):
            grp = range(p0, min(p0 + 32, hi))
            for i, p in enumerate(grp):
                if win[p]:
                    sel[gpos + sum(win[p0:p0 + i])] = li[p]
                if mine[p]:
                    loc[lpos + sum(mine[p0:p0 + i])] = li[p] - base
            gpos += sum(win[p0:p0 + len(grp)])
            lpos += sum(mine[p0:p0 + len(grp)])
    return sel, R, loc, lpos


def test_context_parallel_merge_scheme_matches_sorting():
    rng = np.random.default_rng(0)
    for trial in range(150):
        W, k = int(rng.integers(1, 6)), int(rng.integers(1, 600))
        sizes = [int(rng.integers(0, 1300)) for _ in range(W)]
        bases = np.cumsum([0] + sizes[:-1])
        nvals = int(rng.integers(1, 50))  # few distinct scores: ties at the cut are common
        scores = [rng.integers(0, nvals, sz).astype(np.int64) + 0x80000000 for sz in sizes]
        keys, gidx, gcnt = [], [], []
        for w in range(W):
            s = scores[w]
            loc = sorted(sorted(range(len(s)), key=lambda j: (-int(s[j]), j))[:k])
            keys.append([int(s[j]) for j in loc])
            gidx.append([int(bases[w] + j) for j in loc])
            gcnt.append(len(loc))
        full = np.concatenate(scores) if sum(sizes) else np.zeros(0, np.int64)
        want = sorted(sorted(range(len(full)), key=lambda j: (-int(full[j]), j))[:k])
        for rank in range(W):
            sel, R, loc, lc = _model_merge(keys, gidx, gcnt, W, k, rank, int(bases[rank]))
            assert R == len(want) and sel[:R] == want and all(v == -1 for v in sel[R:]), trial
            mine = [j - int(bases[rank]) for j in want if bases[rank] <= j < bases[rank] + sizes[rank]]
            assert loc[:lc] == mine and all(v == -1 for v in loc[lc:]), trial


def test_fp4_prefill_word_scheme_matches_the_oracle():
    """The prefill kernel widens codes to doubled signed int8 (four to a word,
    word w holding elements 32*(w//8) + 4*(w%8) ..) for queries and keys alike,
    sums each block with dp4a and combines the blocks with their exponents."""
    rng = np.random.default_rng(8)
    keys = (rng.standard_normal((64, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qbits = (rng.standard_normal((5, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kc, ks = O.mxfp4_quantize(keys)
    qc, qs = O.mxfp4_quantize(qbits)

    def s8(code):  # doubled signed value as a byte
        m = _byte_perm(LUT_LO, LUT_HI, code & 7) & 0xFF
        return (-m if code & 8 else m) & 0xFF

    def words_from_codes(row_codes):  # 32 code bytes -> 16 words of 4 bytes
        out = []
        for half in range(2):
            cw = struct.unpack("<4I", bytes(row_codes[16 * half:16 * half + 16]))
            for i in range(4):
                lo = sum(s8((cw[i] >> (4 * j)) & 0xF) << (8 * j) for j in range(4))
                hi = sum(s8((cw[i] >> (4 * (j + 4))) & 0xF) << (8 * j) for j in range(4))
                out += [lo, hi]
        return out
    for qi in range(5):
        qw = words_from_codes(qc[qi])
        ref = O.mxfp4_index_scores(qc[qi], qs[qi], kc, ks)
        for e in range(64):
            kw = words_from_codes(kc[e])
            A = [0, 0]
            for w in range(16):
                A[w // 8] = _dp4a(qw[w], kw[w], A[w // 8])
            s = _mx_sum(A[0], int(qs[qi][0]) + int(ks[e][0]) - 256, A[1], int(qs[qi][1]) + int(ks[e][1]) - 256)
            assert _f2u(s) == _f2u(ref[e]), (qi, e)


# -- prefill selection, second form ---------------------------------------------

def _order_key(s: np.ndarray) -> np.ndarray:
    """The kernels' 32-bit order key of an fp32 score: -0 as +0, then the
    sign-magnitude bits mapped so that unsigned order is numeric order."""
    u = np.ascontiguousarray(s, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    neg = (u >> 31) == 1
    return np.where(neg, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def _find_desc(h, K):
    """The digit d with above(d) < K <= above(d) + h[d], above(d) = the keys in
    the bins above d."""
    above = 0
    for d in range(len(h) - 1, -1, -1):
        if above < K <= above + int(h[d]):
            return d, above
        above += int(h[d])
    raise AssertionError("inconsistent histogram")


def _model_select2(keys, k, list_cap=8192, nw=32):
    nv = len(keys)
    if nv <= k:
        return list(range(nv)) + [-1] * (k - nv), nv
    h1 = np.bincount(keys >> 21, minlength=2048)
    d1, above = _find_desc(h1, k)
    K1 = k - above
    dk = keys[(keys >> 21) == d1] if h1[d1] <= list_cap else keys  # the list, or every key in place
    h2 = np.bincount(((dk >> 10) & 2047)[(dk >> 21) == d1], minlength=2048)
    d2, above = _find_desc(h2, K1)
    K2 = K1 - above
    pre = (d1 << 11) | d2
    h3 = np.bincount((dk & 1023)[(dk >> 10) == pre], minlength=1024)
    d3, above = _find_desc(h3, K2)
    r = K2 - above
    T = np.uint32((pre << 10) | d3)
    run = ((nv + nw - 1) // nw + 31) & ~31  # keys per warp, whole 32-key groups
    runs = [(w * run, min(nv, w * run + run)) for w in range(nw)]
    ngt = [int((keys[lo:hi] > T).sum()) if hi > lo else 0 for lo, hi in runs]
    neq = [int((keys[lo:hi] == T).sum()) if hi > lo else 0 for lo, hi in runs]
    out = [-1] * k
    pos = 0
    for w, (lo, hi) in enumerate(runs):
        pos = sum(ngt[:w]) + min(sum(neq[:w]), r)
        eq_run = sum(neq[:w])
        for j0 in range(lo, hi, 32):
            js = np.arange(j0, min(j0 + 32, hi))
            g, e = keys[js] > T, keys[js] == T
            erank = eq_run + np.cumsum(e) - e  # ties before each lane
            sel = g | (e & (erank < r))
            p = pos + np.cumsum(sel) - sel
            for j, sl, pp in zip(js, sel, p):
                if sl:
                    assert pp < k
                    out[int(pp)] = int(j)
            pos += int(sel.sum())
            eq_run += int(e.sum())
    assert pos == k  # the last warp ends at the total
    return out, k


def test_prefill_select_v2_scheme_matches_the_oracle():
    rng = np.random.default_rng(11)
    cases = []
    for _ in range(25):  # continuous scores
        nv = int(rng.integers(1, 60000))
        cases.append((rng.normal(0, 8, nv).astype(np.float32), int(rng.integers(1, 5000))))
    for _ in range(15):  # few distinct values: ties at the threshold, overflowing bins
        nv = int(rng.integers(1000, 60000))
        vals = rng.normal(0, 8, int(rng.integers(1, 6))).astype(np.float32)
        cases.append((vals[rng.integers(0, len(vals), nv)], int(rng.integers(1, nv))))
    z = np.zeros(20000, np.float32)
    z[::3] = -0.0
    cases += [(np.full(30000, 1.5, np.float32), 2048),      # all equal: one bin of 30,000 keys
              (z, 777),                                     # +0 and -0 tie
              (np.linspace(-4, 4, 45000).astype(np.float32), 40000)]
    for i, (s, k) in enumerate(cases):
        want, wc = O.topk(s, k)
        for nw in (32, 16):  # 1024-thread (second form) and 512-thread (third form) CTAs
            got, gc = _model_select2(_order_key(s), k, nw=nw)
            assert gc == wc and got == list(want), (i, nw)


def test_fp4_scores_of_tiny_blocks_stay_exact():
    # query and keys both scaled far down: the block terms fall below fp32's
    # subnormal grid (e < -149) and the sum lands among fp32 subnormals.  The
    # kernels' fp64 terms give the oracle's single rounding; fp32 terms
    # (the plausible mistake) round each term first and miss some.
    rng = np.random.default_rng(7)
    n = 400
    x = rng.standard_normal((n, 64)).astype(np.float32) * np.float32(2.0 ** -68)
    x[:, :32] *= np.float32(2.0 ** -10)  # both blocks' terms below 2^-149 (e about -151 and -155)
    x[:, 32:] *= np.float32(2.0 ** -14)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    kc, ks = O.mxfp4_quantize(xb)
    q = rng.standard_normal(64).astype(np.float32) * np.float32(2.0 ** -68)
    qb = (q.view(np.uint32) >> 16).astype(np.uint16)
    qp, qn, qe = _model_query(qb)
    qc, qs = O.mxfp4_quantize(qb.reshape(1, -1))
    ref = O.mxfp4_index_scores(qc[0], qs[0], kc, ks)
    assert (ref != 0).sum() > n // 2 and (np.abs(ref) < np.finfo(np.float32).tiny).all()  # subnormal scores
    misses = 0
    for j in range(n):
        got = _model_score(bytes(kc[j]), [int(v) for v in ks[j]], qp, qn, qe)
        assert _f2u(got) == _f2u(ref[j]), j
        A = _block_dots(bytes(kc[j]), qp, qn)  # the same row through fp32 terms
        e = [int(ks[j][b]) + int(qe[b]) - 256 for b in range(2)]
        misses += _f2u(_mx_sum_fp32_terms(A[0], e[0], A[1], e[1])) != _f2u(ref[j])
    assert misses > n // 10  # the case tells the two schemes apart


def test_fp4_scores_of_huge_blocks_match_the_oracle():
    # large scales: the block terms leave fp32's range (e > 114), the fp64
    # routine takes over, and scores that overflow fp32 are +-inf as in the
    # oracle's single rounding
    rng = np.random.default_rng(8)
    n = 300
    x = rng.standard_normal((n, 64)).astype(np.float32) * np.float32(2.0 ** 100)
    x[: n // 2, 32:] *= np.float32(2.0 ** 14)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    kc, ks = O.mxfp4_quantize(xb)
    q = rng.standard_normal(64).astype(np.float32) * np.float32(2.0 ** 12)
    qb = (q.view(np.uint32) >> 16).astype(np.uint16)
    qp, qn, qe = _model_query(qb)
    qc, qs = O.mxfp4_quantize(qb.reshape(1, -1))
    ref = O.mxfp4_index_scores(qc[0], qs[0], kc, ks)
    assert np.isinf(ref).sum() > 0 and np.isfinite(ref).sum() > 0
    slow = 0
    for j in range(n):
        got = _model_score(bytes(kc[j]), [int(v) for v in ks[j]], qp, qn, qe)
        assert _f2u(got) == _f2u(ref[j]), j
        slow += max(int(ks[j][b]) + int(qe[b]) - 256 for b in range(2)) > 114
    assert slow > n // 4  # the fp64 routine's range is exercised


def test_query_pairs_see_the_same_entries():
    # entry c is visible at position t iff (c + 1) * m <= t, i.e. the count is t // m
    for m in (2, 4, 8, 128, 1024):
        for t0 in range(0, 4 * m + 7, 2):
            assert t0 // m == (t0 + 1) // m, (m, t0)
    # an odd m breaks it (the kernel takes the pair path only for even m)
    assert any(t0 // 3 != (t0 + 1) // 3 for t0 in range(0, 12, 2))


def _runs_select(keys, k, threads):
    """The fourth selection form's output stage: T = the k-th largest key;
    per thread, a contiguous run of keys; counts of keys above and equal to
    T per run; exclusive prefixes; each run writes its keys above T and its
    share of the ties (lowest indices first) from its prefix."""
    n = len(keys)
    T = sorted(keys, reverse=True)[k - 1]
    per = (n + threads - 1) // threads
    runs = [(min(n, t * per), min(n, t * per + per)) for t in range(threads)]
    above = [sum(1 for j in range(a, b) if keys[j] > T) for a, b in runs]
    ties = [sum(1 for j in range(a, b) if keys[j] == T) for a, b in runs]
    tot_a = sum(above)
    take = k - tot_a
    out = [None] * k
    pa = pt = 0
    for (a, b), na, nt in zip(runs, above, ties):
        o = pa + min(pt, take)
        tb = pt
        for j in range(a, b):
            sel = keys[j] > T
            if keys[j] == T:
                sel = tb < take
                tb += 1
            if sel:
                out[o] = j
                o += 1
        pa += na
        pt += nt
    return out


def test_prefill_select_v4_runs_match_sorting():
    rng = np.random.default_rng(41)
    for n, k, threads, levels in ((5000, 300, 512, 40), (2049, 2048, 512, 3), (700, 1, 64, 5), (3000, 2999, 512, 1)):
        keys = rng.integers(0, levels, size=n).tolist()   # heavy ties
        got = _runs_select(keys, k, threads)
        order = sorted(range(n), key=lambda j: (-keys[j], j))[:k]
        assert got == sorted(order), (n, k, threads)
