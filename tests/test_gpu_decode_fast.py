"""The fast hybrid decode path (SA_OPT_DECODE_FAST) against the fp64 oracle.

The indexer and top-k of hybrid_attn_decode run three kernels on this path:
a sampled bound on the k-th score, the indexer scan keeping the entries
above it as candidates, and one CTA per sequence selecting exactly from them.
Mode 0 (the default) is the general path; mode 1 the fast path; mode 2 the
fast path with the selection forced over every score (the fallback the kernel
takes when the candidates cannot prove the selection).  Indices and counts: bit-exact against the oracle in every
mode.  Outputs: max-abs <= 1e-2 and rms(err)/rms(oracle) <= 1e-2 (bf16
cache), lse within 1e-3.  Cases cover the sampling regime (more than 8192
entries), k up to 2048, fewer than k entries, empty and 1-entry sequences,
exact ties and near-ties below the screen's resolution, every score equal (a
band far larger than shared memory), and a score pattern that defeats the
sample (the bound leaves fewer than k candidates).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import (SCALE, TOL_BF16, TOL_FP8, TOL_REL, TOL_REL_FP8, Inputs, bf16_to_f64, compress_on_gpu,
                         out_errors)

pytestmark = pytest.mark.gpu

MODES = [1, 2]


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    yield S
    S.set_option(S.SA_OPT_DECODE_FAST, 0)


def _run(S, inp, k, mode, H=None, fp8=False):
    B, Lcap = inp.B, inp.Lcap
    H = inp.H if H is None else H
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap, fp8=fp8)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty(B, H, dtype=torch.float32, device="cuda")
    S.set_option(S.SA_OPT_DECODE_FAST, mode)
    try:
        oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, lse_hca=lh,
                                      idx_out=idx, cnt_out=cnt)
        S.read_device_status()
    finally:
        S.set_option(S.SA_OPT_DECODE_FAST, 0)
    return oc, oh, lc, lh, idx, cnt


def _check(S, inp, k, mode, outputs=True, fp8=False):
    oc, oh, lc, lh, idx, cnt = _run(S, inp, k, mode, fp8=fp8)
    tol, trel = (TOL_FP8, TOL_REL_FP8) if fp8 else (TOL_BF16, TOL_REL)
    for b in range(inp.B):
        L = int(inp.lengths[b])
        r = O.hybrid_query(inp.oracle_seq(b, fp8=fp8), inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        assert cnt[b].item() == r["cnt"], b
        assert np.array_equal(idx[b].cpu().numpy(), r["idx"]), b
        if not outputs:
            continue
        for got, ref in ((oc[b], r["out_csa"]), (oh[b], r["out_hca"])):
            mx, rel = out_errors(got, ref)
            assert mx <= tol and rel <= trel, (b, mx, rel)
        if r["cnt"] > 0:
            assert np.abs(lc[b].cpu().numpy() - r["lse_csa"]).max() < 1e-3, b
        else:
            assert torch.isneginf(lc[b]).all() and not oc[b].float().any(), b
    return oc, oh, idx, cnt


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("B,Lcap,H,k,lengths", [
    (1, 4096, 8, 64, None),                       # 1024 entries, 8 heads
    (3, 9000, 64, 512, [9000, 8995, 3001]),       # every entry a candidate (<= 8192 entries)
    (2, 40000, 64, 700, [40000, 39001]),          # the sampled bound (10,000 entries)
    (2, 70000, 64, 2048, [70000, 65537]),         # k = 2048: eight full 256-entry slices
    (4, 1000, 64, 300, [1000, 1000, 600, 900]),   # n < k for some sequences
    (3, 512, 64, 200, [512, 3, 0]),               # 128 entries, none, none
])
def test_fast_decode_vs_oracle(S, mode, B, Lcap, H, k, lengths):
    inp = Inputs(4100 + Lcap % 997 + k, B, Lcap, H, lengths=lengths)
    _check(S, inp, k, mode)


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_fp8_ragged(S, mode):
    # e4m3 cache with per-64-entry scales, ragged lengths (the fp8 workload's shape, smaller)
    inp = Inputs(4151, 4, 50000, 64, lengths=[50000, 33333, 41001, 16385])
    _check(S, inp, 1024, mode, fp8=True)


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_peaky_queries(S, mode):
    inp = Inputs(4201, 2, 30000, 64, lengths=[30000, 29000], q_scale=8.0)
    _check(S, inp, 700, mode)


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_exact_ties(S, mode):
    # every 4-token block repeated across groups of 8 entries: exact score ties
    B, Lcap, k = 1, 40000, 300
    inp = Inputs(4301, B, Lcap, 64)
    blk = inp.KI[0].reshape(-1, 32, 64)[:, :4]
    inp.KI[0] = np.tile(blk, (1, 8, 1)).reshape(Lcap, 64)
    _check(S, inp, k, mode)


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_near_ties(S, mode):
    # clusters at the top whose scores differ below the fp32 screen's resolution
    B, Lcap, k = 1, 40000, 100
    inp = Inputs(4401, B, Lcap, 64)
    q = bf16_to_f64(inp.qI[0])
    sign = np.where(q >= 0, 1.0, -1.0)
    rows = []
    for base, count in ((1.0, 80), (0.984375, 70)):
        for v in range(count):
            r = sign * base
            r[63] = 0.0
            if v % 3:
                r[63] = sign[63] * 2.0 ** -(18 + v % 7)
            rows.append(r)
    rb = torch.tensor(np.array(rows, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ents = np.random.default_rng(7).choice(Lcap // 4, size=len(rows), replace=False)
    for e, r in zip(ents, rb):
        inp.KI[0, 4 * e:4 * e + 4] = r
    _check(S, inp, k, mode)


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_all_equal_scores(S, mode):
    # 10,000 identical entries: more candidates than shared memory holds and a
    # band far wider than 1024, so the selection runs over every score with
    # the band cut in global memory; the lowest indices win
    B, Lcap, k = 1, 40000, 2000
    inp = Inputs(4501, B, Lcap, 64)
    inp.KI[:] = inp.KI[:, :1, :]
    _, _, idx, cnt = _check(S, inp, k, mode, outputs=False)
    assert (idx[0].cpu().numpy() == np.arange(k)).all() and cnt[0].item() == k


@pytest.mark.parametrize("mode", MODES)
def test_fast_decode_sample_defeated(S, mode):
    # every 16th entry (the sample stride for 10,000 entries and k = 512)
    # scores far above the rest: the sample sees only those, its bound keeps
    # fewer than k candidates, and the selection falls back to every score
    # (about a hundred distinct high scores, so the sample's order statistic
    # lies strictly inside them)
    B, Lcap, k = 1, 40000, 512
    inp = Inputs(4601, B, Lcap, 64)
    q = bf16_to_f64(inp.qI[0])
    sign = np.where(q >= 0, 1.0, -1.0)
    for e in range(0, Lcap // 4, 16):
        r = sign * 0.75
        r[63] = sign[63] * (0.25 + ((e // 16) % 100) * 2.0 ** -7)   # exact in bf16
        rb = torch.tensor(r.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        inp.KI[0, 4 * e:4 * e + 4] = rb
    _check(S, inp, k, mode)


def test_fast_equals_general_path(S):
    # the same selection on both paths, and the same attention kernels after
    # it: every output agrees bit for bit
    B, Lcap, H, k = 3, 50000, 64, 1024
    inp = Inputs(4701, B, Lcap, H, lengths=[50000, 44443, 20001])
    a = _run(S, inp, k, 1)
    b = _run(S, inp, k, 0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fast_decode_deterministic(S):
    inp = Inputs(4801, 2, 40000, 64)
    a = _run(S, inp, 2048, 1)
    b = _run(S, inp, 2048, 1)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
