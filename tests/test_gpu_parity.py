"""CUDA path vs the fp64 oracle on seeded inputs (needs a B200).

Compressed caches and fp8 codes/scales: bit-exact.  Top-k indices and counts:
bit-exact.  Attention outputs: max-abs error <= 1e-2 (bf16 cache) or 3e-2
(fp8 cache), and rms(err) / rms(oracle) <= 1e-2 (bf16) or 3e-2 (fp8) on top.  Sizes span
several tiles and ragged tails; full-size workloads are checked on samples in
test_gpu_fullsize.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import (SCALE, TOL_BF16, TOL_FP8, TOL_REL, TOL_REL_FP8, Inputs, bf16_to_f64, compress_on_gpu, out_errors,
                         torch_bf16_to_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


# ----------------------------------------------------------- compression ---

@pytest.mark.parametrize("fp8", [False, True])
def test_compress_bit_exact(S, fp8):
    B, Lcap = 3, 5000
    lengths = [5000, 4099, 131]        # ragged, with incomplete tails
    inp = Inputs(101, B, Lcap, 8, lengths=lengths)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap, fp8=fp8)
    S.read_device_status()
    assert csa.n.cpu().tolist() == [l // 4 for l in lengths]
    assert hca.n.cpu().tolist() == [l // 128 for l in lengths]
    for b in range(B):
        cs = inp.oracle_seq(b, fp8=fp8)
        nc, nh = cs.n_csa, cs.n_hca
        if fp8:
            assert np.array_equal(csa.k[b, :nc].cpu().numpy(), cs.ck)
            assert np.array_equal(csa.v[b, :nc].cpu().numpy(), cs.cv)
            assert np.array_equal(hca.k[b, :nh].cpu().numpy(), cs.hk)
            assert np.array_equal(hca.v[b, :nh].cpu().numpy(), cs.hv)
            ng, nhg = (nc + 63) // 64, (nh + 63) // 64
            assert np.array_equal(csa.k_scale[b, :ng].cpu().numpy(), cs.cks)
            assert np.array_equal(csa.v_scale[b, :ng].cpu().numpy(), cs.cvs)
            assert np.array_equal(hca.k_scale[b, :nhg].cpu().numpy(), cs.hks)
            assert np.array_equal(hca.v_scale[b, :nhg].cpu().numpy(), cs.hvs)
        else:
            assert np.array_equal(torch_bf16_to_bits(csa.k[b, :nc]), cs.ck)
            assert np.array_equal(torch_bf16_to_bits(csa.v[b, :nc]), cs.cv)
            assert np.array_equal(torch_bf16_to_bits(hca.k[b, :nh]), cs.hk)
            assert np.array_equal(torch_bf16_to_bits(hca.v[b, :nh]), cs.hv)
        assert np.array_equal(torch_bf16_to_bits(csa.kidx[b, :nc]), cs.cidx)


def test_compress_m1_and_m2_identity_and_pairs(S):
    B, Lcap = 1, 300
    inp = Inputs(102, B, Lcap, 8)
    g = inp.to_device()
    c1 = S.alloc_cache(B, Lcap, 1, with_kidx=True)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], c1)
    assert np.array_equal(torch_bf16_to_bits(c1.k[0]), inp.K[0])
    c2 = S.alloc_cache(B, Lcap // 2, 2, with_kidx=True)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], c2)
    assert np.array_equal(torch_bf16_to_bits(c2.k[0]), O.compress(inp.K[0], 2))
    S.read_device_status()


# ---------------------------------------------------------------- top-k ----

def _topk_case(S, inp, k, fp8=False):
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, inp.B, inp.Lcap, fp8=fp8)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, inp.B, 1, inp.H, csa.Ncap, 0, k))
    idx, cnt = S.csa_index_topk(g["qI"], csa, k, ws)
    S.read_device_status()
    return g, csa, hca, idx.cpu().numpy()[:, 0], cnt.cpu().numpy()[:, 0]


@pytest.mark.parametrize("B,Lcap,k", [(1, 4096, 64), (3, 20000, 512), (2, 70000, 1000), (4, 1000, 300)])
def test_decode_topk_bit_exact(S, B, Lcap, k):
    lengths = [Lcap - 3 * b for b in range(B)]
    inp = Inputs(200 + Lcap % 97, B, Lcap, 8, lengths=lengths)
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    for b in range(B):
        cs = inp.oracle_seq(b)
        s = O.index_scores(inp.qI[b], cs.cidx)
        ridx, rcnt = O.topk(s, k)
        assert cnt[b] == rcnt
        assert np.array_equal(idx[b], ridx), b


def test_decode_topk_ties_lowest_index(S):
    # every 4-token block identical within groups of 8 entries: exact score ties
    B, Lcap, k = 1, 8192, 300
    inp = Inputs(301, B, Lcap, 8)
    blk = inp.KI[0].reshape(-1, 32, 64)[:, :4]                 # 4 tokens of each 32-token group
    inp.KI[0] = np.tile(blk, (1, 8, 1)).reshape(Lcap, 64)      # entries repeat 8 times
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    cs = inp.oracle_seq(0)
    s = O.index_scores(inp.qI[0], cs.cidx)
    ridx, rcnt = O.topk(s, k)
    assert np.array_equal(idx[0], ridx) and cnt[0] == rcnt


def test_decode_topk_near_ties_need_exact_rescoring(S):
    # clusters of entries whose scores differ by far less than the fp32 screen
    # can resolve (and often tie exactly after the final fp32 rounding)
    B, Lcap, k = 1, 16384, 100
    inp = Inputs(304, B, Lcap, 8)
    q = bf16_to_f64(inp.qI[0])
    sign = np.where(q >= 0, 1.0, -1.0)
    rows = []
    for base, count in ((1.0, 80), (0.984375, 70)):   # two clusters at the top
        for v in range(count):
            r = sign * base
            r[63] = 0.0
            if v % 3:
                r[63] = sign[63] * 2.0 ** -(18 + v % 7)    # exact bf16, below the screen's resolution
            rows.append(r)
    rows = np.array(rows, dtype=np.float32)
    rb = torch.tensor(rows).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ents = np.random.default_rng(5).choice(Lcap // 4, size=len(rows), replace=False)
    for e, r in zip(ents, rb):
        inp.KI[0, 4 * e:4 * e + 4] = r                   # constant block -> the entry is exactly r
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    cs = inp.oracle_seq(0)
    s = O.index_scores(inp.qI[0], cs.cidx)
    ridx, rcnt = O.topk(s, k)
    assert len(set(s[ents].tolist())) < len(ents)       # exact ties exist among the clusters
    assert np.array_equal(idx[0], ridx) and cnt[0] == rcnt


def test_decode_topk_all_equal_scores(S):
    B, Lcap, k = 2, 4000, 77
    inp = Inputs(302, B, Lcap, 8)
    inp.KI[:] = inp.KI[:, :1, :]                               # every entry identical
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    assert (idx == np.arange(k)[None, :]).all() and (cnt == k).all()


@pytest.mark.parametrize("k", [77, 2000])
def test_decode_topk_all_equal_scores_overflow_paths(S, k):
    # 10,000 identical entries: more candidates than the resolve holds in shared
    # memory (the list goes to global memory), a crowded fine bin (the digit
    # passes) and a band wider than 1024 (the global band cut)
    B, Lcap = 1, 40000
    inp = Inputs(305, B, Lcap, 8)
    inp.KI[:] = inp.KI[:, :1, :]
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    assert (idx == np.arange(k)[None, :]).all() and (cnt == k).all()


def test_decode_topk_mixed_batch(S):
    # 37 sequences of every kind in one call: the score kernel hands its
    # 128-row tiles out dynamically, skipping sequences with n <= k and the
    # tiles past each length, and finishes each sequence when its last tile
    # is counted (whichever CTA scanned it)
    B, Lcap, k = 37, 9000, 300
    rng = np.random.default_rng(17)
    fixed = [0, 3, 4 * k, 4 * k + 4, 4 * (k + 1) + 3, 512 * 4, 512 * 4 + 4, Lcap, Lcap - 1, 128 * 4 * 7]
    lengths = fixed + rng.integers(0, Lcap + 1, size=B - len(fixed)).tolist()
    inp = Inputs(306, B, Lcap, 8, lengths=lengths)
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    for b in range(B):
        cs = inp.oracle_seq(b)
        s = O.index_scores(inp.qI[b], cs.cidx)
        ridx, rcnt = O.topk(s, k)
        assert cnt[b] == rcnt, b
        assert np.array_equal(idx[b], ridx), b


def test_decode_topk_short_and_empty(S):
    B, Lcap, k = 3, 512, 200
    inp = Inputs(303, B, Lcap, 8, lengths=[512, 3, 0])         # 128, 0, 0 entries
    _, _, _, idx, cnt = _topk_case(S, inp, k)
    assert cnt.tolist() == [128, 0, 0]
    assert idx[0, :128].tolist() == list(range(128)) and (idx[0, 128:] == -1).all()
    assert (idx[1:] == -1).all()


# ------------------------------------------------------------- attention ---

def _check_outputs(got, ref, tol):
    mx, rel = out_errors(got, ref)
    assert mx <= tol, (mx, rel)
    assert rel <= (TOL_REL if tol == TOL_BF16 else TOL_REL_FP8), (mx, rel)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("B,Lcap,H,k,q_scale", [(1, 4096, 8, 64, 1.0), (3, 9000, 64, 512, 1.0),
                                                 (2, 30000, 64, 700, 8.0), (2, 2000, 100, 64, 1.0)])
def test_hybrid_decode_vs_oracle(S, B, Lcap, H, k, q_scale, fp8):
    lengths = [Lcap - 5 * b for b in range(B)]
    inp = Inputs(400 + H + k, B, Lcap, H, lengths=lengths, q_scale=q_scale)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap, fp8=fp8)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty(B, H, dtype=torch.float32, device="cuda")
    oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, lse_hca=lh,
                                  idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    tol = TOL_FP8 if fp8 else TOL_BF16
    for b in range(B):
        cs = inp.oracle_seq(b, fp8=fp8)
        r = O.hybrid_query(cs, inp.q[b], inp.qI[b], t=int(inp.lengths[b]), k=k, scale=SCALE)
        assert np.array_equal(idx[b].cpu().numpy(), r["idx"])
        assert cnt[b].item() == r["cnt"]
        _check_outputs(oc[b], r["out_csa"], tol)
        _check_outputs(oh[b], r["out_hca"], tol)
        assert np.abs(lc[b].cpu().numpy() - r["lse_csa"]).max() < 1e-3
        assert np.abs(lh[b].cpu().numpy() - r["lse_hca"]).max() < 1e-3


def test_separate_calls_equal_hybrid(S):
    B, Lcap, H, k = 2, 12000, 64, 256
    inp = Inputs(501, B, Lcap, H)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    ws2 = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, H, csa.Ncap, 0, k))
    idx, cnt = S.csa_index_topk(g["qI"], csa, k, ws2)
    ws3 = S.alloc_workspace(S.workspace_size(S.SA_OP_SPARSE_ATTN, B, 1, H, csa.Ncap, 0, k))
    oc2 = S.csa_sparse_attn(g["q"], csa, idx, cnt, k, ws3, scale=SCALE)
    ws4 = S.alloc_workspace(S.workspace_size(S.SA_OP_DENSE_ATTN, B, 1, H, 0, hca.Ncap, k))
    oh2 = S.hca_dense_attn(g["q"], hca, ws4, scale=SCALE)
    S.read_device_status()
    assert torch.equal(oc.view(torch.int16), oc2.view(torch.int16))
    assert torch.equal(oh.view(torch.int16), oh2.view(torch.int16))


def test_decode_deterministic_and_batch_invariant(S):
    B, Lcap, H, k = 4, 16000, 64, 512
    inp = Inputs(502, B, Lcap, H, lengths=[16000, 15001, 9000, 16000])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    a1 = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    a2 = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    for x, y in zip(a1, a2):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    # sequence 2 alone, with the same cache capacity
    b = 2
    g1 = {kk: v[b:b + 1].clone() for kk, v in g.items()}
    csa1, hca1 = compress_on_gpu(S, g1, 1, Lcap)
    ws1 = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, 1, 1, H, csa1.Ncap, hca1.Ncap, k))
    s1 = S.hybrid_attn_decode(g1["q"], g1["qI"], csa1, hca1, k, ws1, scale=SCALE)
    assert torch.equal(s1[0][0].view(torch.int16), a1[0][b].view(torch.int16))
    assert torch.equal(s1[1][0].view(torch.int16), a1[1][b].view(torch.int16))


def test_csa_with_k_covering_all_equals_dense(S):
    # k >= N: CSA attends over every entry, i.e. dense attention over the CSA cache
    B, Lcap, H = 1, 2048, 64
    inp = Inputs(503, B, Lcap, H)
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, Lcap)
    n = Lcap // 4
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, H, csa.Ncap, 0, n + 5))
    idx, cnt = S.csa_index_topk(g["qI"], csa, n + 5, ws)
    wsa = S.alloc_workspace(S.workspace_size(S.SA_OP_SPARSE_ATTN, B, 1, H, csa.Ncap, 0, n + 5))
    oc = S.csa_sparse_attn(g["q"], csa, idx, cnt, n + 5, wsa, scale=SCALE)
    wsd = S.alloc_workspace(S.workspace_size(S.SA_OP_DENSE_ATTN, B, 1, H, 0, csa.Ncap, 0))
    od = S.hca_dense_attn(g["q"], csa, wsd, scale=SCALE)
    S.read_device_status()
    cs = inp.oracle_seq(0)
    ref, _ = O.attention(inp.q[0], cs.ck, cs.cv, np.arange(n), SCALE)
    _check_outputs(oc[0], ref, TOL_BF16)
    _check_outputs(od[0], ref, TOL_BF16)


# ---------------------------------------------------------------- prefill --

@pytest.mark.parametrize("fp8", [False, True])
def test_prefill_vs_oracle_every_row(S, fp8):
    B, T, H, k = 1, 1500, 8, 32
    inp = Inputs(601, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T, fp8=fp8)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE, lse_csa=lc)
    S.read_device_status()
    cs = inp.oracle_seq(0, fp8=fp8)
    tol = TOL_FP8 if fp8 else TOL_BF16
    idx_h, cnt_h = idx.cpu().numpy()[0], cnt.cpu().numpy()[0]
    ocf = oc.float().cpu().numpy()[0]
    ohf = oh.float().cpu().numpy()[0]
    worst_c = worst_h = 0.0
    for t in range(T):
        r = O.hybrid_query(cs, inp.q[0, t], inp.qI[0, t], t=t, k=k, scale=SCALE)
        assert cnt_h[t] == r["cnt"], t
        assert np.array_equal(idx_h[t], r["idx"]), t
        worst_c = max(worst_c, float(np.abs(ocf[t] - r["out_csa"]).max()))
        worst_h = max(worst_h, float(np.abs(ohf[t] - r["out_hca"]).max()))
        if t < 4:
            assert not ocf[t].any() and np.isneginf(lc[0, t].cpu().numpy()).all()
    assert worst_c <= tol and worst_h <= tol, (worst_c, worst_h)


@pytest.mark.parametrize("T,k", [(1001, 96), (640, 256)])
def test_prefill_tensor_core_path_vs_oracle_every_row(S, T, k):
    """64 heads over a bf16 cache: the HCA branch runs on the tcgen05 prefill
    kernel (two query positions per CTA; an odd T leaves one alone), the CSA
    branch on the transposed tcgen05 kernel (k not a multiple of its
    128-entry tile)."""
    B, H = 2, 64
    inp = Inputs(611 + T, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    lh = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE, lse_csa=lc, lse_hca=lh)
    S.read_device_status()
    for b in range(B):
        cs = inp.oracle_seq(b)
        ocf, ohf = oc[b].float().cpu().numpy(), oh[b].float().cpu().numpy()
        lcf, lhf = lc[b].cpu().numpy(), lh[b].cpu().numpy()
        worst = 0.0
        for t in range(T):
            r = O.hybrid_query(cs, inp.q[b, t], inp.qI[b, t], t=t, k=k, scale=SCALE)
            worst = max(worst, float(np.abs(ocf[t] - r["out_csa"]).max()), float(np.abs(ohf[t] - r["out_hca"]).max()))
            if r["cnt"] == 0:
                assert not ocf[t].any() and np.isneginf(lcf[t]).all(), t
            else:
                assert np.abs(lcf[t] - r["lse_csa"]).max() < 1e-3, t
            if t >= 128:
                assert np.abs(lhf[t] - r["lse_hca"]).max() < 1e-3, t
        assert worst <= TOL_BF16, (b, worst)


def test_prefill_row_equals_decode(S):
    B, T, H, k = 1, 3000, 64, 128
    inp = Inputs(602, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE)
    for t in (5, 128, 700, 2999):
        lens = torch.tensor([t], dtype=torch.int32, device="cuda")
        dc = S.alloc_cache(1, T // 4, 4, with_kidx=True)
        dh = S.alloc_cache(1, T // 128, 128)
        S.csa_compress(g["K"], g["V"], g["KI"], lens, dc)
        S.hca_compress(g["K"], g["V"], lens, dh)
        wsd = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, 1, 1, H, dc.Ncap, dh.Ncap, k))
        di = torch.empty(1, k, dtype=torch.int32, device="cuda")
        dcnt = torch.empty(1, dtype=torch.int32, device="cuda")
        a, bb = S.hybrid_attn_decode(g["q"][:, t].contiguous(), g["qI"][:, t].contiguous(), dc, dh, k, wsd,
                                     scale=SCALE, idx_out=di, cnt_out=dcnt)
        assert torch.equal(di[0], idx[0, t]) and dcnt.item() == cnt[0, t].item()
        assert (a[0].float() - oc[0, t].float()).abs().max().item() <= 2e-3
        assert (bb[0].float() - oh[0, t].float()).abs().max().item() <= 2e-3
    S.read_device_status()


# ------------------------------------------------------------ device status --

def test_device_status_flags_bad_length(S):
    B, Lcap = 2, 256
    inp = Inputs(701, B, Lcap, 8, lengths=[256, 999])          # 999 > Lcap: clamped and flagged
    g = inp.to_device()
    csa = S.alloc_cache(B, Lcap // 4, 4, with_kidx=True)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    with pytest.raises(S.SparseAttnError) as e:
        S.read_device_status()
    assert "SA_ERR_DEVICE" in str(e.value)
    assert csa.n.cpu().tolist() == [64, 64]
    S.read_device_status()                                     # cleared
