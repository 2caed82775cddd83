"""Mixed KV storage against the oracle ("DeepSeek-V4 ... Review", section 3-2
(2) component table, "Mixed KV storage": rotary dims in BF16, the rest in
FP8).  The cache keeps K's dims 0..63 as e4m3 codes with one fp32 scale per
64 entries and its rotary dims 64..127 in bf16 (192-byte rows), V in e4m3.
Compression and appends must give the oracle's bytes exactly; the attention
kernels the oracle's output within the fp8 tolerance, in decode and in causal
prefill.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, TOL_FP8, Inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _caches(S, B, Lcap):
    return (S.alloc_cache(B, Lcap // 4, 4, mixed=True, with_kidx=True), S.alloc_cache(B, Lcap // 128, 128, mixed=True))


def _oracle_mixed(Kb, Vb, m):
    """The oracle's mixed storage of one sequence: (K codes, K scales, K rope,
    V codes, V scales)."""
    kc, vc = O.compress(Kb, m), O.compress(Vb, m)
    codes, ks, rope = O.mixed_quantize(kc, 64)
    vcodes, vs = O.fp8_quantize(vc)
    return codes, ks, rope, vcodes, vs


def _check_cache(cache, b, ref, n):
    codes, ks, rope, vcodes, vs = ref
    assert int(cache.n[b]) == n
    k = cache.k[b, :n].cpu().numpy()
    assert np.array_equal(k[:, :64], codes), b
    assert np.array_equal(k[:, 64:].copy().view(np.uint16), rope), b
    assert np.array_equal(cache.v[b, :n].cpu().numpy(), vcodes), b
    ng = (n + 63) // 64
    assert np.array_equal(cache.k_scale[b, :ng].cpu().numpy(), ks.astype(np.float32)), b
    assert np.array_equal(cache.v_scale[b, :ng].cpu().numpy(), vs.astype(np.float32)), b


def test_compress_matches_oracle(S):
    B, Lcap = 3, 40000
    inp = Inputs(901, B, Lcap, 8, lengths=[40000, 17003, 1000])  # ragged, partial last groups
    g = inp.to_device()
    csa, hca = _caches(S, B, Lcap)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    S.read_device_status()
    for b in range(B):
        L = int(inp.lengths[b])
        _check_cache(csa, b, _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 4), L // 4)
        _check_cache(hca, b, _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 128), L // 128)
        # the indexer keys stay bf16
        ki = csa.kidx[b, :L // 4].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(ki, O.compress(inp.KI[b, :L], 4)), b


def test_append_equals_full_compression(S):
    B, Lcap = 2, 12000
    inp = Inputs(902, B, Lcap, 8, lengths=[Lcap] * B)
    g = inp.to_device()
    cur = [250, 5000]
    csa, hca = _caches(S, B, Lcap)
    lens = torch.tensor(cur, dtype=torch.int32, device="cuda")
    S.csa_compress(g["K"], g["V"], g["KI"], lens, csa)
    S.hca_compress(g["K"], g["V"], lens, hca)
    for d in [1] * 8 + [300, 2100]:  # sequence 0 crosses the 64-entry group at 256 tokens
        cur = [min(Lcap, c + d) for c in cur]
        lens = torch.tensor(cur, dtype=torch.int32, device="cuda")
        S.csa_append(g["K"], g["V"], g["KI"], lens, csa, d)
        S.hca_append(g["K"], g["V"], lens, hca, d)
        S.read_device_status()
    for b in range(B):
        L = cur[b]
        _check_cache(csa, b, _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 4), L // 4)
        _check_cache(hca, b, _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 128), L // 128)


def _oracle_attn(q, ref, rows):
    codes, ks, rope, vcodes, vs = ref
    return O.attention_kv(q, {"mode": "mixed", "data": codes, "scales": ks, "rope": rope},
                          {"mode": "fp8", "data": vcodes, "scales": vs}, rows, SCALE, 64)


@pytest.mark.parametrize("H,k", [(64, 2048), (8, 256)])
def test_hybrid_decode_matches_oracle(S, H, k):
    B, Lcap = 3, 20000
    inp = Inputs(903 + H, B, Lcap, H, lengths=[20000, 9001, 300])
    g = inp.to_device()
    csa, hca = _caches(S, B, Lcap)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty_like(lc)
    oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, lse_hca=lh,
                                  idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    for b in range(B):
        L = int(inp.lengths[b])
        # the selection depends on the bf16 indexer keys only
        r = O.hybrid_query(inp.oracle_seq(b), inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        assert int(cnt[b]) == r["cnt"] and np.array_equal(idx[b].cpu().numpy(), r["idx"]), b
        ref_c = _oracle_attn(inp.q[b], _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 4), r["idx"][:r["cnt"]])
        ref_h = _oracle_attn(inp.q[b], _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 128), np.arange(L // 128))
        assert np.abs(oc[b].float().cpu().numpy() - ref_c[0]).max() <= TOL_FP8, b
        assert np.abs(oh[b].float().cpu().numpy() - ref_h[0]).max() <= TOL_FP8, b
        assert np.abs(lc[b].cpu().numpy() - ref_c[1]).max() < 1e-2, b
        if L >= 128:
            assert np.abs(lh[b].cpu().numpy() - ref_h[1]).max() < 1e-2, b


def test_prefill_matches_oracle_every_row(S):
    B, T, H, k = 1, 1200, 64, 64
    inp = Inputs(905, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = _caches(S, B, T)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE)
    S.read_device_status()
    cs = inp.oracle_seq(0)
    refc = _oracle_mixed(inp.K[0], inp.V[0], 4)
    refh = _oracle_mixed(inp.K[0], inp.V[0], 128)
    ocf, ohf = oc[0].float().cpu().numpy(), oh[0].float().cpu().numpy()
    worst = 0.0
    for t in range(0, T, 7):
        r = O.hybrid_query(cs, inp.q[0, t], inp.qI[0, t], t=t, k=k, scale=SCALE)
        assert np.array_equal(idx[0, t].cpu().numpy(), r["idx"]), t
        rc, _ = _oracle_attn(inp.q[0, t], refc, r["idx"][:r["cnt"]])
        rh, _ = _oracle_attn(inp.q[0, t], refh, np.arange(t // 128))
        worst = max(worst, float(np.abs(ocf[t] - rc).max()), float(np.abs(ohf[t] - rh).max()))
    assert worst <= TOL_FP8, worst


def test_fp4_selection_on_mixed_storage(S):
    """FP4 indexer scores and mixed KV storage together (the low-precision
    decode step): indices bit for bit against the oracle's FP4 selection,
    outputs within the fp8 tolerance against attention over the oracle's mixed
    storage."""
    B, Lcap, H, k = 2, 20000, 64, 512
    inp = Inputs(907, B, Lcap, H, lengths=[20000, 7777])
    g = inp.to_device()
    csa, hca = _caches(S, B, Lcap)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    codes, scales = S.csa_index_quantize_mxfp4(csa)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    oc, oh = S.hybrid_attn_decode_mxfp4(g["q"], g["qI"], csa, hca, codes, scales, k, ws, scale=SCALE,
                                        idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    for b in range(B):
        L = int(inp.lengths[b])
        r = O.hybrid_query_mxfp4(inp.oracle_seq(b), inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        assert int(cnt[b]) == r["cnt"] and np.array_equal(idx[b].cpu().numpy(), r["idx"]), b
        ref_c = _oracle_attn(inp.q[b], _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 4), r["idx"][:r["cnt"]])
        ref_h = _oracle_attn(inp.q[b], _oracle_mixed(inp.K[b, :L], inp.V[b, :L], 128), np.arange(L // 128))
        assert np.abs(oc[b].float().cpu().numpy() - ref_c[0]).max() <= TOL_FP8, b
        assert np.abs(oh[b].float().cpu().numpy() - ref_h[0]).max() <= TOL_FP8, b


def test_mixed_decode_deterministic(S):
    B, Lcap, H, k = 2, 16000, 64, 512
    inp = Inputs(908, B, Lcap, H, lengths=[16000, 5000])
    g = inp.to_device()
    csa, hca = _caches(S, B, Lcap)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    a = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    b = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    S.read_device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
