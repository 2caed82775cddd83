"""The FP4 (MXFP4) CSA indexer against the oracle: csa_index_quantize_mxfp4
must give the oracle's codes and scales bit for bit, and csa_index_topk_mxfp4
the oracle's top-k of its FP4 scores ("DeepSeek-V4 ... Review", section 3-2
(4), FP4 on the CSA indexer QK path; section 3-2 (2) top-k).
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_attention_pool_b200 import synth
from tests._util import bits_to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _cache_with_keys(S, kidx_bits: np.ndarray, n):
    """A CSA cache whose indexer keys are the given bf16 bits [B][Ncap][64]."""
    B, Ncap, _ = kidx_bits.shape
    c = S.alloc_cache(B, Ncap, 4, with_kidx=True)
    c.kidx.copy_(bits_to_torch_bf16(kidx_bits).cuda())
    c.n.copy_(torch.tensor(n, dtype=torch.int32))
    return c


def _edge_rows(x: np.ndarray):
    """Plant rows that exercise the format: zero blocks, tiny and huge
    magnitudes, -0, exact e2m1 midpoints and saturation."""
    x[0, :32] = 0.0
    x[1] *= 1e-30
    x[2] *= 1e30
    x[3, 5] = -0.0
    x[4, :8] = [4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -0.25]
    x[5, :4] = [6.0, 5.0, -5.0, 7.0]
    x[6] = 0.0
    return x


def test_quantize_matches_oracle(S):
    B, Ncap = 3, 3000
    n = [3000, 1234, 7]
    xf = synth.bf16_bits_to_f32(synth.normal_bf16(71, "kidx", (B, Ncap, 64))).copy()
    xf[0] = _edge_rows(xf[0])
    bits = (xf.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    c = _cache_with_keys(S, bits, n)
    codes = torch.full((B, Ncap, 32), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((B, Ncap, 2), 0xCD, dtype=torch.uint8, device="cuda")
    S.csa_index_quantize_mxfp4(c, codes=codes, scales=scales)
    S.read_device_status()
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    for b in range(B):
        oc, osc = O.mxfp4_quantize(bits[b, :n[b]])
        assert np.array_equal(gc[b, :n[b]], oc), b
        assert np.array_equal(gs[b, :n[b]], osc), b
        assert (gc[b, n[b]:] == 0xAB).all() and (gs[b, n[b]:] == 0xCD).all(), b  # past n: untouched
    # row_from: earlier rows are left alone
    codes.fill_(0x11)
    scales.fill_(0x22)
    S.csa_index_quantize_mxfp4(c, codes=codes, scales=scales, row_from=1000)
    S.read_device_status()
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    assert (gc[:, :1000] == 0x11).all() and (gs[:, :1000] == 0x22).all()
    oc, osc = O.mxfp4_quantize(bits[0, :3000])
    assert np.array_equal(gc[0, 1000:3000], oc[1000:]) and np.array_equal(gs[0, 1000:3000], osc[1000:])


def _oracle_topk(qI_bits, kidx_bits, n, k):
    qc, qs = O.mxfp4_quantize(qI_bits.reshape(1, -1))
    kc, ks = O.mxfp4_quantize(kidx_bits[:n])
    s = O.mxfp4_index_scores(qc[0], qs[0], kc, ks)
    return O.topk(s, k)


@pytest.mark.parametrize("k", [64, 512])
def test_topk_matches_oracle(S, k):
    B, Ncap = 6, 20000
    n = [20000, 9000, k + 1, k, 3, 0]  # large, ragged, one above k, exactly k, fewer than k, empty
    bits = synth.normal_bf16(72, "kidx", (B, Ncap, 64))
    qI = synth.normal_bf16(72, "qidx", (B, 64))
    c = _cache_with_keys(S, bits, n)
    codes, scales = S.csa_index_quantize_mxfp4(c)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, 8, Ncap, 0, k))
    idx, cnt = S.csa_index_topk_mxfp4(bits_to_torch_bf16(qI).cuda(), c, codes, scales, k, ws)
    S.read_device_status()
    gi, gn = idx[:, 0].cpu().numpy(), cnt[:, 0].cpu().numpy()
    for b in range(B):
        ref, rc = _oracle_topk(qI[b], bits[b], n[b], k)
        assert gn[b] == rc, b
        assert np.array_equal(gi[b], ref), b


def test_topk_all_equal_scores_take_the_lowest_indices(S):
    B, Ncap, k = 2, 8192, 300
    row = synth.normal_bf16(73, "kidx", (1, 64))[0]
    bits = np.broadcast_to(row, (B, Ncap, 64)).copy()
    qI = synth.normal_bf16(73, "qidx", (B, 64))
    c = _cache_with_keys(S, bits, [Ncap, 5000])
    codes, scales = S.csa_index_quantize_mxfp4(c)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, 8, Ncap, 0, k))
    idx, cnt = S.csa_index_topk_mxfp4(bits_to_torch_bf16(qI).cuda(), c, codes, scales, k, ws)
    S.read_device_status()
    assert (cnt[:, 0].cpu() == k).all()
    assert (idx[:, 0].cpu().numpy() == np.arange(k)).all()


def _scaled_bits(rng, shape, scale0, scale1):
    """bf16 bits of normals times 2^scale0 (dims 0..31) and 2^scale1 (32..63)."""
    x = rng.standard_normal(shape).astype(np.float32)
    x[..., :32] *= np.float32(2.0 ** scale0)
    x[..., 32:] *= np.float32(2.0 ** scale1)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def test_topk_of_tiny_and_huge_blocks(S):
    """Scores whose block terms leave fp32's exact range: subnormal scores
    (both blocks tiny) and scores that overflow to +-inf (both blocks huge),
    where the kernels switch to their fp64 routine; decode and every row of a
    short prefill against the oracle."""
    rng = np.random.default_rng(76)
    B, Ncap, k = 2, 5000, 300
    bits = np.stack([_scaled_bits(rng, (Ncap, 64), -78, -82), _scaled_bits(rng, (Ncap, 64), 100, 114)])
    qI = np.stack([_scaled_bits(rng, (64,), -68, -68), _scaled_bits(rng, (64,), 12, 12)])
    c = _cache_with_keys(S, bits, [Ncap, Ncap])
    codes, scales = S.csa_index_quantize_mxfp4(c)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, 8, Ncap, 0, k))
    idx, cnt = S.csa_index_topk_mxfp4(bits_to_torch_bf16(qI).cuda(), c, codes, scales, k, ws)
    S.read_device_status()
    gi, gn = idx[:, 0].cpu().numpy(), cnt[:, 0].cpu().numpy()
    for b in range(B):
        ref, rc = _oracle_topk(qI[b], bits[b], Ncap, k)
        assert gn[b] == rc and np.array_equal(gi[b], ref), b
    # prefill: every row of 600 positions over the tiny keys
    T, kp = 600, 32
    qP = _scaled_bits(rng, (1, T, 64), -68, -70)
    c1 = _cache_with_keys(S, bits[:1, : T // 4], [T // 4])
    codes1, scales1 = S.csa_index_quantize_mxfp4(c1)
    pos = torch.arange(T, dtype=torch.int32, device="cuda").view(1, T).contiguous()
    ws1 = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, 1, T, 8, c1.Ncap, 0, kp))
    pi, pn = S.csa_index_topk_mxfp4(bits_to_torch_bf16(qP).cuda(), c1, codes1, scales1, kp, ws1, q_pos=pos)
    S.read_device_status()
    pi, pn = pi[0].cpu().numpy(), pn[0].cpu().numpy()
    for t in range(T):
        ref, rc = _oracle_topk(qP[0, t], bits[0], t // 4, kp)
        assert pn[t] == rc and np.array_equal(pi[t], ref), t


def test_topk_full_size_decode(S):
    """Four sequences of 262,144 entries (1M tokens each), k = 2048: every
    index against the oracle."""
    B, Ncap, k = 4, 262144, 2048
    bits = synth.normal_bf16(74, "kidx", (B, Ncap, 64), scale=0.5)
    qI = synth.normal_bf16(74, "qidx", (B, 64))
    c = _cache_with_keys(S, bits, [Ncap] * B)
    codes, scales = S.csa_index_quantize_mxfp4(c)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, 64, Ncap, 0, k))
    idx, cnt = S.csa_index_topk_mxfp4(bits_to_torch_bf16(qI).cuda(), c, codes, scales, k, ws)
    S.read_device_status()
    gi = idx[:, 0].cpu().numpy()
    for b in range(B):
        ref, rc = _oracle_topk(qI[b], bits[b], Ncap, k)
        assert rc == k and np.array_equal(gi[b], ref), b


def test_hybrid_decode_mxfp4_matches_oracle(S):
    """One decode step of both branches with the CSA selection on FP4 scores:
    indices bit for bit, outputs within the bf16 tolerance."""
    from tests._util import SCALE, TOL_BF16, Inputs, compress_on_gpu
    B, Lcap, H, k = 3, 6000, 64, 256
    inp = Inputs(75, B, Lcap, H, lengths=[6000, 3001, 700])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
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
        assert np.abs(oc[b].float().cpu().numpy() - r["out_csa"]).max() <= TOL_BF16, b
        assert np.abs(oh[b].float().cpu().numpy() - r["out_hca"]).max() <= TOL_BF16, b


def test_topk_prefill_every_row(S):
    """Causal prefill on FP4 scores: row t sees the entries with (c+1)*4 <= t;
    every row's indices against the oracle."""
    from tests._util import compress_on_gpu, Inputs
    B, T, k = 1, 1500, 64
    inp = Inputs(76, B, T, 8, Tq=T)
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, T)
    codes, scales = S.csa_index_quantize_mxfp4(csa)
    pos = torch.arange(T, dtype=torch.int32, device="cuda").view(1, T).contiguous()
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, T, 8, csa.Ncap, 0, k))
    idx, cnt = S.csa_index_topk_mxfp4(g["qI"], csa, codes, scales, k, ws, q_pos=pos)
    S.read_device_status()
    ci = O.compress(inp.KI[0], 4)
    kc, ks = O.mxfp4_quantize(ci)
    gi, gn = idx[0].cpu().numpy(), cnt[0].cpu().numpy()
    for t in range(T):
        qc, qs = O.mxfp4_quantize(inp.qI[0, t].reshape(1, -1))
        nv = t // 4
        s = O.mxfp4_index_scores(qc[0], qs[0], kc[:nv], ks[:nv])
        ref, rc = O.topk(s, k)
        assert gn[t] == rc and np.array_equal(gi[t], ref), t


def test_hybrid_prefill_mxfp4_matches_oracle(S):
    """Causal prefill of both branches with the CSA selection on FP4 scores:
    every row's indices bit for bit, sampled rows' outputs within the bf16
    tolerance."""
    from tests._util import SCALE, TOL_BF16, Inputs, compress_on_gpu
    B, T, H, k = 1, 1100, 64, 64
    inp = Inputs(77, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    codes, scales = S.csa_index_quantize_mxfp4(csa)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    oc, oh = S.hybrid_attn_prefill_mxfp4(g["q"], g["qI"], csa, hca, codes, scales, k, ws, idx, cnt, scale=SCALE)
    S.read_device_status()
    cs = inp.oracle_seq(0)
    for t in list(range(0, T, 11)) + [T - 1]:
        r = O.hybrid_query_mxfp4(cs, inp.q[0, t], inp.qI[0, t], t=t, k=k, scale=SCALE)
        assert int(cnt[0, t]) == r["cnt"] and np.array_equal(idx[0, t].cpu().numpy(), r["idx"]), t
        assert np.abs(oc[0, t].float().cpu().numpy() - r["out_csa"]).max() <= TOL_BF16, t
        assert np.abs(oh[0, t].float().cpu().numpy() - r["out_hca"]).max() <= TOL_BF16, t


def test_fp4_selection_deterministic_and_batch_invariant(S):
    """Run to run the same bits, and a sequence alone selects what it selects
    inside a batch."""
    B, Ncap, k = 3, 30000, 512
    bits = synth.normal_bf16(78, "kidx", (B, Ncap, 64))
    qI = synth.normal_bf16(78, "qidx", (B, 64))
    n = [30000, 17000, 900]
    c = _cache_with_keys(S, bits, n)
    codes, scales = S.csa_index_quantize_mxfp4(c)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, 8, Ncap, 0, k))
    q = bits_to_torch_bf16(qI).cuda()
    i1, c1 = S.csa_index_topk_mxfp4(q, c, codes, scales, k, ws)
    i2, c2 = S.csa_index_topk_mxfp4(q, c, codes, scales, k, ws)
    S.read_device_status()
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
    for b in range(B):
        cb = _cache_with_keys(S, bits[b:b + 1], [n[b]])
        cdb, scb = S.csa_index_quantize_mxfp4(cb)
        wsb = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, 1, 1, 8, Ncap, 0, k))
        ib, cnb = S.csa_index_topk_mxfp4(q[b:b + 1].contiguous(), cb, cdb, scb, k, wsb)
        S.read_device_status()
        assert torch.equal(ib[0], i1[b]) and torch.equal(cnb[0], c1[b]), b
