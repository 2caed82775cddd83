"""Context-parallel decode on one GPU: W ranks emulated one after another
(each rank's shard compressed on its own, the all-gathers replaced by
stacking the ranks' arrays in rank order) must select exactly the entries of
the single-GPU decode step and give its outputs; cp_decode_step itself runs
in a one-rank NCCL group.  Kernels that wait on other ranks do not exist in
this path (the exchange is between launches), so the emulation runs the same
kernels a multi-GPU step runs.
"""
from __future__ import annotations

import datetime
import socket

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_attention_pool_b200 import cp
from tests._util import SCALE, TOL_BF16, Inputs, bits_to_torch_bf16, compress_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _shards(S, inp, W):
    """Per emulated rank: its compressed CSA / HCA shard and base [B]."""
    B = inp.B
    bounds = [cp.shard_bounds(int(inp.lengths[b]), W) for b in range(B)]
    out = []
    for w in range(W):
        span = [bounds[b][w] for b in range(B)]
        Lw = max(1, max(t1 - t0 for t0, t1 in span))
        Lw = -(-Lw // 128) * 128
        K = np.zeros((B, Lw, 128), np.uint16)
        V = np.zeros((B, Lw, 128), np.uint16)
        KI = np.zeros((B, Lw, 64), np.uint16)
        for b, (t0, t1) in enumerate(span):
            K[b, :t1 - t0], V[b, :t1 - t0], KI[b, :t1 - t0] = inp.K[b, t0:t1], inp.V[b, t0:t1], inp.KI[b, t0:t1]
        g = {"K": bits_to_torch_bf16(K).cuda(), "V": bits_to_torch_bf16(V).cuda(),
             "KI": bits_to_torch_bf16(KI).cuda(),
             "len": torch.tensor([t1 - t0 for t0, t1 in span], dtype=torch.int32, device="cuda")}
        csa, hca = compress_on_gpu(S, g, B, Lw)
        base = torch.tensor([cp.entry_base(bounds[b], w, 4) for b in range(B)], dtype=torch.int32, device="cuda")
        out.append((csa, hca, base))
    return out


@pytest.mark.parametrize("W,k,lengths", [(2, 512, [40000, 23457, 1000]), (4, 2048, [40000, 23457, 1000]),
                                         (3, 64, [40000, 23457, 1000]),
                                         (3, 64, [5000, 200, 130])])  # shards of 200 / 130 tokens: some empty
def test_emulated_ranks_match_the_single_gpu_step(S, W, k, lengths):
    B, Lcap, H = 3, max(lengths), 64
    inp = Inputs(921 + W, B, Lcap, H, lengths=lengths)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty_like(lc)
    oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, lse_hca=lh,
                                  idx_out=idx, cnt_out=cnt)
    shards = _shards(S, inp, W)
    wss = [S.alloc_workspace(cp.workspace_size(B, H, c.Ncap, h.Ncap, k)) for c, h, _ in shards]
    cands = [S.cp_decode_candidates(g["qI"], c, k, base, w_) for (c, _, base), w_ in zip(shards, wss)]
    all_keys = torch.stack([x[0] for x in cands])
    all_gidx = torch.stack([x[1] for x in cands])
    all_gcnt = torch.stack([x[2] for x in cands])
    part_o = torch.empty(W, 2, B, H, 128, dtype=torch.bfloat16, device="cuda")
    part_l = torch.empty(W, 2, B, H, dtype=torch.float32, device="cuda")
    for w, ((c, h, base), w_) in enumerate(zip(shards, wss)):
        li, ln, si, sn = S.cp_decode_merge_select(all_keys, all_gidx, all_gcnt, w, base)
        assert torch.equal(si, idx) and torch.equal(sn, cnt), w  # every rank: the single-GPU selection
        S.csa_sparse_attn(g["q"], c, li, ln, k, w_, scale=SCALE, out=part_o[w, 0], lse=part_l[w, 0])
        S.hca_dense_attn(g["q"], h, w_, scale=SCALE, out=part_o[w, 1], lse=part_l[w, 1])
    out, lse = S.attn_lse_merge_n(part_o, part_l)
    S.read_device_status()
    assert (out[0].float() - oc.float()).abs().max().item() <= TOL_BF16
    assert (out[1].float() - oh.float()).abs().max().item() <= TOL_BF16
    assert (lse[0] - lc).abs().max().item() < 1e-3
    for b in range(B):
        if int(inp.lengths[b]) >= 128:
            assert (lse[1, b] - lh[b]).abs().max().item() < 1e-3, b
        L = int(inp.lengths[b])
        r = O.hybrid_query(inp.oracle_seq(b), inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        assert np.abs(out[0, b].float().cpu().numpy() - r["out_csa"]).max() <= TOL_BF16, b
        assert np.abs(out[1, b].float().cpu().numpy() - r["out_hca"]).max() <= TOL_BF16, b


def test_merge_n_of_one_and_of_empty_parts(S):
    rows = 40
    a = torch.randn(1, rows, 128, device="cuda").to(torch.bfloat16)
    la = torch.randn(1, rows, device="cuda")
    out, lse = S.attn_lse_merge_n(a, la)
    S.read_device_status()
    assert torch.equal(out, a[0]) and torch.allclose(lse, la[0])
    z = torch.zeros(3, rows, 128, dtype=torch.bfloat16, device="cuda")
    lz = torch.full((3, rows), float("-inf"), device="cuda")
    out, lse = S.attn_lse_merge_n(z, lz)
    assert not out.float().any() and torch.isneginf(lse).all()


def test_cp_decode_step_in_a_one_rank_group(S):
    import torch.distributed as dist
    B, Lcap, H, k = 2, 8000, 64, 256
    inp = Inputs(931, B, Lcap, H, lengths=[8000, 5000])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        ws = S.alloc_workspace(cp.workspace_size(B, H, csa.Ncap, hca.Ncap, k))
        base = torch.zeros(B, dtype=torch.int32, device="cuda")
        oc, oh, lc, lh, sel, scnt = cp.cp_decode_step(g["q"], g["qI"], csa, hca, base, k, ws, scale=SCALE)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    S.read_device_status()
    ws2 = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    rc, rh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws2, scale=SCALE, idx_out=idx, cnt_out=cnt)
    assert torch.equal(sel, idx) and torch.equal(scnt, cnt)
    assert (oc.float() - rc.float()).abs().max().item() <= TOL_BF16
    assert (oh.float() - rh.float()).abs().max().item() <= TOL_BF16
