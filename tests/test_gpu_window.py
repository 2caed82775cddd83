"""The sliding-window branch and its merge with a compressed branch, against
the oracle: swa_attn over the last `window` raw tokens before the query, and
attn_lse_merge giving the attention over the union of the CSA selection and
the window (one softmax over both), in decode and in causal prefill.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, TOL_BF16, Inputs, compress_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def test_window_and_merge_decode(S):
    B, Lcap, H, k, w = 3, 3000, 64, 256, 128
    inp = Inputs(901, B, Lcap, H, lengths=[3000, 97, 1500])   # 97 < window: every token
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(max(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, H, csa.Ncap, 0, k),
                               S.workspace_size(S.SA_OP_SPARSE_ATTN, B, 1, H, csa.Ncap, 0, k),
                               S.workspace_size(S.SA_OP_WINDOW_ATTN, B, 1, H, 0, 0, w)))
    idx, cnt = S.csa_index_topk(g["qI"], csa, k, ws)
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lw = torch.empty_like(lc)
    lm = torch.empty_like(lc)
    oc = S.csa_sparse_attn(g["q"], csa, idx, cnt, k, ws, scale=SCALE, lse=lc)
    ow = S.swa_attn(g["q"], g["K"], g["V"], g["len"], w, ws, scale=SCALE, lse=lw)
    om = S.attn_lse_merge(oc, lc, ow, lw, lse=lm)
    S.read_device_status()
    for b in range(B):
        L = int(inp.lengths[b])
        cs = inp.oracle_seq(b)
        r = O.hybrid_query(cs, inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        wrows = O.window_rows(L, L, w)
        ref_w, ref_lw = O.union_attention(inp.q[b], [(inp.K[b], inp.V[b], wrows)], SCALE)
        ref_u, ref_lu = O.union_attention(inp.q[b], [(cs.ck, cs.cv, r["idx"][:r["cnt"]]),
                                                     (inp.K[b], inp.V[b], wrows)], SCALE)
        assert np.abs(ow[b].float().cpu().numpy() - ref_w).max() <= TOL_BF16, b
        assert np.abs(lw[b].cpu().numpy() - ref_lw).max() < 1e-3, b
        assert np.abs(om[b].float().cpu().numpy() - ref_u).max() <= TOL_BF16, b
        assert np.abs(lm[b].cpu().numpy() - ref_lu).max() < 1e-3, b


def test_window_prefill_every_row(S):
    B, T, H, w = 1, 700, 8, 64
    inp = Inputs(902, B, T, H, Tq=T)
    g = inp.to_device()
    pos = torch.arange(T, dtype=torch.int32, device="cuda").view(1, T).contiguous()
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_WINDOW_ATTN, B, T, H, 0, 0, w))
    lw = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    ow = S.swa_attn(g["q"], g["K"], g["V"], g["len"], w, ws, q_pos=pos, scale=SCALE, lse=lw)
    S.read_device_status()
    owf, lwf = ow[0].float().cpu().numpy(), lw[0].cpu().numpy()
    worst = 0.0
    for t in range(T):
        ref, ref_l = O.union_attention(inp.q[0, t], [(inp.K[0], inp.V[0], O.window_rows(t, T, w))], SCALE)
        worst = max(worst, float(np.abs(owf[t] - ref).max()))
        if t == 0:
            assert not owf[t].any() and np.isneginf(lwf[t]).all()
        else:
            assert np.abs(lwf[t] - ref_l).max() < 1e-3, t
    assert worst <= TOL_BF16, worst


def test_merge_with_an_empty_side_is_the_other_side(S):
    rows = 16
    a = torch.randn(rows, 128, device="cuda").to(torch.bfloat16)
    la = torch.randn(rows, device="cuda")
    b = torch.zeros_like(a)
    lb = torch.full((rows,), float("-inf"), device="cuda")
    lm = torch.empty_like(la)
    om = S.attn_lse_merge(a, la, b, lb, lse=lm)
    S.read_device_status()
    assert (om.float() - a.float()).abs().max().item() <= 2 ** -8 * a.float().abs().max().item()
    assert torch.allclose(lm, la)
    both = S.attn_lse_merge(b, lb, b, lb, lse=lm)
    assert not both.float().any() and torch.isneginf(lm).all()
