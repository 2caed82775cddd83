"""hybrid_attn_decode_swa: one decode step whose CSA and HCA outputs each
include the sliding window over the last raw tokens, against the oracle's
attention over the union of each branch's entries and the window.
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


@pytest.mark.parametrize("w", [128, 64])
def test_both_branches_with_the_window_match_the_oracle(S, w):
    B, Lcap, H, k = 3, 6000, 64, 256
    inp = Inputs(951 + w, B, Lcap, H, lengths=[6000, 2999, 90])  # 90 < window: every raw token
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE_SWA, B, 1, H, csa.Ncap, hca.Ncap, k))
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty_like(lc)
    oc, oh = S.hybrid_attn_decode_swa(g["q"], g["qI"], csa, hca, g["K"], g["V"], g["len"], w, k, ws, scale=SCALE,
                                      lse_csa=lc, lse_hca=lh)
    S.read_device_status()
    for b in range(B):
        L = int(inp.lengths[b])
        cs = inp.oracle_seq(b)
        r = O.hybrid_query(cs, inp.q[b], inp.qI[b], t=L, k=k, scale=SCALE)
        win = (inp.K[b], inp.V[b], O.window_rows(L, L, w))
        ref_c, ref_lc = O.union_attention(inp.q[b], [(cs.ck, cs.cv, r["idx"][:r["cnt"]]), win], SCALE)
        ref_h, ref_lh = O.union_attention(inp.q[b], [(cs.hk, cs.hv, np.arange(cs.n_hca)), win], SCALE)
        assert np.abs(oc[b].float().cpu().numpy() - ref_c).max() <= TOL_BF16, b
        assert np.abs(oh[b].float().cpu().numpy() - ref_h).max() <= TOL_BF16, b
        assert np.abs(lc[b].cpu().numpy() - ref_lc).max() < 1e-3, b
        assert np.abs(lh[b].cpu().numpy() - ref_lh).max() < 1e-3, b
    # without lse outputs the call keeps its own
    oc2, oh2 = S.hybrid_attn_decode_swa(g["q"], g["qI"], csa, hca, g["K"], g["V"], g["len"], w, k, ws, scale=SCALE)
    S.read_device_status()
    assert torch.equal(oc2, oc) and torch.equal(oh2, oh)
