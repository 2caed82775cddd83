"""The gathered (CSA) attention of a causal prefill on the tensor cores
(tcgen05, transposed tiles: 128 list entries x 64 heads per MMA) against the
fp64 oracle.  Every query position has its own top-k list; the kernel walks
it in tiles of 128 entries with an online softmax per head.  Cases: lists of
several tiles with a ragged last tile, rows that see fewer entries than k
(including none), fewer than 64 heads (the missing heads' MMA columns are
zero), peaky queries, and the standalone csa_sparse_attn call.  Outputs:
max-abs <= 1e-2 and rms(err)/rms(oracle) <= 1e-2 (bf16 cache), lse within
1e-3; indices bit-exact.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, TOL_BF16, TOL_REL, Inputs, compress_on_gpu, out_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _prefill(S, inp, k):
    B, T, H = inp.B, inp.Lcap, inp.H
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    oc, _ = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE, lse_csa=lc)
    S.read_device_status()
    return g, csa, oc, lc, idx, cnt


def _check_rows(inp, k, oc, lc, idx, cnt, rows, b=0):
    cs = inp.oracle_seq(b)
    ocf, lcf = oc[b].float().cpu().numpy(), lc[b].cpu().numpy()
    idx_h, cnt_h = idx[b].cpu().numpy(), cnt[b].cpu().numpy()
    for t in rows:
        r = O.hybrid_query(cs, inp.q[b, t], inp.qI[b, t], t=int(t), k=k, scale=SCALE)
        assert cnt_h[t] == r["cnt"] and np.array_equal(idx_h[t], r["idx"]), t
        if r["cnt"] == 0:
            assert not ocf[t].any() and np.isneginf(lcf[t]).all(), t
            continue
        mx, rel = out_errors(torch.from_numpy(ocf[t]), r["out_csa"])
        assert mx <= TOL_BF16 and rel <= TOL_REL, (t, mx, rel)
        assert np.abs(lcf[t] - r["lse_csa"]).max() < 1e-3, t


@pytest.mark.parametrize("H,k,T", [(64, 300, 2600), (16, 200, 1500)])
def test_every_row(S, H, k, T):
    inp = Inputs(7100 + H + k, 1, T, H, Tq=T)
    _, _, oc, lc, idx, cnt = _prefill(S, inp, k)
    _check_rows(inp, k, oc, lc, idx, cnt, range(T))


def test_long_lists_sampled_rows(S):
    # k = 1000: eight tiles per full list (the last one ragged)
    B, T, H, k = 2, 9000, 64, 1000
    inp = Inputs(7201, B, T, H, Tq=T)
    _, _, oc, lc, idx, cnt = _prefill(S, inp, k)
    rng = np.random.default_rng(3)
    rows = sorted(set(rng.choice(T, 120, replace=False).tolist()) | {0, 3, 4, 127, 128, 3999, 4000, 4003, T - 1})
    for b in range(B):
        _check_rows(inp, k, oc, lc, idx, cnt, rows, b=b)


def test_peaky_queries(S):
    B, T, H, k = 1, 3000, 64, 256
    inp = Inputs(7301, B, T, H, Tq=T, q_scale=8.0)
    _, _, oc, lc, idx, cnt = _prefill(S, inp, k)
    _check_rows(inp, k, oc, lc, idx, cnt, range(0, T, 7))


def test_standalone_sparse_attention(S):
    # csa_sparse_attn over the prefill's lists gives the hybrid call's outputs bit for bit
    B, T, H, k = 1, 2000, 64, 160
    inp = Inputs(7401, B, T, H, Tq=T)
    g, csa, oc, lc, idx, cnt = _prefill(S, inp, k)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_SPARSE_ATTN, B, T, H, csa.Ncap, 0, k))
    o2 = S.csa_sparse_attn(g["q"], csa, idx, cnt, k, ws, scale=SCALE)
    S.read_device_status()
    assert torch.equal(o2, oc)
