"""The second, third and fourth forms of the prefill selection
(SA_OPT_PREFILL_SELECT = 2, 3, 4) against the oracle and against the first form: the exact top-k of every
query row, ties at the threshold by lowest index, ascending output.  Cases:
every row of a short prefill; equal scores (one crowded bin, larger than
the in-shared-memory list, and ties at the threshold); rows that see more
than the 40,960 keys the kernel stages, whose keys are read from the global
scratch; the FP4 scores; and the hybrid prefill's outputs, identical under
every form.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, Inputs, compress_on_gpu

pytestmark = pytest.mark.gpu

STAGED = 40 * 1024  # keys the second form stages in shared memory


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _topk_forms(S, qI, csa, k, pos, fp4=None):
    """(idx, cnt) under every selection form (1 to 4)."""
    Tq = qI.shape[1]
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, csa.B, Tq, 8, csa.Ncap, 0, k))
    out = []
    for form in (1, 2, 3, 4):
        S.set_option(S.SA_OPT_PREFILL_SELECT, form)
        try:
            if fp4 is None:
                i, c = S.csa_index_topk(qI, csa, k, ws, q_pos=pos)
            else:
                i, c = S.csa_index_topk_mxfp4(qI, csa, fp4[0], fp4[1], k, ws, q_pos=pos)
            S.read_device_status()
        finally:
            S.set_option(S.SA_OPT_PREFILL_SELECT, 4)
        out.append((i.clone(), c.clone()))
    return out


def _all_equal(forms):
    return all(torch.equal(f[0], forms[0][0]) and torch.equal(f[1], forms[0][1]) for f in forms[1:])


def _check_rows(inp, csa_keys, pos, got, k):
    """got[0] = (idx, cnt) of one form; sequence 0's rows against the oracle."""
    gi, gn = got[0][0][0].cpu().numpy(), got[0][1][0].cpu().numpy()  # [Tq][k], [Tq]
    for i, t in enumerate(pos):
        ref, rc = O.topk(O.index_scores(inp.qI[0, i], csa_keys[:t // 4]), k)
        assert gn[i] == rc and np.array_equal(gi[i], ref), (i, t)


def test_every_row_of_a_short_prefill(S):
    B, T, k = 1, 1500, 64
    inp = Inputs(1301, B, T, 8, Tq=T)
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, T)
    pos = list(range(T))
    forms = _topk_forms(S, g["qI"], csa, k, torch.tensor([pos], dtype=torch.int32, device="cuda"))
    assert _all_equal(forms)
    _check_rows(inp, O.compress(inp.KI[0], 4), pos, forms[1:], k)


@pytest.mark.parametrize("k", [77, 2048])
def test_equal_scores_overflow_the_list(S, k):
    # every indexer key equal: one bin of up to 10,000 keys (above the list's
    # 8,192), every selection cut inside the ties
    L = 40000
    inp = Inputs(1302, 1, L, 8, Tq=12)
    inp.KI[:] = inp.KI[:, :1, :]
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, 1, L)
    pos = [4 * k + 4, 4 * k + 7, 9000, 20000, 32768, 33000, 36000, 36001, 38000, 39000, 39996, L - 1]
    forms = _topk_forms(S, g["qI"], csa, k, torch.tensor([pos], dtype=torch.int32, device="cuda"))
    assert _all_equal(forms)
    want = np.arange(k, dtype=np.int32)
    assert (forms[1][0][0].cpu().numpy() == want[None, :]).all() and (forms[1][1] == k).all()


def test_rows_past_the_staged_keys(S):
    L, k = 1 << 18, 2048
    edge = 4 * STAGED
    rng = np.random.default_rng(1303)
    pos = sorted({edge - 4, edge, edge + 3, edge + 4, edge + 7, L - 1,
                  *(int(x) for x in rng.integers(edge - 3000, L, 30))})
    inp = Inputs(1303, 1, L, 8, Tq=len(pos))
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, 1, L)
    forms = _topk_forms(S, g["qI"], csa, k, torch.tensor([pos], dtype=torch.int32, device="cuda"))
    assert _all_equal(forms)
    _check_rows(inp, O.compress(inp.KI[0], 4), pos, forms[1:], k)
    assert sum(t // 4 > STAGED for t in pos) >= 10 and sum(k < t // 4 <= STAGED for t in pos) >= 2


def test_fp4_scores_under_both_forms(S):
    B, T, k = 1, 3000, 128
    inp = Inputs(1304, B, T, 8, Tq=T)
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, T)
    codes, scales = S.csa_index_quantize_mxfp4(csa)
    pos = torch.arange(T, dtype=torch.int32, device="cuda").view(1, T).contiguous()
    assert _all_equal(_topk_forms(S, g["qI"], csa, k, pos, fp4=(codes, scales)))


def test_hybrid_prefill_identical_under_both_forms(S):
    B, T, H, k = 1, 2100, 64, 128
    inp = Inputs(1305, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    res = []
    for form in (1, 2, 3, 4):
        idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
        cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
        S.set_option(S.SA_OPT_PREFILL_SELECT, form)
        try:
            oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE)
            S.read_device_status()
        finally:
            S.set_option(S.SA_OPT_PREFILL_SELECT, 4)
        res.append((oc, oh, idx, cnt))
    for other in res[1:]:
        for a, b in zip(res[0], other):
            assert torch.equal(a, b)
