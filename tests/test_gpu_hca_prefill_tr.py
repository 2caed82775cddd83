"""The dense (HCA) attention of a causal prefill on the tensor cores against
the fp64 oracle, in every kernel form (SA_OPT_HCA_PREFILL: 0 the transposed
kernel, 128 entries per MMA, with two query positions per tile when there
are 64 heads; 1 the two-query kernel, 2 queries x 64 heads as the MMA's M;
2 the transposed kernel one query at a time).  Rows see up to 312 entries
(three 128-entry tiles, the last one ragged) and none before token 128;
heads 64 and, on the transposed kernel, 16; peaky queries.  Outputs: max-abs
<= 1e-2 and rms(err)/rms(oracle) <= 1e-2 (bf16 cache), lse within 1e-3; the
hybrid prefill call gives the standalone call's HCA output bit for bit.
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
    yield S
    S.set_option(S.SA_OPT_HCA_PREFILL, 0)


def _hca(S, inp, form, pos=None):
    B, T, H = inp.B, inp.Lcap, inp.H
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    if pos is None:
        pos = torch.arange(T, dtype=torch.int32, device="cuda").repeat(B, 1).contiguous()
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_DENSE_ATTN, B, T, H, 0, hca.Ncap, 0))
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    S.set_option(S.SA_OPT_HCA_PREFILL, form)
    try:
        out = S.hca_dense_attn(g["q"], hca, ws, q_pos=pos, scale=SCALE, lse=lse)
        S.read_device_status()
    finally:
        S.set_option(S.SA_OPT_HCA_PREFILL, 0)
    return g, csa, hca, out, lse


def _check(inp, out, lse, rows, b=0, pos=None):
    cs = inp.oracle_seq(b)
    of, lf = out[b].float().cpu().numpy(), lse[b].cpu().numpy()
    for t in rows:
        tp = int(t) if pos is None else int(pos[b, t])
        n = min(tp // 128, cs.n_hca)
        if n == 0:
            assert not of[t].any() and np.isneginf(lf[t]).all(), t
            continue
        ro, rl = O.attention(inp.q[b, t], cs.hk, cs.hv, range(n), SCALE)
        mx, rel = out_errors(torch.from_numpy(of[t]), ro)
        assert mx <= TOL_BF16 and rel <= TOL_REL, (t, mx, rel)
        assert np.abs(lf[t] - rl).max() < 1e-3, t


def _rows(T, rng, count):
    edges = {0, 1, 127, 128, 129, 255, 256, 16383, 16384, 16385, 32767, 32768, T - 2, T - 1}
    return sorted({t for t in edges if 0 <= t < T} | set(rng.choice(T, count, replace=False).tolist()))


@pytest.mark.parametrize("form", [0, 1, 2])
def test_long_rows_sampled(S, form):
    B, T, H = 2, 40000, 64
    inp = Inputs(7501, B, T, H, Tq=T)
    _, _, _, out, lse = _hca(S, inp, form)
    rng = np.random.default_rng(11)
    for b in range(B):
        _check(inp, out, lse, _rows(T, rng, 100), b=b)


def test_sixteen_heads_transposed(S):
    B, T, H = 1, 33000, 16
    inp = Inputs(7502, B, T, H, Tq=T)
    _, _, _, out, lse = _hca(S, inp, 0)
    _check(inp, out, lse, _rows(T, np.random.default_rng(12), 150))


@pytest.mark.parametrize("form", [0, 1, 2])
def test_peaky_queries(S, form):
    B, T, H = 1, 20000, 64
    inp = Inputs(7503, B, T, H, Tq=T, q_scale=8.0)
    _, _, _, out, lse = _hca(S, inp, form)
    _check(inp, out, lse, _rows(T, np.random.default_rng(13), 150))


@pytest.mark.parametrize("form", [0, 2])
def test_every_row_short(S, form):
    # every row of a short prefill (entries 0 .. 23) on the transposed kernel;
    # T odd: the last position has no partner in the paired form
    B, T, H = 1, 3101, 64
    inp = Inputs(7504, B, T, H, Tq=T)
    _, _, _, out, lse = _hca(S, inp, form)
    _check(inp, out, lse, range(T))


def test_pairs_with_unequal_positions(S):
    # positions that are not consecutive: the two queries of a tile see
    # different entry counts (and some see none), so each masks its own
    B, T, H = 2, 20000, 64
    inp = Inputs(7506, B, T, H, Tq=T)
    rng = np.random.default_rng(14)
    pos = torch.from_numpy(rng.integers(0, T, size=(B, T), dtype=np.int32)).cuda()
    _, _, _, out, lse = _hca(S, inp, 0, pos=pos)
    posh = pos.cpu().numpy()
    for b in range(B):
        _check(inp, out, lse, _rows(T, rng, 120), b=b, pos=posh)


def test_forms_agree_and_hybrid_equals_standalone(S):
    B, T, H, k = 1, 17000, 64, 256
    inp = Inputs(7505, B, T, H, Tq=T)
    g, csa, hca, o0, l0 = _hca(S, inp, 0)
    fin = torch.isfinite(l0)
    for form in (1, 2):
        _, _, _, o1, l1 = _hca(S, inp, form)
        assert (o0.float() - o1.float()).abs().max().item() <= 2 * TOL_BF16
        assert torch.equal(fin, torch.isfinite(l1)) and (l0[fin] - l1[fin]).abs().max().item() < 1e-3
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
    _, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE)
    S.read_device_status()
    assert torch.equal(oh, o0)
