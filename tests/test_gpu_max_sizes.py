"""The library's limits on one B200, against the oracle: the largest k the
entry points accept (65,536) at a 1M-token context, k above the entry count,
and prefill rows that see more indexer entries than the selection kernel
stages in shared memory (49,152), so that the keys are read from the global
scratch instead.

Indices: bit-exact.  Outputs: max-abs <= 1e-2 and rms(err)/rms(oracle) <=
1e-2 (bf16 cache).  The oracle builds its own caches from the same seeded raw
tokens.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, TOL_BF16, TOL_REL, Inputs, compress_on_gpu, out_errors

pytestmark = pytest.mark.gpu

K_MAX = 65536
SELECT_SMEM_KEYS = 49152  # keys the prefill selection stages in shared memory


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _check(got, ref):
    mx, rel = out_errors(got, ref)
    assert mx <= TOL_BF16 and rel <= TOL_REL, (mx, rel)


def _hybrid_decode(S, inp, k):
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, inp.B, inp.Lcap)
    B, H = inp.B, inp.H
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, idx_out=idx,
                                  cnt_out=cnt)
    S.read_device_status()
    return oc, oh, lc, idx, cnt


@pytest.mark.parametrize("L", [1 << 20, 200_000])  # 262,144 entries > k; 50,000 entries < k
def test_hybrid_decode_at_the_largest_k(S, L):
    inp = Inputs(1201, 1, L, 64)
    oc, oh, lc, idx, cnt = _hybrid_decode(S, inp, K_MAX)
    r = O.hybrid_query(inp.oracle_seq(0), inp.q[0], inp.qI[0], t=L, k=K_MAX, scale=SCALE)
    assert int(cnt[0]) == r["cnt"] == min(K_MAX, L // 4)
    assert np.array_equal(idx[0].cpu().numpy(), r["idx"])
    _check(oc[0], r["out_csa"])
    _check(oh[0], r["out_hca"])
    assert np.abs(lc[0].cpu().numpy() - r["lse_csa"]).max() < 1e-3


@pytest.mark.parametrize("k", [2048, 40000])
def test_prefill_rows_past_the_staged_keys(S, k):
    """Query rows whose visible entries (t // 4) straddle the selection's
    shared-memory staging: up to 49,152 keys staged, beyond that read from
    the global scratch; every row bit-exact against the oracle."""
    L = 1 << 18
    edge = 4 * SELECT_SMEM_KEYS
    rng = np.random.default_rng(1202)
    pos = sorted({edge - 4, edge - 1, edge, edge + 3, edge + 4, edge + 5, L - 1,
                  *(int(x) for x in rng.integers(edge - 4000, L, 40))})
    Tq = len(pos)
    inp = Inputs(1202, 1, L, 8, Tq=Tq)
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, 1, L)
    qpos = torch.tensor([pos], dtype=torch.int32, device="cuda")
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, 1, Tq, 8, csa.Ncap, 0, k))
    idx, cnt = S.csa_index_topk(g["qI"], csa, k, ws, q_pos=qpos)
    S.read_device_status()
    ci = O.compress(inp.KI[0], 4)
    gi, gn = idx[0].cpu().numpy(), cnt[0].cpu().numpy()
    staged = global_ = 0
    for i, t in enumerate(pos):
        nv = t // 4
        ref, rc = O.topk(O.index_scores(inp.qI[0, i], ci[:nv]), k)
        assert gn[i] == rc and np.array_equal(gi[i], ref), (i, t)
        if nv > k:
            staged += nv <= SELECT_SMEM_KEYS
            global_ += nv > SELECT_SMEM_KEYS
    assert staged >= 2 and global_ >= 10  # both paths ran
