"""Failure detection without a GPU fault: a kernel whose bounded wait cannot
complete (a barrier that nothing arrives at) gives up, records a timeout in
the device status word and returns; the host reads SA_ERR_TIMEOUT, the word
is cleared, and the context keeps computing correct results.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import SCALE, Inputs, compress_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def test_a_wait_that_runs_out_is_reported_and_the_context_survives(S):
    S.read_device_status()  # start clean
    S.selftest_wait_timeout(1 << 14)
    with pytest.raises(S.SparseAttnError) as e:
        S.read_device_status()
    assert "SA_ERR_TIMEOUT" in str(e.value)
    S.read_device_status()  # cleared
    # the context still computes: one small decode step against the oracle
    B, L, H, k = 1, 4096, 8, 64
    inp = Inputs(961, B, L, H)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, L)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    r = O.hybrid_query(inp.oracle_seq(0), inp.q[0], inp.qI[0], t=L, k=k, scale=SCALE)
    assert np.array_equal(idx[0].cpu().numpy(), r["idx"])
