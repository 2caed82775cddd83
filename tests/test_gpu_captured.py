"""CapturedDecode: the hybrid decode step captured once into a CUDA graph.
Replays with new queries (copied in from pinned host memory) must give the
eager call's outputs bit for bit, and must see cache appends made between
steps.
"""
from __future__ import annotations


import pytest
import torch

from tests._util import SCALE, Inputs, compress_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _eager(S, q, qI, csa, hca, k):
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, csa.B, 1, q.shape[1], csa.Ncap, hca.Ncap, k))
    idx = torch.empty(csa.B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(csa.B, dtype=torch.int32, device="cuda")
    oc, oh = S.hybrid_attn_decode(q, qI, csa, hca, k, ws, scale=SCALE, idx_out=idx, cnt_out=cnt)
    return oc, oh, idx


def test_replays_equal_eager_calls_and_see_appends(S):
    B, Lcap, H, k = 2, 20000, 64, 512
    inp = Inputs(941, B, Lcap, H, lengths=[12000, 7000])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    cap = S.CapturedDecode(csa, hca, k, H, scale=SCALE)
    oc_pin = torch.empty(B, H, 128, dtype=torch.int16).pin_memory()
    for step in range(3):
        q = torch.randn(B, H, 128, device="cuda").to(torch.bfloat16)
        qI = torch.randn(B, 64, device="cuda").to(torch.bfloat16)
        q_pin = q.view(torch.int16).cpu().pin_memory()
        qi_pin = qI.view(torch.int16).cpu().pin_memory()
        cap.step(q_pin, qi_pin, out_csa=oc_pin)
        torch.cuda.synchronize()
        oc, oh, idx = _eager(S, q, qI, csa, hca, k)
        assert torch.equal(cap.out_csa, oc) and torch.equal(cap.out_hca, oh) and torch.equal(cap.idx, idx), step
        assert torch.equal(oc_pin, oc.view(torch.int16).cpu()), step
        # the sequences grow between steps: the graph reads the caches in place
        lens = torch.tensor([12000 + 700 * (step + 1), 7000 + 300 * (step + 1)], dtype=torch.int32, device="cuda")
        S.csa_append(g["K"], g["V"], g["KI"], lens, csa, 700)
        S.hca_append(g["K"], g["V"], lens, hca, 700)
    S.read_device_status()
