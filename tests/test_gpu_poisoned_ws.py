"""Reads of scratch that a call never wrote: every call is repeated with its
workspace filled with 0xFF bytes and must give the zeroed workspace's results
bit for bit (decode with bf16 and e4m3 caches, the FP4 selection, causal
prefill), also when the poisoned workspace first served a larger call.
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


def _decode(S, g, csa, hca, k, ws, H, B, codes=None, scales=None):
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    lh = torch.empty_like(lc)
    if codes is None:
        oc, oh = S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE, lse_csa=lc, lse_hca=lh,
                                      idx_out=idx, cnt_out=cnt)
    else:
        oc, oh = S.hybrid_attn_decode_mxfp4(g["q"], g["qI"], csa, hca, codes, scales, k, ws, scale=SCALE,
                                            lse_csa=lc, lse_hca=lh, idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    return [oc, oh, lc, lh, idx, cnt]


@pytest.mark.parametrize("fp8,fp4", [(False, False), (True, False), (False, True)])
def test_decode_with_a_poisoned_workspace(S, fp8, fp4):
    B, Lcap, H, k = 3, 30000, 64, 512
    inp = Inputs(971, B, Lcap, H, lengths=[30000, 12345, 400])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap, fp8=fp8)
    codes, scales = S.csa_index_quantize_mxfp4(csa) if fp4 else (None, None)
    size = S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k)
    clean = _decode(S, g, csa, hca, k, S.alloc_workspace(size), H, B, codes, scales)
    ws = S.alloc_workspace(size)
    ws.fill_(0xFF)
    assert all(torch.equal(a, b) for a, b in zip(clean, _decode(S, g, csa, hca, k, ws, H, B, codes, scales)))
    # the same scratch after a call with other lengths and k
    g2 = dict(g)
    g2["len"] = torch.tensor([29000, 30000, 20000], dtype=torch.int32, device="cuda")
    csa2, hca2 = compress_on_gpu(S, g2, B, Lcap, fp8=fp8)
    _decode(S, g2, csa2, hca2, 64, ws, H, B)
    assert all(torch.equal(a, b) for a, b in zip(clean, _decode(S, g, csa, hca, k, ws, H, B, codes, scales)))


def test_prefill_with_a_poisoned_workspace(S):
    B, T, H, k = 1, 3000, 64, 128
    inp = Inputs(972, B, T, H, Tq=T)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, T)
    size = S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k)
    res = []
    for poison in (False, True):
        ws = S.alloc_workspace(size)
        if poison:
            ws.fill_(0xFF)
        idx = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
        cnt = torch.empty(B, T, dtype=torch.int32, device="cuda")
        oc, oh = S.hybrid_attn_prefill(g["q"], g["qI"], csa, hca, k, ws, idx, cnt, scale=SCALE)
        S.read_device_status()
        res.append((oc, oh, idx, cnt))
    assert all(torch.equal(a, b) for a, b in zip(*res))
