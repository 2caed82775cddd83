"""CapturedDecode and DecodeGraph: the hybrid decode step captured once into
a CUDA graph (by torch, or by the library together with its packed host
copies).  Replays with new queries (copied in from pinned host memory) must
give the eager call's outputs bit for bit, and must see cache appends made
between steps.
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
    lc = torch.empty(csa.B, q.shape[1], dtype=torch.float32, device="cuda")
    lh = torch.empty_like(lc)
    oc, oh = S.hybrid_attn_decode(q, qI, csa, hca, k, ws, scale=SCALE, idx_out=idx, cnt_out=cnt, lse_csa=lc,
                                  lse_hca=lh)
    return oc, oh, idx, cnt, lc, lh


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
        oc, oh, idx, _, _, _ = _eager(S, q, qI, csa, hca, k)
        assert torch.equal(cap.out_csa, oc) and torch.equal(cap.out_hca, oh) and torch.equal(cap.idx, idx), step
        assert torch.equal(oc_pin, oc.view(torch.int16).cpu()), step
        # the sequences grow between steps: the graph reads the caches in place
        lens = torch.tensor([12000 + 700 * (step + 1), 7000 + 300 * (step + 1)], dtype=torch.int32, device="cuda")
        S.csa_append(g["K"], g["V"], g["KI"], lens, csa, 700)
        S.hca_append(g["K"], g["V"], lens, hca, 700)
    S.read_device_status()


@pytest.mark.parametrize("decode_fast,flags", [(0, 0), (0, 1), (0, 2), (0, 3), (1, 3)])
def test_decode_graph_equals_eager_calls_and_sees_appends(S, decode_fast, flags):
    # the library's own graph: packed queries in, both outputs and both lse
    # out, one launch per step; the options in force at capture are kept
    B, Lcap, H, k = 3, 40000, 64, 1024
    inp = Inputs(943, B, Lcap, H, lengths=[30000, 21000, 9001])
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    S.set_option(S.SA_OPT_DECODE_FAST, decode_fast)
    try:
        dg = S.DecodeGraph(csa, hca, k, H, scale=SCALE, flags=flags)
    finally:
        S.set_option(S.SA_OPT_DECODE_FAST, 0)
    assert dg.h2d_bytes >= B * (H * 128 + 64) * 2 and dg.d2h_bytes >= 2 * B * H * (128 * 2 + 4)
    for step in range(3):
        q = torch.randn(B, H, 128, device="cuda").to(torch.bfloat16)
        qI = torch.randn(B, 64, device="cuda").to(torch.bfloat16)
        dg.q.copy_(q.cpu())
        dg.q_idx.copy_(qI.cpu())
        dg.host_out.fill_(0xFF)
        dg.step()
        torch.cuda.synchronize()
        oc, oh, idx, cnt, lc, lh = _eager(S, q, qI, csa, hca, k)
        torch.cuda.synchronize()
        assert torch.equal(dg.idx, idx) and torch.equal(dg.cnt, cnt), step
        assert torch.equal(dg.out_csa.view(torch.int16), oc.view(torch.int16).cpu()), step
        assert torch.equal(dg.out_hca.view(torch.int16), oh.view(torch.int16).cpu()), step
        assert torch.equal(dg.lse_csa.view(torch.int32), lc.view(torch.int32).cpu()), step
        assert torch.equal(dg.lse_hca.view(torch.int32), lh.view(torch.int32).cpu()), step
        lens = torch.tensor([30000 + 900 * (step + 1), 21000 + 128 * (step + 1), 9001 + 4 * (step + 1)],
                            dtype=torch.int32, device="cuda")
        S.csa_append(g["K"], g["V"], g["KI"], lens, csa, 900)
        S.hca_append(g["K"], g["V"], lens, hca, 900)
    dg.close()
    S.read_device_status()


def test_decode_graph_rejects_pageable_host_memory(S):
    B, Lcap, H, k = 1, 4096, 8, 64
    inp = Inputs(945, B, Lcap, H)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    io = S.decode_io_layout(B, H)
    from sparse_attention_pool_b200 import _lib
    import ctypes
    pageable = torch.zeros(io.in_bytes + io.out_bytes, dtype=torch.uint8)
    din = torch.zeros(io.in_bytes, dtype=torch.uint8, device="cuda")
    dout = torch.zeros(io.out_bytes, dtype=torch.uint8, device="cuda")
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    cs, hs = csa.struct(), hca.struct()
    h = ctypes.c_void_p()
    L = _lib.lib()
    st = L.sa_decode_graph_create(ctypes.byref(cs), ctypes.byref(hs), H, k, 0.0, None, None,
                                  ctypes.c_void_p(pageable.data_ptr()),
                                  ctypes.c_void_p(pageable.data_ptr() + io.in_bytes), ctypes.c_void_p(din.data_ptr()),
                                  ctypes.c_void_p(dout.data_ptr()), None, None, ctypes.c_void_p(ws.data_ptr()),
                                  ws.numel(), 0, ctypes.byref(h))
    assert st == _lib.SA_ERR_INVALID_ARG and not h.value
    assert "pinned" in L.sa_last_error().decode()


def test_decode_graph_rejects_unknown_flags(S):
    B, Lcap, H, k = 1, 4096, 8, 64
    inp = Inputs(947, B, Lcap, H)
    g = inp.to_device()
    csa, hca = compress_on_gpu(S, g, B, Lcap)
    with pytest.raises(S.SparseAttnError, match="flags"):
        S.DecodeGraph(csa, hca, k, H, flags=4)
