"""csa_index_topk_noalloc: the decode top-k for callers that cannot allocate.

Some callers cannot hand the library a workspace: a C caller that only holds
its input and output buffers, or a serving loop whose device memory belongs
to another allocator and which may not call cudaMalloc (the call can also
synchronise the device).  For them the library keeps a static device scratch
array of SA_NOALLOC_SCRATCH_BYTES per GPU.  These tests check that the
variant gives exactly the indices of csa_index_topk on two calls in a row
(the second with a different query, so leftovers of the first cannot
matter), and that requests too large for the array are refused up front.

This file is collected last on purpose.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from sparse_attention_pool_b200 import _lib


def test_noalloc_refuses_requests_larger_than_the_static_scratch():
    L = _lib.lib()
    fake = 0x10000  # aligned and never dereferenced: the size check fails first
    c = _lib.SaCache(fake, fake, None, None, fake, fake, 64, 1 << 20, 128, 64, 4, _lib.SA_BF16)
    P = ctypes.c_void_p
    st = L.csa_index_topk_noalloc(P(fake), ctypes.byref(c), 2048, P(fake), P(fake), None)
    assert st == _lib.SA_ERR_UNSUPPORTED
    msg = L.sa_last_error().decode()
    assert "static scratch" in msg and str(_lib.SA_NOALLOC_SCRATCH_BYTES) in msg


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    from sparse_attention_pool_b200 import synth
    from tests._util import Inputs, bits_to_torch_bf16, compress_on_gpu

    B, Lcap, H, k = 3, 50000, 8, 500
    inp = Inputs(901, B, Lcap, H, lengths=[50000, 41234, 30001])
    g = inp.to_device()
    csa, _ = compress_on_gpu(S, g, B, Lcap)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, 1, H, csa.Ncap, 0, k))
    q2 = bits_to_torch_bf16(synth.normal_bf16(902, "qidx", (B, 64))).cuda()
    for qI in (g["qI"], q2):
        ref_idx, ref_cnt = S.csa_index_topk(qI, csa, k, ws)
        idx, cnt = S.csa_index_topk_noalloc(qI, csa, k)
        S.read_device_status()
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx, ref_idx)  # integer results: exact
