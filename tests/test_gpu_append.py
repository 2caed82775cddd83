"""Compress-when-ready: csa_append / hca_append bring a cache up to date with
grown raw sequences and must give exactly the bits of a full compression of
the new lengths (bf16 and fp8; growth of one token at a time across block and
64-entry group boundaries, and larger jumps), plus the oracle's compression.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests._util import Inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _caches(S, B, Lcap, fp8):
    return (S.alloc_cache(B, Lcap // 4, 4, fp8=fp8, with_kidx=True), S.alloc_cache(B, Lcap // 128, 128, fp8=fp8))


def _same(a, b):
    assert torch.equal(a.n, b.n)
    nmax = int(a.n.max().item())
    for name in ("k", "v", "kidx"):
        x, y = getattr(a, name), getattr(b, name)
        if x is None:
            continue
        for s in range(a.B):
            ns = int(a.n[s].item())
            assert torch.equal(x[s, :ns], y[s, :ns]), (name, s)
    if a.fp8:
        for name in ("k_scale", "v_scale"):
            x, y = getattr(a, name), getattr(b, name)
            for s in range(a.B):
                ng = (int(a.n[s].item()) + 63) // 64
                assert torch.equal(x[s, :ng], y[s, :ng]), (name, s)
    return nmax


@pytest.mark.parametrize("fp8", [False, True])
def test_append_equals_full_compression(S, fp8):
    B, Lcap = 3, 20000
    start = [1000, 255, 16383]
    inp = Inputs(801 + fp8, B, Lcap, 8, lengths=[Lcap] * B)
    g = inp.to_device()
    lens = torch.tensor(start, dtype=torch.int32, device="cuda")
    csa, hca = _caches(S, B, Lcap, fp8)
    S.csa_compress(g["K"], g["V"], g["KI"], lens, csa)
    S.hca_compress(g["K"], g["V"], lens, hca)
    cur = list(start)
    # one token at a time (crosses CSA blocks and, for sequence 1, a 64-entry
    # group at 256 tokens), then jumps that cross HCA blocks and many groups
    steps = [1] * 10 + [3, 120, 129, 1024, 2500]
    for d in steps:
        cur = [min(Lcap, c + d) for c in cur]
        lens = torch.tensor(cur, dtype=torch.int32, device="cuda")
        S.csa_append(g["K"], g["V"], g["KI"], lens, csa, d)
        S.hca_append(g["K"], g["V"], lens, hca, d)
        S.read_device_status()
        ref_c, ref_h = _caches(S, B, Lcap, fp8)
        S.csa_compress(g["K"], g["V"], g["KI"], lens, ref_c)
        S.hca_compress(g["K"], g["V"], lens, ref_h)
        _same(csa, ref_c)
        _same(hca, ref_h)
    assert csa.n.cpu().tolist() == [c // 4 for c in cur]
    # and the oracle's own compression of the final lengths (sequence 2)
    b, L = 2, cur[2]
    kc = O.compress(inp.K[b, :L], 4)
    if not fp8:
        assert np.array_equal(csa.k[b, :L // 4].view(torch.int16).cpu().numpy().view(np.uint16), kc)
    else:
        codes, scales = O.fp8_quantize(kc)
        assert np.array_equal(csa.k[b, :L // 4].cpu().numpy(), codes)
        assert np.array_equal(csa.k_scale[b, :len(scales)].cpu().numpy(), scales.astype(np.float32))


def test_append_beyond_the_bound_is_flagged_and_partial(S):
    B, Lcap = 1, 8192
    inp = Inputs(811, B, Lcap, 8, lengths=[Lcap])
    g = inp.to_device()
    csa, _ = _caches(S, B, Lcap, False)
    S.csa_compress(g["K"], g["V"], g["KI"], torch.tensor([100], dtype=torch.int32, device="cuda"), csa)
    # grows by 2000 tokens (500 entries) while the bound says 4: the launch
    # covers the group of entry 25 and one more (entries < 128)
    lens = torch.tensor([2100], dtype=torch.int32, device="cuda")
    S.csa_append(g["K"], g["V"], g["KI"], lens, csa, 4)
    with pytest.raises(S.SparseAttnError) as e:
        S.read_device_status()
    assert "SA_ERR_DEVICE" in str(e.value)
    assert csa.n.item() == 128
    ref, _ = _caches(S, B, Lcap, False)
    S.csa_compress(g["K"], g["V"], g["KI"], torch.tensor([512], dtype=torch.int32, device="cuda"), ref)
    assert torch.equal(csa.k[0, :128], ref.k[0, :128])
    S.read_device_status()  # cleared
