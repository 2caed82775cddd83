"""The five workloads at full size, in the launch configuration the bench
times, checked against the fp64 oracle on sampled sequences / query rows.

Indices: bit-exact.  Outputs: max-abs <= 1e-2 (bf16 cache) or 3e-2 (fp8),
rms(err)/rms(oracle) <= 1e-2 (bf16) or 3e-2 (fp8).  The oracle builds its own
caches from the same seeded raw tokens (nothing here comes from the GPU).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_attention_pool_b200 import configs, synth
from tests._util import (SCALE, TOL_BF16, TOL_FP8, TOL_REL, TOL_REL_FP8, bits_to_torch_bf16, out_errors)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_pool_b200 as S
    return S


def _workload_inputs(w):
    seed = synth.BASE_SEED + w.index
    if w.L_min is not None:
        lengths = synth.ragged_lengths(seed, w.B, w.L_min, w.L)
    else:
        lengths = np.full((w.B,), w.L, dtype=np.int32)
    K = synth.normal_bf16(seed, "k", (w.B, w.L, 128))
    V = synth.normal_bf16(seed, "v", (w.B, w.L, 128))
    KI = synth.normal_bf16(seed, "kidx", (w.B, w.L, 64))
    if w.mode == "decode":
        q = synth.normal_bf16(seed, "q", (w.B, w.H, 128))
        qI = synth.normal_bf16(seed, "qidx", (w.B, 64))
    else:
        q = synth.normal_bf16(seed, "q", (w.B, w.L, w.H, 128))
        qI = synth.normal_bf16(seed, "qidx", (w.B, w.L, 64))
    return lengths, K, V, KI, q, qI


def _compress(S, w, lengths, K, V, KI):
    dev = "cuda"
    Kd, Vd, KId = bits_to_torch_bf16(K).to(dev), bits_to_torch_bf16(V).to(dev), bits_to_torch_bf16(KI).to(dev)
    lens = torch.from_numpy(lengths).to(dev)
    csa = S.alloc_cache(w.B, w.L // w.m_csa, w.m_csa, fp8=w.fp8, with_kidx=True)
    hca = S.alloc_cache(w.B, w.L // w.m_hca, w.m_hca, fp8=w.fp8)
    S.csa_compress(Kd, Vd, KId, lens, csa)
    S.hca_compress(Kd, Vd, lens, hca)
    torch.cuda.synchronize()
    del Kd, Vd, KId
    return csa, hca


def _check(got, ref, fp8):
    mx, rel = out_errors(got, ref)
    assert mx <= (TOL_FP8 if fp8 else TOL_BF16), (mx, rel)
    assert rel <= (TOL_REL_FP8 if fp8 else TOL_REL), (mx, rel)


@pytest.mark.parametrize("name,sample", [
    ("decode_b16_t64k_h64_k512", [0, 7, 15]),
    ("decode_b4_t1m_h64_k2048", [0, 3]),
    ("ragged_fp8_b32_t64k-256k_h64_k1024", None),   # shortest, longest and one more
])
def test_decode_workload_full_size(S, name, sample):
    w = configs.BY_NAME[name]
    lengths, K, V, KI, q, qI = _workload_inputs(w)
    csa, hca = _compress(S, w, lengths, K, V, KI)
    B, H, k = w.B, w.H, w.topk
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    lc = torch.empty(B, H, dtype=torch.float32, device="cuda")
    oc, oh = S.hybrid_attn_decode(bits_to_torch_bf16(q).cuda(), bits_to_torch_bf16(qI).cuda(), csa, hca, k, ws,
                                  scale=SCALE, lse_csa=lc, idx_out=idx, cnt_out=cnt)
    S.read_device_status()
    if sample is None:
        order = np.argsort(lengths)
        sample = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2])})
    for b in sample:
        Lb = int(lengths[b])
        cs = O.CompressedSeq(K[b, :Lb], V[b, :Lb], KI[b, :Lb], fp8=w.fp8)
        r = O.hybrid_query(cs, q[b], qI[b], t=Lb, k=k, scale=SCALE)
        assert cnt[b].item() == r["cnt"]
        assert np.array_equal(idx[b].cpu().numpy(), r["idx"]), b
        _check(oc[b], r["out_csa"], w.fp8)
        _check(oh[b], r["out_hca"], w.fp8)
        assert np.abs(lc[b].cpu().numpy() - r["lse_csa"]).max() < 1e-3


def test_prefill_workload_full_size_sampled_rows(S):
    w = configs.BY_NAME["prefill_b1_t128k_h64_k2048"]
    lengths, K, V, KI, q, qI = _workload_inputs(w)
    csa, hca = _compress(S, w, lengths, K, V, KI)
    T, H, k = w.L, w.H, w.topk
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, 1, T, H, csa.Ncap, hca.Ncap, k))
    idx = torch.empty(1, T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, T, dtype=torch.int32, device="cuda")
    qd = bits_to_torch_bf16(q).cuda()
    qId = bits_to_torch_bf16(qI).cuda()
    oc, oh = S.hybrid_attn_prefill(qd, qId, csa, hca, k, ws, idx, cnt, scale=SCALE)
    S.read_device_status()
    rng = np.random.default_rng(4)
    rows = sorted({0, 3, 4, 5, 127, 128, 129, 8191, 8192, 8195, 8196, 8200, 65536, T - 1,
                   *rng.integers(0, T, size=10).tolist()})
    cs = O.CompressedSeq(K[0], V[0], KI[0])
    idx_h = idx[0].cpu().numpy()
    cnt_h = cnt[0].cpu().numpy()
    for t in rows:
        r = O.hybrid_query(cs, q[0, t], qI[0, t], t=t, k=k, scale=SCALE)
        assert cnt_h[t] == r["cnt"], t
        assert np.array_equal(idx_h[t], r["idx"]), t
        _check(oc[0, t], r["out_csa"], False)
        _check(oh[0, t], r["out_hca"], False)
    # every row's count follows the causal rule min(k, t // 4)
    t_all = np.arange(T)
    assert np.array_equal(cnt_h, np.minimum(k, t_all // 4))
