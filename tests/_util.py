"""Shared helpers of the tests: seeded inputs, the oracle side and comparisons.

The CUDA path is called only through the package binding (which calls the C
ABI); the expected values come only from ``oracle/``.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import oracle as O
from sparse_attention_pool_b200 import synth

SCALE = float(np.float32(1.0 / math.sqrt(128.0)))
TOL_BF16 = 1e-2   # max-abs, bf16 cache, fp32 accumulation
TOL_FP8 = 3e-2    # max-abs, e4m3 cache
TOL_REL = 1e-2    # rms(err) / rms(oracle output), bf16 cache
TOL_REL_FP8 = 3e-2


def bits_to_torch_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def torch_bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


class Inputs:
    """Raw tokens, queries and lengths of one workload (numpy bf16 bit patterns)."""

    def __init__(self, seed, B, Lcap, H, lengths=None, Tq=1, q_scale=1.0):
        self.B, self.Lcap, self.H, self.Tq = B, Lcap, H, Tq
        self.K = synth.normal_bf16(seed, "k", (B, Lcap, 128))
        self.V = synth.normal_bf16(seed, "v", (B, Lcap, 128))
        self.KI = synth.normal_bf16(seed, "kidx", (B, Lcap, 64))
        if Tq == 1:
            self.q = synth.normal_bf16(seed, "q", (B, H, 128), scale=q_scale)
            self.qI = synth.normal_bf16(seed, "qidx", (B, 64))
        else:
            self.q = synth.normal_bf16(seed, "q", (B, Tq, H, 128), scale=q_scale)
            self.qI = synth.normal_bf16(seed, "qidx", (B, Tq, 64))
        self.lengths = np.full((B,), Lcap, dtype=np.int32) if lengths is None else np.asarray(lengths, np.int32)

    def to_device(self, dev="cuda"):
        g = {}
        for name in ("K", "V", "KI", "q", "qI"):
            g[name] = bits_to_torch_bf16(getattr(self, name)).to(dev)
        g["len"] = torch.from_numpy(self.lengths).to(dev)
        return g

    def oracle_seq(self, b, fp8=False, m_csa=4, m_hca=128):
        L = int(self.lengths[b])
        return O.CompressedSeq(self.K[b, :L], self.V[b, :L], self.KI[b, :L], m_csa=m_csa, m_hca=m_hca, fp8=fp8)


def compress_on_gpu(S, g, B, Lcap, fp8=False, m_csa=4, m_hca=128):
    ncap_c, ncap_h = Lcap // m_csa, Lcap // m_hca
    csa = S.alloc_cache(B, ncap_c, m_csa, fp8=fp8, with_kidx=True)
    hca = S.alloc_cache(B, ncap_h, m_hca, fp8=fp8)
    S.csa_compress(g["K"], g["V"], g["KI"], g["len"], csa)
    S.hca_compress(g["K"], g["V"], g["len"], hca)
    return csa, hca


def out_errors(gpu_out: torch.Tensor, ref: np.ndarray):
    """(max |err|, rms(err) / rms(ref))."""
    got = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    mx = float(err.max()) if err.size else 0.0
    rerr = float(np.sqrt(np.mean(err ** 2))) if err.size else 0.0
    return mx, (rerr / rms if rms > 0 else rerr)
