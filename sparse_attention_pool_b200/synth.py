"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds only the input recipe -- random numbers, rounded to bf16 --
and none of the method's arithmetic.  Both the CUDA path and the CPU oracle
consume exactly these arrays.

Recipe: every tensor is filled from independent chunks of 2**22 values; chunk
``c`` of tensor ``name`` of sequence ``b`` draws float32 standard normals from
numpy's PCG64 seeded with ``SeedSequence([seed, TENSOR_ID[name], b, c])`` and
rounds them to the nearest bf16 (ties to even).  Chunks are independent, so the
result does not depend on the number of threads that fill them.  Ragged
lengths are integers drawn uniformly from an inclusive range with
``SeedSequence([seed, TENSOR_ID["len"]])``.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os

import numpy as np

CHUNK = 1 << 22
TENSOR_ID = {"k": 0, "v": 1, "kidx": 2, "q": 3, "qidx": 4, "len": 5}
BASE_SEED = 20261202


def _round_bf16(x: np.ndarray) -> np.ndarray:
    u = x.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def _fill_chunk(out: np.ndarray, seed: int, tid: int, b: int, c: int, scale: float):
    lo = c * CHUNK
    hi = min(out.shape[0], lo + CHUNK)
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, b, c])))
    x = g.standard_normal(hi - lo, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    out[lo:hi] = _round_bf16(x)


def _pool():
    return _cf.ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1)))


def normal_bf16(seed: int, name: str, shape, scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns [shape[0]][...] of N(0, scale^2); one stream per leading index."""
    shape = tuple(int(s) for s in shape)
    per = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    out = np.empty((shape[0], per), dtype=np.uint16)
    tid = TENSOR_ID[name]
    jobs = []
    with _pool() as ex:
        for b in range(shape[0]):
            row = out[b]
            for c in range((per + CHUNK - 1) // CHUNK):
                jobs.append(ex.submit(_fill_chunk, row, seed, tid, b, c, scale))
        for j in jobs:
            j.result()
    return out.reshape(shape)


def normal_bf16_span(seed: int, name: str, b: int, lo: int, hi: int) -> np.ndarray:
    """Values [lo, hi) of leading index b's stream of `name`: the same bits that
    normal_bf16 puts there, drawn from the chunks that cover the span only."""
    tid = TENSOR_ID[name]
    c0, c1 = lo // CHUNK, (hi + CHUNK - 1) // CHUNK
    buf = np.empty(((c1 - c0) * CHUNK,), dtype=np.uint16)
    for c in range(c0, c1):
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, b, c])))
        buf[(c - c0) * CHUNK:(c - c0 + 1) * CHUNK] = _round_bf16(g.standard_normal(CHUNK, dtype=np.float32))
    return buf[lo - c0 * CHUNK:hi - c0 * CHUNK].copy()


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """B integers uniform in the inclusive range [lo, hi]."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, TENSOR_ID["len"]])))
    return g.integers(lo, hi + 1, size=B).astype(np.int32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (used only for display / tolerances)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
