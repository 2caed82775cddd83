"""The bench's roofline arithmetic: algorithmic bytes of a decode step.

Per sequence: N^C * 128 (indexer keys) + min(k, N^C) * 2 * 128 * b_kv
(gathered K and V) + N^H * 2 * 128 * b_kv (HCA K and V) + H * 256 (q) + 128
(q_I) + 2 * H * 256 (two outputs), with 8 more bytes per gathered entry and
per 64 HCA entries for fp8 scales.  The totals are checked against the
figures worked out by hand for the three uniform decode workloads, and the
fp8 terms against a sum written out term by term.  Also: the argument
checks of the profiling option.
"""
from __future__ import annotations

import os
import subprocess
import sys

import numpy as np
import pytest

import bench
from sparse_attention_pool_b200 import configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_decode_step_bytes_match_the_worked_figures():
    expect = {  # bytes per step (all sequences)
        "decode_b1_t4k_h8_k64": 186_496,
        "decode_b16_t64k_h64_k512": 42_731_520,
        "decode_b4_t1m_h64_k2048": 155_386_368,
    }
    for name, total in expect.items():
        w = configs.BY_NAME[name]
        step, score = bench.decode_bytes(w, np.full((w.B,), w.L))
        assert step == total, name
        nc = w.L // 4
        assert score == w.B * nc * 128, name  # the indexer keys read once; scores never reach HBM


def test_fp8_step_bytes_term_by_term():
    w = configs.BY_NAME["ragged_fp8_b32_t64k-256k_h64_k1024"]
    lengths = np.array([65536, 262144, 100003], dtype=np.int32)
    step, _ = bench.decode_bytes(w, lengths)
    ref = 0
    for L in lengths:
        nc, nh = int(L) // 4, int(L) // 128
        sel = min(w.topk, nc)
        ref += nc * 128                            # indexer keys (bf16)
        ref += sel * 2 * 128 + sel * 8             # gathered e4m3 K, V + their two scales
        ref += nh * 2 * 128 + ((nh + 63) // 64) * 8  # HCA e4m3 K, V + scales per 64 entries
        ref += w.H * 256 + 128 + 2 * w.H * 256     # q, q_I, two outputs
    assert step == ref


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(units_per_rank=40, world=1, max_ms=10.0) == 4000.0
    assert bench.job_throughput(units_per_rank=40, world=8, max_ms=10.0) == 32000.0


def test_mxfp4_indexer_bytes():
    """With MXFP4 indexer keys an entry's key is 32 bytes of e2m1 codes plus 2
    E8M0 scale bytes instead of 128 bytes of bf16; nothing else changes."""
    w = configs.BY_NAME["decode_b4_t1m_h64_k2048"]
    lengths = np.full((w.B,), w.L)
    step16, score16 = bench.decode_bytes(w, lengths)
    step4, score4 = bench.decode_bytes(w, lengths, "mxfp4")
    nc = w.L // 4
    assert score4 == w.B * nc * 34 == 35_651_584
    assert step16 - step4 == w.B * nc * (128 - 34)
    assert step4 == 56_820_224


def test_mixed_kv_bytes_term_by_term():
    """Mixed storage: a K + V entry is 192 + 128 bytes, with a K and a V scale
    (4 bytes each) per gathered entry and per 64 HCA entries."""
    w = configs.BY_NAME["decode_b1_t4k_h8_k64"]
    lengths = np.array([4096])
    step, score = bench.decode_bytes(w, lengths, kv="mixed")
    nc, nh, sel = 1024, 32, 64
    ref = nc * 128 + sel * (192 + 128) + sel * 8 + nh * (192 + 128) + 8 + w.H * 256 + 128 + 2 * w.H * 256
    assert step == ref == 168_584
    assert score == nc * 128  # the indexer is unchanged
    step4, score4 = bench.decode_bytes(w, lengths, "mxfp4", "mixed")
    assert step4 == ref - nc * (128 - 34) and score4 == nc * 34


def test_compress_bytes_match_the_worked_figures():
    """1M-token decode workload: CSA reads 4 x 1M x (512 + 128) B of raw K, V and
    indexer keys and writes 4 x 262,144 x 640 B of entries; HCA reads the raw
    K and V of 4 x 8192 blocks and writes 4 x 8192 x 512 B."""
    w = configs.BY_NAME["decode_b4_t1m_h64_k2048"]
    csa, hca = bench.compress_bytes(w, np.full((w.B,), w.L))
    assert csa == 4 * (1 << 20) * 640 + 4 * 262144 * 640 == 3_355_443_200
    assert hca == 4 * 8192 * 128 * 512 + 4 * 8192 * 512 == 2_164_260_864
    wf = configs.BY_NAME["ragged_fp8_b32_t64k-256k_h64_k1024"]
    c8, h8 = bench.compress_bytes(wf, np.array([65536 + 5]))
    nc, nh = 16385, 512
    assert c8 == nc * 4 * 640 + nc * (256 + 128) + ((nc + 63) // 64) * 8
    assert h8 == nh * 128 * 512 + nh * 256 + ((nh + 63) // 64) * 8


def test_mixed_storage_oracle_leg_is_the_pinned_pieces():
    """The bench's oracle leg for mixed storage selects what the bf16 oracle
    selects and attends with attention_kv over the oracle's mixed storage."""
    from oracle import oracle as O
    w = configs.BY_NAME["decode_b1_t4k_h8_k64"]
    lengths, K, V, KI, q, qI = bench.make_inputs(w, 0)
    L = int(lengths[0])
    cs = O.CompressedSeq(K[0, :L], V[0, :L], KI[0, :L])
    r = bench.oracle_query(w, cs, q[0], qI[0], L, "bf16", "mixed")
    r16 = O.hybrid_query(cs, q[0], qI[0], t=L, k=w.topk, scale=bench.SCALE)
    assert r["cnt"] == r16["cnt"] and np.array_equal(r["idx"], r16["idx"])
    codes, ks, rope = O.mixed_quantize(cs.ck_bf16, 64)
    vc, vs = O.fp8_quantize(cs.cv_bf16)
    oc, _ = O.attention_kv(q[0], {"mode": "mixed", "data": codes, "scales": ks, "rope": rope},
                           {"mode": "fp8", "data": vc, "scales": vs}, r16["idx"][:r16["cnt"]], bench.SCALE)
    assert np.array_equal(r["out_csa"], oc)
    assert np.abs(r["out_csa"] - r16["out_csa"]).max() < 3e-2  # storage rounding only


@pytest.mark.parametrize("extra", [["--cp"], ["--impl", "reference"]])
def test_trace_option_refuses_other_arms(extra):
    """--trace loads the profiling build for one GPU on our arm; it is refused
    (argument error, nothing run) with --cp or the reference arm."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--trace", os.devnull, *extra],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 2 and "--trace runs our arm on one GPU" in r.stderr, r.stderr[-500:]


@pytest.mark.parametrize("extra", [[], ["--workload", "prefill_b1_t128k_h64_k2048", "--impl", "reference"]])
def test_prefill_select_option_applies_to_our_prefill_only(extra):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--prefill-select", "2", *extra],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 2 and "--prefill-select applies to prefill workloads" in r.stderr, r.stderr[-500:]
