"""The seeded input recipe: spans drawn alone equal the same spans of the full tensors."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import numpy as np

from sparse_attention_pool_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_span_equals_the_full_tensor_rows():
    full = synth.normal_bf16(5, "q", (2, 3000, 8, 128))
    for b, t in [(0, 0), (1, 2999), (1, 1500), (0, 511), (0, 512)]:
        row = synth.normal_bf16_span(5, "q", b, t * 1024, (t + 1) * 1024).reshape(8, 128)
        assert np.array_equal(row, full[b, t])


def test_chunks_do_not_depend_on_the_tensor_shape():
    a = synth.normal_bf16(7, "k", (1, synth.CHUNK + 100))
    b = synth.normal_bf16(7, "k", (1, 1000))
    assert np.array_equal(a[0, :1000], b[0])


def test_reference_arm_times_prefill_rows_on_the_oracle():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "prefill_b1_t128k_h64_k2048",
           "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["config"]["workload"] == "prefill_b1_t128k_h64_k2048"
