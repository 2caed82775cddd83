"""The profiling build's device timeline: a traced decode step records, for
every decode-path kernel, its phases in order, with one filter record per
filter CTA.  Runs in a child process (the library variant is chosen per
process by SA_TRACE_LIB).

The module runs only with SA_LOWP_GPU_TESTS=1 until its first B200 run.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(os.environ.get("SA_LOWP_GPU_TESTS") != "1",
                                 reason="the profiling build has not yet run on a B200 (set SA_LOWP_GPU_TESTS=1)")]

CHILD = r"""
import os, sys
sys.path.insert(0, ROOT)
os.environ["SA_TRACE_LIB"] = "1"
import numpy as np, torch
import sparse_attention_pool_b200 as S
from sparse_attention_pool_b200 import _lib, trace
from tests._util import SCALE, Inputs, compress_on_gpu
assert _lib.lib()._name.endswith("libsparse_attn_trace.so")
B, L, H, k = 2, 40000, 64, 512
inp = Inputs(981, B, L, H)
g = inp.to_device()
csa, hca = compress_on_gpu(S, g, B, L)
ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k))
S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)   # warm-up, untraced
torch.cuda.synchronize()
buf = trace.install(1 << 15)
S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
rec = trace.records(buf)
trace.uninstall()
S.read_device_status()
print(trace.format_summary(rec))
names = {trace.KERNELS[int(x)] for x in np.unique(rec["kernel"])}
assert {"score", "filter", "resolve", "emit", "attn_split"} <= names, names
nfch = -(-csa.Ncap // 2048)
assert int(((rec["kernel"] == 2) & (rec["phase"] == 1)).sum()) == nfch * B
res = rec[rec["kernel"] == 3]
for cta in np.unique(res["cta"]):
    ts = res[res["cta"] == cta]
    order = np.argsort(ts["phase"], kind="stable")
    assert (np.diff(ts["t"][order].astype(np.int64)) >= 0).all()
print("TRACE_OK")
"""


def test_traced_decode_step_records_every_kernel_phase():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "TRACE_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
