"""The profiling build's device timeline: a traced decode step records, for
every decode-path kernel, its phases in order (the general kernels: one
filter record per filter CTA; the fast path: one bound and one selection
record set per sequence); a traced prefill top-k records every query's selection CTA and
its phases, and gives the untraced indices.  Runs in child processes (the
library variant is chosen per process by SA_TRACE_LIB).
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

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

def traced_step():
    S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)   # warm-up, untraced
    torch.cuda.synchronize()
    buf = trace.install(1 << 15)
    S.hybrid_attn_decode(g["q"], g["qI"], csa, hca, k, ws, scale=SCALE)
    rec = trace.records(buf)
    trace.uninstall()
    S.read_device_status()
    print(trace.format_summary(rec))
    return rec, {trace.KERNELS[int(x)] for x in np.unique(rec["kernel"])}

def phases_in_order(rec, kid):
    r = rec[rec["kernel"] == kid]
    for cta in np.unique(r["cta"]):
        ts = r[r["cta"] == cta]
        order = np.argsort(ts["phase"], kind="stable")
        assert (np.diff(ts["t"][order].astype(np.int64)) >= 0).all(), (kid, cta)

# the general kernels
S.set_option(S.SA_OPT_DECODE_FAST, 0)
rec, names = traced_step()
assert {"score", "filter", "resolve", "emit", "attn_split"} <= names, names
nfch = -(-csa.Ncap // 2048)
assert int(((rec["kernel"] == 2) & (rec["phase"] == 1)).sum()) == nfch * B
phases_in_order(rec, 3)
# the fast path: the bound (one "bound found" per sequence), the scan, one
# selection CTA per sequence through its last phase, the attention
S.set_option(S.SA_OPT_DECODE_FAST, 1)
rec, names = traced_step()
assert {"bound", "score", "select_fast", "attn_split"} <= names and "filter" not in names, names
assert int(((rec["kernel"] == 12) & (rec["phase"] == 2)).sum()) == B
assert int(((rec["kernel"] == 13) & (rec["phase"] == 5)).sum()) == B
phases_in_order(rec, 13)
print("TRACE_OK")
"""


def test_traced_decode_step_records_every_kernel_phase():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "TRACE_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


CHILD_PREFILL = r"""
import os, sys
sys.path.insert(0, ROOT)
os.environ["SA_TRACE_LIB"] = "1"
import numpy as np, torch
import sparse_attention_pool_b200 as S
from sparse_attention_pool_b200 import _lib, trace
from tests._util import Inputs, compress_on_gpu
assert _lib.lib()._name.endswith("libsparse_attn_trace.so")
B, T, k = 1, 6000, 256
inp = Inputs(982, B, T, 8, Tq=T)
g = inp.to_device()
csa, _ = compress_on_gpu(S, g, B, T)
pos = torch.arange(T, dtype=torch.int32, device="cuda").view(1, T).contiguous()
ws = S.alloc_workspace(S.workspace_size(S.SA_OP_INDEX_TOPK, B, T, 8, csa.Ncap, 0, k))
S.set_option(S.SA_OPT_PREFILL_SELECT, 1)   # the first selection form's phases
i0, c0 = S.csa_index_topk(g["qI"], csa, k, ws, q_pos=pos)   # untraced
i0, c0 = i0.clone(), c0.clone()
torch.cuda.synchronize()
buf = trace.install(1 << 17)
i1, c1 = S.csa_index_topk(g["qI"], csa, k, ws, q_pos=pos)
rec = trace.records(buf)
trace.uninstall()
S.read_device_status()
assert torch.equal(i0, i1) and torch.equal(c0, c1)
sel = rec[rec["kernel"] == 9]
full = T - 4 * (k + 1)   # queries that see more than k entries: t // 4 > k
assert int((sel["phase"] == 0).sum()) == T, int((sel["phase"] == 0).sum())
for ph in range(1, 7):
    assert int((sel["phase"] == ph).sum()) == full, (ph, int((sel["phase"] == ph).sum()))
sc = rec[rec["kernel"] == 8]
assert (sc["phase"] == 0).sum() > 0 and (sc["phase"] == 0).sum() == (sc["phase"] == 2).sum()
rows = trace.cta_phase_durations(rec, "prefill_select")
assert len(rows) == 6 and all(r["runs"] == full for r in rows), rows
for r in rows + trace.cta_phase_durations(rec, "prefill_score"):
    print(r)
# the default (fourth) form: its own phases, the same indices
S.set_option(S.SA_OPT_PREFILL_SELECT, 4)
buf = trace.install(1 << 17)
i4, c4 = S.csa_index_topk(g["qI"], csa, k, ws, q_pos=pos)
rec = trace.records(buf)
trace.uninstall()
S.read_device_status()
assert torch.equal(i0, i4) and torch.equal(c0, c4)
sel = rec[rec["kernel"] == 14]
assert int((sel["phase"] == 0).sum()) == T, int((sel["phase"] == 0).sum())
for ph in range(1, 5):
    assert int((sel["phase"] == ph).sum()) == full, (ph, int((sel["phase"] == ph).sum()))
rows = trace.cta_phase_durations(rec, "prefill_select4")
assert len(rows) == 4 and all(r["runs"] == full for r in rows), rows
print("TRACE_PREFILL_OK")
"""


def test_traced_prefill_topk_records_every_selection_phase():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD_PREFILL.replace("ROOT", repr(ROOT))], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "TRACE_PREFILL_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
