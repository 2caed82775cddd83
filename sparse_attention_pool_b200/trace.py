"""Device timelines from the profiling build of the library.

``libsparse_attn_trace.so`` is the library compiled with -DSA_TRACE: its
decode-path kernels and the prefill indexer's score and selection kernels
append one record per CTA and phase (global nanosecond timer, kernel, phase,
SM, CTA) to a device buffer.  Set SA_TRACE_LIB=1
before the first library call of the process to load it; the default
library has no marks (its kernels are unchanged) and refuses these calls.

    os.environ["SA_TRACE_LIB"] = "1"
    import sparse_attention_pool_b200 as S
    from sparse_attention_pool_b200 import trace
    buf = trace.install(1 << 16)
    S.hybrid_attn_decode(...)
    print(trace.format_summary(trace.records(buf)))

For a prefill, ``cta_phase_durations(records, "prefill_select")`` gives the
time a selection CTA spends in each phase (median, 90th percentile, max).
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._lib import check, lib

KERNELS = {1: "score", 2: "filter", 3: "resolve", 4: "emit", 5: "attn_split", 6: "attn_merge", 7: "score_fp4",
           8: "prefill_score", 9: "prefill_select", 10: "prefill_score_fp4", 11: "prefill_select2", 12: "bound",
           13: "select_fast", 14: "prefill_select4", 15: "prefill_attn"}
PHASES = {
    "score": ["start", "scan done", "threshold found"],
    "score_fp4": ["start", "scan done", "threshold found"],
    "filter": ["start", "rows done"],
    "resolve": ["start", "counts scanned", "gathered", "t~ known", "band done", "cut done", "positions written"],
    "emit": ["start", "end"],
    "attn_split": ["start", "end"],
    "attn_merge": ["start"],
    # prefill indexer: only the score CTAs whose tile some query sees mark
    "prefill_score": ["start", "staged", "end"],
    "prefill_score_fp4": ["start", "staged", "end"],
    # one CTA per query; a query that sees at most k entries marks only its start
    "prefill_select": ["start", "keys staged", "digit 1", "digit 2", "digit 3", "ties", "end"],
    "prefill_select2": ["start", "keys staged", "digit 1", "digit 2", "digit 3", "counted", "end"],
    # the fast decode path: the sampled bound (CTA 0 of each cluster finds it)
    # and the selection (one CTA per sequence; "band rescored" only when the
    # band is not inside the staged bins)
    "bound": ["start", "sampled", "bound found"],
    "select_fast": ["start", "list loaded", "t~ known", "band rescored", "cut done", "selected"],
    # prefill selection, fourth form: one CTA per query
    "prefill_select4": ["start", "keys staged", "threshold found", "runs counted", "end"],
    # per tile of a query's list (the record's CTA field holds the tile)
    "prefill_attn": ["tile start", "S ready", "softmax done", "copies landed", "MMAs issued", "V copies out"],
}
RECORD = np.dtype([("t", "<u8"), ("kernel", "<u2"), ("phase", "<u2"), ("sm", "<u2"), ("cta", "<u2")])


def install(capacity: int, device="cuda", stream=None) -> torch.Tensor:
    """A zeroed device buffer of `capacity` records, installed as the
    destination of the marks (the count starts at 0)."""
    buf = torch.zeros(capacity * RECORD.itemsize, dtype=torch.uint8, device=device)
    s = torch.cuda.current_stream() if stream is None else stream
    check("sa_trace_install", lib().sa_trace_install(ctypes.c_void_p(buf.data_ptr()), capacity,
                                                     ctypes.c_void_p(s.cuda_stream)))
    return buf


def uninstall(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    check("sa_trace_install", lib().sa_trace_install(None, 0, ctypes.c_void_p(s.cuda_stream)))


def records(buf: torch.Tensor, stream=None) -> np.ndarray:
    """The records written so far (waits for the stream), in append order."""
    s = torch.cuda.current_stream() if stream is None else stream
    n = ctypes.c_uint32(0)
    check("sa_trace_count", lib().sa_trace_count(ctypes.byref(n), ctypes.c_void_p(s.cuda_stream)))
    cap = buf.numel() // RECORD.itemsize
    m = min(int(n.value), cap)
    return buf[:m * RECORD.itemsize].cpu().numpy().view(RECORD)


def summary(rec: np.ndarray) -> list[dict]:
    """Per (kernel, phase): the CTAs that reached it and the first, median
    and last time (µs from the earliest mark), in time order."""
    if rec.size == 0:
        return []
    t0 = int(rec["t"].min())
    rows = []
    for kid in np.unique(rec["kernel"]):
        name = KERNELS.get(int(kid), f"kernel{int(kid)}")
        sel = rec[rec["kernel"] == kid]
        for ph in np.unique(sel["phase"]):
            ts = (sel["t"][sel["phase"] == ph].astype(np.int64) - t0) / 1e3
            labels = PHASES.get(name, [])
            rows.append({"kernel": name, "phase": labels[ph] if ph < len(labels) else str(int(ph)),
                         "ctas": int(ts.size), "first_us": float(ts.min()), "median_us": float(np.median(ts)),
                         "last_us": float(ts.max())})
    return sorted(rows, key=lambda r: r["first_us"])


def _runs(sel: np.ndarray):
    """The records of one kernel sorted by CTA index, SM, time and append
    order, and a run number per record (a new run at every start mark or
    change of CTA / SM)."""
    s = sel[np.lexsort((np.arange(sel.size), sel["t"], sel["sm"], sel["cta"]))]
    new = np.ones(s.size, dtype=bool)
    new[1:] = (s["cta"][1:] != s["cta"][:-1]) | (s["sm"][1:] != s["sm"][:-1]) | (s["phase"][1:] == 0)
    return s, np.cumsum(new) - 1


def cta_phase_durations(rec: np.ndarray, kernel: str) -> list[dict]:
    """Per phase transition of one kernel's CTAs (start -> next mark -> ...):
    how many CTA runs made it and the median / 90th-percentile / maximum time
    between the two marks, in µs.  A CTA run is the records of one (CTA
    index, SM) pair from one start mark to the next in time order, so
    launches of the kernel must not overlap (true of launches without
    programmatic dependent launch on one stream)."""
    kid = next(k for k, v in KERNELS.items() if v == kernel)
    sel = rec[rec["kernel"] == kid]
    if sel.size < 2:
        return []
    s, run = _runs(sel)
    same = run[1:] == run[:-1]
    p0, p1 = s["phase"][:-1][same].astype(np.int64), s["phase"][1:][same].astype(np.int64)
    dt = (s["t"][1:].astype(np.int64) - s["t"][:-1].astype(np.int64))[same] / 1e3
    labels = PHASES.get(kernel, [])
    name = lambda p: labels[p] if p < len(labels) else str(p)  # noqa: E731
    rows = []
    for a, b in sorted({(int(x), int(y)) for x, y in zip(p0, p1)}):
        v = dt[(p0 == a) & (p1 == b)]
        rows.append({"from": name(a), "to": name(b), "runs": int(v.size), "median_us": float(np.median(v)),
                     "p90_us": float(np.percentile(v, 90)), "max_us": float(np.max(v))})
    return rows


def kernel_busy(rec: np.ndarray) -> dict[str, float]:
    """Per kernel: the time (µs) covered by the union of its CTA runs, each
    from its first to its last mark -- over several launches, the time the
    GPU spent in that kernel as far as the marks see it."""
    out = {}
    for kid in sorted({int(x) for x in np.unique(rec["kernel"])}):
        sel = rec[rec["kernel"] == kid]
        s, run = _runs(sel)
        starts = np.minimum.reduceat(s["t"].astype(np.int64), np.flatnonzero(np.r_[True, run[1:] != run[:-1]]))
        ends = np.maximum.reduceat(s["t"].astype(np.int64), np.flatnonzero(np.r_[True, run[1:] != run[:-1]]))
        order = np.argsort(starts, kind="stable")
        starts, ends = starts[order], ends[order]
        reach = np.maximum.accumulate(ends)  # the furthest end among the runs so far
        prev = np.r_[np.iinfo(np.int64).min, reach[:-1]]
        covered = np.clip(ends - np.maximum(starts, prev), 0, None)
        out[KERNELS.get(kid, f"kernel{kid}")] = float(covered.sum()) / 1e3
    return out


def count(stream=None) -> int:
    """Marks made since the buffer was installed, dropped ones included."""
    s = torch.cuda.current_stream() if stream is None else stream
    n = ctypes.c_uint32(0)
    check("sa_trace_count", lib().sa_trace_count(ctypes.byref(n), ctypes.c_void_p(s.cuda_stream)))
    return int(n.value)


def report(rec: np.ndarray) -> str:
    """The per-(kernel, phase) summary, then each kernel's per-CTA phase
    durations."""
    out = [format_summary(rec), "", "time covered by each kernel's CTA runs (µs): " +
           ", ".join(f"{k} {v:.1f}" for k, v in kernel_busy(rec).items())]
    for kid in sorted({int(x) for x in np.unique(rec["kernel"])}):
        name = KERNELS.get(kid)
        rows = cta_phase_durations(rec, name) if name else []
        if rows:
            out.append("")
            out.append(f"{name}: per-CTA phase durations (µs)")
            out.append(f"  {'from':<16} {'to':<16} {'runs':>8} {'median':>9} {'p90':>9} {'max':>9}")
            for r in rows:
                out.append(f"  {r['from']:<16} {r['to']:<16} {r['runs']:>8} {r['median_us']:>9.2f} "
                           f"{r['p90_us']:>9.2f} {r['max_us']:>9.2f}")
    return "\n".join(out)


def format_summary(rec: np.ndarray) -> str:
    lines = [f"{'kernel':<11} {'phase':<18} {'CTAs':>6} {'first':>9} {'median':>9} {'last':>9}  (µs)"]
    for r in summary(rec):
        lines.append(f"{r['kernel']:<11} {r['phase']:<18} {r['ctas']:>6} {r['first_us']:>9.2f} "
                     f"{r['median_us']:>9.2f} {r['last_us']:>9.2f}")
    return "\n".join(lines)
