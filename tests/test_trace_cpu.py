"""The profiling build's timeline decoding (sparse_attention_pool_b200.trace)
on synthetic records: per (kernel, phase) counts and first / median / last
times from the earliest mark, in time order, with the phase names."""
from __future__ import annotations

import numpy as np
import pytest

from sparse_attention_pool_b200 import trace


def test_summary_of_synthetic_records():
    recs = [  # (t ns, kernel, phase, sm, cta)
        (1_000, 1, 0, 0, 0), (1_200, 1, 0, 1, 1), (9_000, 1, 1, 0, 0), (9_400, 1, 1, 1, 1), (9_900, 1, 2, 1, 1),
        (10_500, 2, 0, 3, 0), (12_000, 2, 1, 3, 0),
        (13_000, 3, 0, 5, 0), (13_500, 3, 1, 5, 0), (20_000, 3, 6, 5, 0),
    ]
    rec = np.array(recs, dtype=trace.RECORD)
    assert trace.RECORD.itemsize == 16
    rows = trace.summary(rec)
    assert [r["first_us"] for r in rows] == sorted(r["first_us"] for r in rows)
    by = {(r["kernel"], r["phase"]): r for r in rows}
    assert by[("score", "start")]["ctas"] == 2 and by[("score", "start")]["first_us"] == 0.0
    assert by[("score", "scan done")]["last_us"] == 8.4
    assert by[("score", "threshold found")]["ctas"] == 1
    assert by[("filter", "rows done")]["first_us"] == 11.0
    assert by[("resolve", "positions written")]["first_us"] == 19.0
    text = trace.format_summary(rec)
    assert "resolve" in text and "counts scanned" in text
    assert trace.summary(np.zeros(0, dtype=trace.RECORD)) == []


def test_cta_phase_durations_split_runs_at_start_marks():
    # two launches of the prefill selection: CTA 0 runs twice on SM 4 (phases
    # 0..6, then 0 only: a query that sees at most k entries), CTA 1 once on SM 7
    recs = [(100, 9, 0, 4, 0), (300, 9, 1, 4, 0), (800, 9, 2, 4, 0), (900, 9, 3, 4, 0), (1_000, 9, 4, 4, 0),
            (1_000, 9, 5, 4, 0), (3_000, 9, 6, 4, 0),
            (150, 9, 0, 7, 1), (250, 9, 1, 7, 1), (1_250, 9, 2, 7, 1), (1_300, 9, 3, 7, 1), (1_400, 9, 4, 7, 1),
            (1_400, 9, 5, 7, 1), (5_400, 9, 6, 7, 1),
            (9_000, 9, 0, 4, 0),
            (50, 8, 0, 4, 3), (90, 8, 2, 4, 3)]  # another kernel: not counted
    rec = np.array(recs, dtype=trace.RECORD)
    rows = trace.cta_phase_durations(rec, "prefill_select")
    by = {(r["from"], r["to"]): r for r in rows}
    assert [(r["from"], r["to"]) for r in rows] == [
        ("start", "keys staged"), ("keys staged", "digit 1"), ("digit 1", "digit 2"), ("digit 2", "digit 3"),
        ("digit 3", "ties"), ("ties", "end")]
    assert all(r["runs"] == 2 for r in rows)  # the start-only run adds no transition
    assert by[("start", "keys staged")]["median_us"] == pytest.approx(0.15)
    assert by[("keys staged", "digit 1")]["max_us"] == 1.0
    assert by[("ties", "end")]["median_us"] == 3.0 and by[("ties", "end")]["max_us"] == 4.0
    score = trace.cta_phase_durations(rec, "prefill_score")
    assert [(r["from"], r["to"], r["runs"]) for r in score] == [("start", "end", 1)]
    assert trace.cta_phase_durations(np.zeros(0, dtype=trace.RECORD), "prefill_select") == []


def test_report_at_prefill_scale():
    # 40,000 selection runs of 7 marks on 148 SMs (a long prefill's worth):
    # the decoding stays vectorised, and every run shows in every transition
    rng = np.random.default_rng(5)
    runs, ph = 40_000, 7
    cta = np.repeat(np.arange(runs) % 1024, ph).astype(np.uint16)
    sm = np.repeat(rng.integers(0, 148, runs), ph).astype(np.uint16)
    start = np.repeat(np.arange(runs, dtype=np.uint64) * 50_000, ph)
    t = start + np.tile(np.arange(ph, dtype=np.uint64) * 1_000, runs)
    rec = np.zeros(runs * ph, dtype=trace.RECORD)
    rec["t"], rec["kernel"], rec["phase"], rec["sm"], rec["cta"] = t, 9, np.tile(np.arange(ph), runs), sm, cta
    rec = rec[rng.permutation(rec.size)]  # append order is not time order across CTAs
    rows = trace.cta_phase_durations(rec, "prefill_select")
    assert len(rows) == 6 and all(r["runs"] == runs and r["median_us"] == 1.0 and r["max_us"] == 1.0 for r in rows)
    text = trace.report(rec)
    assert "prefill_select: per-CTA phase durations" in text and "digit 3" in text


def test_kernel_busy_is_the_union_of_cta_runs():
    recs = [  # prefill score CTAs 0 and 1 overlap (100..400 and 300..600), a later launch 1000..1100
        (100, 8, 0, 1, 0), (400, 8, 2, 1, 0), (300, 8, 0, 2, 1), (600, 8, 2, 2, 1),
        (1000, 8, 0, 1, 0), (1100, 8, 2, 1, 0),
        # selection: one run 700..900 and a start-only run (no span)
        (700, 9, 0, 3, 0), (900, 9, 6, 3, 0), (950, 9, 0, 3, 1)]
    rec = np.array(recs, dtype=trace.RECORD)
    busy = trace.kernel_busy(rec[np.random.default_rng(0).permutation(rec.size)])
    assert busy["prefill_score"] == pytest.approx(0.6)   # (600 - 100) + (1100 - 1000) ns
    assert busy["prefill_select"] == pytest.approx(0.2)
    assert "time covered by each kernel's CTA runs" in trace.report(rec)
