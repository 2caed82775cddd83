"""The profiling build's timeline decoding (sparse_attention_pool_b200.trace)
on synthetic records: per (kernel, phase) counts and first / median / last
times from the earliest mark, in time order, with the phase names."""
from __future__ import annotations

import numpy as np

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
