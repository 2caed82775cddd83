#!/usr/bin/env python
"""Throughput of the CSA + HCA hybrid-attention decode step on B200.

One step = one hybrid_attn_decode call (indexer scores + exact top-k + CSA
attention over the chosen entries + HCA attention over all entries) for every
sequence of the batch, caches already compressed and resident in HBM.  The
default workload is decode at 1M tokens of context: B=4, 64 query heads, one
shared KV head, head_dim 128, CSA m=4 top-k 2048, HCA m=128, bf16 N(0,1)
inputs from a fixed seed.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the same workload

Under torchrun every rank runs its own batch of independent sequences (weak
scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import signal
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_pool_b200 import configs, synth  # noqa: E402

DEFAULT_WORKLOAD = "decode_b4_t1m_h64_k2048"
METRIC = "hybrid-attn decode tokens/s @1M ctx; achieved HBM GB/s (% of peak), 1 B200"
SCALE = float(np.float32(1.0 / math.sqrt(128.0)))
L2_FLUSH_BYTES = 512 << 20  # > 126 MB L2: written, then read, between timed steps


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak for kernels timed inside a long step (TFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if d.get("bf16_tflops_sustained"):
            return float(d["bf16_tflops_sustained"]), "measured (sustained)"
    return 1400.0, "fallback (sustained)"


def kernel_source_hash(kernel):
    """Hash of the named kernel's own source (its __global__ function) and of the
    shared device helpers: recorded ncu counters stay valid until these change."""
    d = os.path.join(ROOT, "sparse_attention_pool_b200", "csrc")
    h = hashlib.sha256()
    with open(os.path.join(d, "sa_common.cuh"), "rb") as fh:
        h.update(fh.read())
    body = None
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f)) as fh:
            src = fh.read()
        at = src.find(kernel + "(")
        while at >= 0 and "__global__" not in src[src.rfind("\n\n", 0, at):at]:
            at = src.find(kernel + "(", at + 1)
        if at < 0:
            continue
        start = src.rfind("\n\n", 0, at)
        depth, i = 0, src.index("{", at)
        while True:
            depth += {"{": 1, "}": -1}.get(src[i], 0)
            i += 1
            if depth == 0:
                break
        body = src[start:i]
        break
    if body is None:
        return None
    h.update(body.encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged since."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    r = rec.get(f"{kernel}@{workload}")
    if not r or r.get("source_hash") != kernel_source_hash(kernel):
        return None
    return r.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self._summary = None
        self.path = f"/tmp/sa_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            # -f writes every sample straight to the file (stdout to a file would be block-buffered)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def lines(self):
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except OSError:
            return 0

    def keep_busy(self, work, min_samples, max_s=10.0):
        """Run untimed work until the sampler has written `min_samples` more lines."""
        if not self.proc:
            return
        import torch
        start, t0 = self.lines(), time.time()
        while self.lines() < start + min_samples and time.time() - t0 < max_s:
            for _ in range(20):
                work()
            torch.cuda.synchronize()

    def __exit__(self, *exc):
        if self.proc:
            self.proc.send_signal(signal.SIGINT)
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()

    def summary(self):
        """The samples' median SM clock and the throttle reasons seen (read once)."""
        if self._summary is not None:
            return self._summary
        if not self.proc or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        self._summary = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                         "reasons": sorted(reasons), "samples": len(sm)}
        return self._summary


def decode_bytes(w, lengths, indexer="bf16", kv="workload"):
    """Algorithmic HBM bytes of one decode step and of its indexer score kernel
    (an indexer key is 128 bytes in bf16, 32 + 2 in MXFP4; a K + V entry is
    512 bytes in bf16, 256 in e4m3 and 192 + 128 in mixed storage, the last
    two with a scale each per gathered entry and per 64 HCA entries)."""
    fp8 = w.fp8 or kv == "mixed"
    kvb = 320 if kv == "mixed" else 2 * 128 * (1 if w.fp8 else 2)
    ib = 128 if indexer == "bf16" else 34
    step = 0
    score = 0
    for L in lengths:
        nc, nh = int(L) // w.m_csa, int(L) // w.m_hca
        sel = min(w.topk, nc)
        step += nc * ib + sel * kvb + nh * kvb + w.H * 256 + 128 + 2 * w.H * 256
        if fp8:
            step += sel * 8 + ((nh + 63) // 64) * 8
        score += nc * ib  # the indexer keys, read once (no score reaches HBM by definition)
    return step, score


def compress_bytes(w, lengths, kv="workload"):
    """Algorithmic HBM bytes of compressing the raw tokens once: (CSA, HCA),
    each the complete blocks' raw K, V (+ indexer keys for CSA) read once and
    the entries (+ fp8 scales per 64 entries) written once."""
    fp8 = w.fp8 or kv == "mixed"
    kv_entry = 320 if kv == "mixed" else 2 * 128 * (1 if w.fp8 else 2)
    csa = hca = 0
    for L in lengths:
        nc, nh = int(L) // w.m_csa, int(L) // w.m_hca
        csa += nc * w.m_csa * (128 + 128 + 64) * 2 + nc * (kv_entry + 128)
        hca += nh * w.m_hca * (128 + 128) * 2 + nh * kv_entry
        if fp8:
            csa += ((nc + 63) // 64) * 8
            hca += ((nh + 63) // 64) * 8
    return csa, hca


def time_compress(S, w, lengths, Kd, Vd, KId, lens, csa, hca, kv, reps=5):
    """CUDA-event time of csa_compress and hca_compress over the bench's raw
    tokens (inputs far larger than L2), after two warm-up calls each."""
    import torch
    stream = torch.cuda.current_stream()
    out = {}
    for name, fn in (("csa", lambda: S.csa_compress(Kd, Vd, KId, lens, csa)),
                     ("hca", lambda: S.hca_compress(Kd, Vd, lens, hca))):
        fn()
        fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        e1.synchronize()
        out[name + "_ms"] = e0.elapsed_time(e1) / reps
    S.read_device_status()
    cb, hb = compress_bytes(w, lengths, kv)
    peak, kind = measured_peaks()
    out["csa_bytes"], out["hca_bytes"] = cb, hb
    out["csa_gbs"] = cb / (out["csa_ms"] / 1e3) / 1e9
    out["hca_gbs"] = hb / (out["hca_ms"] / 1e3) / 1e9
    out["csa_frac"], out["hca_frac"] = out["csa_gbs"] / peak, out["hca_gbs"] / peak
    out["peak_gbs"], out["peak_kind"] = peak, kind
    return out


def traced_run(path, fn, capacity=1 << 22):
    """One untimed run of `fn` with the profiling build's per-CTA marks
    recorded (the library loaded with SA_TRACE_LIB=1); the timeline report is
    written to `path`."""
    import torch

    from sparse_attention_pool_b200 import trace

    torch.cuda.synchronize()
    buf = trace.install(capacity)
    fn()
    rec = trace.records(buf)
    n = trace.count()
    trace.uninstall()
    with open(path, "w") as f:
        f.write(trace.report(rec) + "\n")
    return {"path": path, "records": int(rec.size), "dropped": max(0, n - int(rec.size)),
            "library": "profiling build (marks compiled in): this line's timings are not headline figures"}


def max_over_ranks(ms, world, device):
    """The job's time is the slowest rank's: every rank calls this at the same point."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, max_ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def make_inputs(w, rank):
    seed = synth.BASE_SEED + w.index + 7919 * rank
    B, L = w.B, w.L
    if w.L_min is not None:
        lengths = synth.ragged_lengths(seed, B, w.L_min, w.L)
    else:
        lengths = np.full((B,), L, dtype=np.int32)
    K = synth.normal_bf16(seed, "k", (B, L, 128))
    V = synth.normal_bf16(seed, "v", (B, L, 128))
    KI = synth.normal_bf16(seed, "kidx", (B, L, 64))
    q = synth.normal_bf16(seed, "q", (B, w.H, 128))
    qI = synth.normal_bf16(seed, "qidx", (B, 64))
    return lengths, K, V, KI, q, qI


def to_bf16_tensor(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


# ---------------------------------------------------------------- our arm ---

def run_ours(args, w, rank, world, dev):
    import torch
    import torch.distributed as dist

    import sparse_attention_pool_b200 as S
    from sparse_attention_pool_b200 import _lib

    lengths, K, V, KI, q_h, qI_h = make_inputs(w, rank)
    t_gen = time.time()
    Kd, Vd, KId = to_bf16_tensor(K, dev), to_bf16_tensor(V, dev), to_bf16_tensor(KI, dev)
    lens = torch.from_numpy(lengths).to(dev)
    mixed = args.kv == "mixed"
    csa = S.alloc_cache(w.B, w.L // w.m_csa, w.m_csa, fp8=w.fp8, mixed=mixed, with_kidx=True, device=dev)
    hca = S.alloc_cache(w.B, w.L // w.m_hca, w.m_hca, fp8=w.fp8, mixed=mixed, device=dev)
    S.csa_compress(Kd, Vd, KId, lens, csa)
    S.hca_compress(Kd, Vd, lens, hca)
    fp4 = args.indexer == "mxfp4"
    codes4, scales4 = S.csa_index_quantize_mxfp4(csa) if fp4 else (None, None)  # like compression: untimed
    torch.cuda.synchronize()
    try:  # compression on its own (recompressing gives the same caches)
        compress_info = time_compress(S, w, lengths, Kd, Vd, KId, lens, csa, hca, args.kv)
    except Exception as ex:  # noqa: BLE001 -- recorded in the JSON line
        compress_info = {"error": str(ex)[:160]}
    del Kd, Vd, KId
    torch.cuda.empty_cache()
    q = to_bf16_tensor(q_h, dev)
    qI = to_bf16_tensor(qI_h, dev)
    B, H, k = w.B, w.H, w.topk
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k), device=dev)
    out_c = torch.empty(B, H, 128, dtype=torch.bfloat16, device=dev)
    out_h = torch.empty_like(out_c)
    lse_c = torch.empty(B, H, dtype=torch.float32, device=dev)
    lse_h = torch.empty_like(lse_c)
    idx = torch.empty(B, k, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty(1, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # Writing a buffer larger than L2 evicts the step's data; reading it back
        # then leaves L2 holding clean lines, so the timed step pays no write-back
        # of the flush itself.
        flush.fill_(1)
        flush_sink.copy_(flush.view(torch.int64).sum())
    L = _lib.lib()
    S.set_option(S.SA_OPT_DECODE_FAST, args.decode_fast)

    def decode(qq, qqI):
        if fp4:
            S.hybrid_attn_decode_mxfp4(qq, qqI, csa, hca, codes4, scales4, k, ws, scale=SCALE, out_csa=out_c,
                                       out_hca=out_h, lse_csa=lse_c, lse_hca=lse_h, idx_out=idx, cnt_out=cnt)
        else:
            S.hybrid_attn_decode(qq, qqI, csa, hca, k, ws, scale=SCALE, out_csa=out_c, out_hca=out_h,
                                 lse_csa=lse_c, lse_hca=lse_h, idx_out=idx, cnt_out=cnt)

    def step():
        decode(q, qI)

    # events around every stage of the step (captured into the graph as record nodes)
    stage_names = ["index_score", "topk_select", "csa_attn", "hca_attn"]
    stage_ev = []
    for si in range(len(stage_names)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)  # creates the events; the library re-records them around the stage
        e1.record(stream)
        L.sa_set_stage_events(si, e0.cuda_event, e1.cuda_event)
        stage_ev.append((e0, e1))
    step()  # eager first call: one-time kernel attributes
    torch.cuda.synchronize()
    S.read_device_status()
    n0 = L.sa_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = int(L.sa_launch_count() - n0)

    # two graphs of the same step: one with the stage events as record nodes
    # (for the per-stage breakdown and the roofline kernel's time), and one
    # without them, which the headline number times
    graph_staged = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_staged):
        step()
    torch.cuda.synchronize()
    # the roofline kernel alone between two events (the score kernel's stage)
    for si in range(1, len(stage_names)):
        L.sa_set_stage_events(si, None, None)
    graph_score = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_score):
        step()
    torch.cuda.synchronize()
    L.sa_set_stage_events(0, None, None)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush_l2()
        graph.replay()
        flush_l2()
        graph_staged.replay()
        flush_l2()
        graph_score.replay()
    torch.cuda.synchronize()

    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    step_ms = []
    stage_ms = [[] for _ in stage_names]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.keep_busy(lambda: (flush_l2(), graph.replay()), min_samples=3)  # clocks under load first
        for i in range(args.steps):
            flush_l2()  # untimed: evict the caches from L2
            ev0[i].record(stream)
            graph.replay()
            ev1[i].record(stream)
            ev1[i].synchronize()
            step_ms.append(ev0[i].elapsed_time(ev1[i]))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        total_ms = max_over_ranks(sum(step_ms), world, dev)
        # the same steps again with the stage events inside (not the headline)
        staged_ms = []
        for i in range(args.steps):
            flush_l2()
            ev0[i].record(stream)
            graph_staged.replay()
            ev1[i].record(stream)
            ev1[i].synchronize()
            staged_ms.append(ev0[i].elapsed_time(ev1[i]))
            for si, (e0, e1) in enumerate(stage_ev):
                stage_ms[si].append(e0.elapsed_time(e1))
        score_ms = []
        for i in range(args.steps):
            flush_l2()
            graph_score.replay()
            stage_ev[0][1].synchronize()
            score_ms.append(stage_ev[0][0].elapsed_time(stage_ev[0][1]))
        # the same kernel between the same two events in eager calls: queued
        # behind the flush (far longer than the host's submission), so the
        # events bracket the kernel alone, without a graph's event nodes
        L.sa_set_stage_events(0, stage_ev[0][0].cuda_event, stage_ev[0][1].cuda_event)
        score_eager_ms = []
        for i in range(args.steps):
            flush_l2()
            step()
            stage_ev[0][1].synchronize()
            score_eager_ms.append(stage_ev[0][0].elapsed_time(stage_ev[0][1]))
        L.sa_set_stage_events(0, None, None)
        clk.keep_busy(lambda: (flush_l2(), graph.replay()), min_samples=2)
    torch.cuda.synchronize()
    S.read_device_status()
    trace_info = traced_run(args.trace, lambda: (flush_l2(), graph.replay())) if args.trace else None

    # end to end through the public API: pinned host q / q_idx in, outputs back out
    q_pin = torch.from_numpy(np.ascontiguousarray(q_h).view(np.int16)).pin_memory()
    qi_pin = torch.from_numpy(np.ascontiguousarray(qI_h).view(np.int16)).pin_memory()
    oc_pin = torch.empty(B, H, 128, dtype=torch.int16).pin_memory()
    oh_pin = torch.empty_like(oc_pin).pin_memory()
    lc_pin = torch.empty(B, H, dtype=torch.float32).pin_memory()
    lh_pin = torch.empty_like(lc_pin).pin_memory()
    q_dev = torch.empty(B, H, 128, dtype=torch.int16, device=dev)
    qi_dev = torch.empty(B, 64, dtype=torch.int16, device=dev)
    h2d = q_pin.numel() * 2 + qi_pin.numel() * 2
    d2h = oc_pin.numel() * 2 * 2 + lc_pin.numel() * 4 * 2
    # the public API a serving loop uses: the step captured once by the library
    # together with its packed host copies (DecodeGraph: one H2D copy of the
    # queries, the outputs and lse copied back inside the graph, one launch per
    # step); checked bit for bit against the eager call first, else the eager
    # call with separate copies is timed instead
    api_name = "hybrid_attn_decode_mxfp4" if fp4 else "hybrid_attn_decode"
    e2e_api = f"{api_name} (eager) + pinned-host copies"
    cap = None
    try:
        cap = S.DecodeGraph(csa, hca, k, H, scale=SCALE, codes=codes4, scales=scales4, flags=args.e2e_io)
        cap.q.view(torch.int16).copy_(q_pin)
        cap.q_idx.view(torch.int16).copy_(qi_pin)
        cap.step()
        decode(q, qI)
        torch.cuda.synchronize()
        if not (torch.equal(cap.out_csa.view(torch.int16), out_c.view(torch.int16).cpu())
                and torch.equal(cap.out_hca.view(torch.int16), out_h.view(torch.int16).cpu())
                and torch.equal(cap.idx, idx) and torch.equal(cap.lse_csa, lse_c.cpu())
                and torch.equal(cap.lse_hca, lse_h.cpu())):
            raise RuntimeError("the captured step differs from the eager call")
        h2d, d2h = cap.h2d_bytes, cap.d2h_bytes
        io_in = "a kernel reading the mapped pinned queries" if cap.flags & 1 else "one packed H2D copy"
        io_out = ("the kernels writing outputs + lse into mapped pinned memory" if cap.flags & 2
                  else "the outputs + lse copied back by the copy engine")
        e2e_api = (f"sa_decode_graph_step (C ABI: {api_name} captured with {io_in} and {io_out}, "
                   f"all inside the graph; one launch per step; flags {cap.flags})")
    except Exception as ex:  # noqa: BLE001 -- recorded in the JSON line
        cap = None
        e2e_api += f"; captured step not used: {str(ex)[:120]}"
    e2e_ms = []
    if world > 1:
        dist.barrier()
    for i in range(args.steps):
        flush_l2()
        ev0[i].record(stream)
        if cap is not None:
            cap.step(stream)
        else:
            q_dev.copy_(q_pin, non_blocking=True)
            qi_dev.copy_(qi_pin, non_blocking=True)
            decode(q_dev.view(torch.bfloat16), qi_dev.view(torch.bfloat16))
            oc_pin.copy_(out_c.view(torch.int16), non_blocking=True)
            oh_pin.copy_(out_h.view(torch.int16), non_blocking=True)
            lc_pin.copy_(lse_c, non_blocking=True)
            lh_pin.copy_(lse_h, non_blocking=True)
        ev1[i].record(stream)
        ev1[i].synchronize()
        e2e_ms.append(ev0[i].elapsed_time(ev1[i]))
    e2e_total = max_over_ranks(sum(e2e_ms), world, dev)
    S.read_device_status()
    del graph, graph_staged, graph_score, cap

    value = job_throughput(B * args.steps, world, total_ms)
    step_bytes, score_bytes = decode_bytes(w, lengths, args.indexer, args.kv)
    peak, peak_kind = measured_peaks()
    score_avg = statistics.mean(score_eager_ms)
    score_avg_graph = statistics.mean(score_ms)
    achieved = score_bytes / (score_avg / 1e3) / 1e9
    step_gbs = step_bytes / (total_ms / args.steps / 1e3) / 1e9
    result = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("mixed-kv(e4m3+bf16-rope)/bf16" if mixed else "bf16" if not w.fp8 else "fp8e4m3-kv/bf16")
        + ("+mxfp4-indexer" if fp4 else ""),
        "data": "synthetic",
        "config": {"workload": w.name, "B_per_gpu": B, "context": int(w.L), "heads": H, "head_dim": 128,
                   "csa_m": w.m_csa, "topk": k, "hca_m": w.m_hca,
                   "kv_dtype": "mixed" if mixed else "e4m3" if w.fp8 else "bf16",
                   "decode_fast": args.decode_fast,
                   "indexer": args.indexer,
                   "parallelism": f"replicas x{world} (independent sequences)",
                   "l2": "flushed between timed steps: 512 MB written then read back (clean L2)", "launch": "CUDA graph replay"},
        "hbm": {"step_bytes": step_bytes, "step_gbs": step_gbs, "step_frac": step_gbs / peak,
                "step_frac_of_8tbs": step_gbs / 8000.0},
        "roofline": {"kernel": "score_decode_mxfp4_kernel" if fp4 else "score_decode_kernel", "bound": "hbm",
                     "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "bytes_per_launch": score_bytes, "avg_launch_ms": score_avg,
                     "timing": "CUDA events on the launching stream around the kernel in eager calls queued "
                               "behind the L2 flush",
                     "avg_launch_ms_graph_events": score_avg_graph,
                     "traffic": None if fp4 else recorded_traffic("score_decode_kernel", w.name)},
        "stages_ms": {n: statistics.mean(v) for n, v in zip(stage_names, stage_ms)},
        "compress": compress_info,
        "staged_step_ms": statistics.mean(staged_ms),
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": job_throughput(B * args.steps, world, e2e_total), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "api": e2e_api},
        "clocks": clk.summary(),
        "setup_s": round(time.time() - t_gen, 1),
    }
    if trace_info:
        result["trace"] = trace_info
    if step_bytes < 8_000_000:  # a step this small is bound by launch latency, not by HBM
        result["roofline"]["note"] = (f"{step_bytes / 1e6:.2f} MB per step: launch-latency bound; "
                                      "the fraction does not measure the kernel")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"], cs = cpu_baseline(w, lengths, K, V, KI, q_h, qI_h, budget_s=args.cpu_budget,
                                                  indexer=args.indexer, kv=args.kv)
        result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(w, lengths, K, V, KI, q_h, qI_h, cs=cs,
                                                                  budget_s=args.cpu_budget / 2, indexer=args.indexer,
                                                                  kv=args.kv)
    return result


# ------------------------------------------------- context-parallel mode ---

def run_cp(args, w, rank, world, dev):
    """--cp: one batch sharded by context over the ranks (each rank holds and
    compresses its shard of every sequence); a step is cp_decode_step, the
    exchange over NCCL.  Strong scaling: the same B tokens per step at every
    world size.  With one rank the selection is checked against
    hybrid_attn_decode on the same caches."""
    import socket

    import torch
    import torch.distributed as dist

    import sparse_attention_pool_b200 as S
    from sparse_attention_pool_b200 import _lib, cp

    own_group = not dist.is_initialized()
    if own_group:  # a one-rank NCCL group for the exchange calls
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = dist.TCPStore("127.0.0.1", port, 1, True)
        dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=300), device_id=dev)
    try:
        lengths, K, V, KI, q_h, qI_h = make_inputs(w, 0)  # one batch, the same on every rank
        B, H, k = w.B, w.H, w.topk
        t_gen = time.time()
        bounds = [cp.shard_bounds(int(lengths[b]), world) for b in range(B)]
        span = [bounds[b][rank] for b in range(B)]
        Lw = max(1, max(t1 - t0 for t0, t1 in span))
        Lw = -(-Lw // 128) * 128
        Ks = np.zeros((B, Lw, 128), np.uint16)
        Vs = np.zeros((B, Lw, 128), np.uint16)
        KIs = np.zeros((B, Lw, 64), np.uint16)
        for b, (t0, t1) in enumerate(span):
            Ks[b, :t1 - t0], Vs[b, :t1 - t0], KIs[b, :t1 - t0] = K[b, t0:t1], V[b, t0:t1], KI[b, t0:t1]
        del K, V, KI
        lens = torch.tensor([t1 - t0 for t0, t1 in span], dtype=torch.int32, device=dev)
        Kd, Vd, KId = to_bf16_tensor(Ks, dev), to_bf16_tensor(Vs, dev), to_bf16_tensor(KIs, dev)
        csa = S.alloc_cache(B, Lw // w.m_csa, w.m_csa, fp8=w.fp8, with_kidx=True, device=dev)
        hca = S.alloc_cache(B, Lw // w.m_hca, w.m_hca, fp8=w.fp8, device=dev)
        S.csa_compress(Kd, Vd, KId, lens, csa)
        S.hca_compress(Kd, Vd, lens, hca)
        torch.cuda.synchronize()
        del Kd, Vd, KId
        base = torch.tensor([cp.entry_base(bounds[b], rank, w.m_csa) for b in range(B)], dtype=torch.int32,
                            device=dev)
        q, qI = to_bf16_tensor(q_h, dev), to_bf16_tensor(qI_h, dev)
        ws = S.alloc_workspace(cp.workspace_size(B, H, csa.Ncap, hca.Ncap, k), device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        flush_sink = torch.empty(1, dtype=torch.int64, device=dev)
        stream = torch.cuda.current_stream()

        def flush_l2():  # written then read back: L2 ends up clean (as in the main line)
            flush.fill_(1)
            flush_sink.copy_(flush.view(torch.int64).sum())

        def step():
            return cp.cp_decode_step(q, qI, csa, hca, base, k, ws, scale=SCALE)

        oc, oh, lc, lh, sel, scnt = step()
        torch.cuda.synchronize()
        S.read_device_status()
        check = None
        if world == 1:
            ws1 = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k),
                                    device=dev)
            idx = torch.empty(B, k, dtype=torch.int32, device=dev)
            cnt = torch.empty(B, dtype=torch.int32, device=dev)
            S.hybrid_attn_decode(q, qI, csa, hca, k, ws1, scale=SCALE, idx_out=idx, cnt_out=cnt)
            torch.cuda.synchronize()
            check = "selection equals hybrid_attn_decode" if torch.equal(idx, sel) and torch.equal(cnt, scnt) \
                else "MISMATCH with hybrid_attn_decode"
        L = _lib.lib()
        n0 = L.sa_launch_count()
        step()
        torch.cuda.synchronize()
        launches_per_step = int(L.sa_launch_count() - n0)
        for _ in range(args.warmup):
            flush_l2()
            step()
        torch.cuda.synchronize()
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        step_ms = []
        dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(torch.cuda.current_device()) as clk:
            for i in range(args.steps):
                flush_l2()  # untimed: evict the shards from L2
                ev0[i].record(stream)
                step()
                ev1[i].record(stream)
                ev1[i].synchronize()
                step_ms.append(ev0[i].elapsed_time(ev1[i]))
        torch.cuda.synchronize()
        dist.barrier()
        total_ms = max_over_ranks(sum(step_ms), world, dev)
        S.read_device_status()
        return {
            "metric": METRIC, "value": B * args.steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16" if not w.fp8 else "fp8e4m3-kv/bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "context": int(w.L), "heads": H, "topk": k,
                       "parallelism": f"context-parallel x{world} (one batch sharded by context)",
                       "l2": "flushed between timed steps: 512 MB written then read back (clean L2)",
                       "launch": "eager, NCCL all-gathers"},
            "gpu_launches": launches_per_step * args.steps, "check": check,
            "e2e": {"value": None, "note": "not measured in --cp mode"},
            "clocks": clk.summary(), "setup_s": round(time.time() - t_gen, 1),
        }
    finally:
        if own_group:
            dist.destroy_process_group()


# ------------------------------------------------------------ prefill arm ---

FP64_FMA_PER_CLK_PER_SM = 64  # B200: 64 fp64 lanes per SM (nominal 37 TFLOP/s at 1965 MHz)


def run_prefill(args, w, rank, world, dev):
    """One step = a whole causal prefill of one T-token sequence (both branches)."""
    import torch

    import sparse_attention_pool_b200 as S
    from sparse_attention_pool_b200 import _lib

    seed = synth.BASE_SEED + w.index + 7919 * rank
    t_gen = time.time()
    B, T, H, k = w.B, w.L, w.H, w.topk
    K = synth.normal_bf16(seed, "k", (B, T, 128))
    V = synth.normal_bf16(seed, "v", (B, T, 128))
    KI = synth.normal_bf16(seed, "kidx", (B, T, 64))
    Kd, Vd, KId = to_bf16_tensor(K, dev), to_bf16_tensor(V, dev), to_bf16_tensor(KI, dev)
    del K, V, KI
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    csa = S.alloc_cache(B, T // w.m_csa, w.m_csa, with_kidx=True, device=dev)
    hca = S.alloc_cache(B, T // w.m_hca, w.m_hca, device=dev)
    S.csa_compress(Kd, Vd, KId, lens, csa)
    S.hca_compress(Kd, Vd, lens, hca)
    torch.cuda.synchronize()
    del Kd, Vd, KId
    q = to_bf16_tensor(synth.normal_bf16(seed, "q", (B, T, H, 128)), dev)
    qI = to_bf16_tensor(synth.normal_bf16(seed, "qidx", (B, T, 64)), dev)
    ws = S.alloc_workspace(S.workspace_size(S.SA_OP_HYBRID_PREFILL, B, T, H, csa.Ncap, hca.Ncap, k), device=dev)
    idx = torch.empty(B, T, k, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, T, dtype=torch.int32, device=dev)
    out_c = torch.empty_like(q)
    out_h = torch.empty_like(q)
    pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    L = _lib.lib()
    stream = torch.cuda.current_stream()
    S.set_option(S.SA_OPT_PREFILL_SELECT, args.prefill_select)
    S.set_option(S.SA_OPT_HCA_PREFILL, args.hca_prefill)

    def step():
        S.hybrid_attn_prefill(q, qI, csa, hca, k, ws, idx, cnt, scale=SCALE, out_csa=out_c, out_hca=out_h)

    step()
    torch.cuda.synchronize()
    S.read_device_status()
    n0 = L.sa_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = int(L.sa_launch_count() - n0)
    for _ in range(args.warmup - 2):
        step()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.keep_busy(step, min_samples=3)
        step_ms = []
        for i in range(args.steps):
            ev0[i].record(stream)
            step()
            ev1[i].record(stream)
            ev1[i].synchronize()
            step_ms.append(ev0[i].elapsed_time(ev1[i]))
        # the stages through their own entry points (not the headline)
        stages = {}

        def timed(name, fn):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fn()
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            stages[name] = e0.elapsed_time(e1)
        timed("index_topk", lambda: S.csa_index_topk(qI, csa, k, ws, q_pos=pos, idx=idx, cnt=cnt))
        timed("csa_attn", lambda: S.csa_sparse_attn(q, csa, idx, cnt, k, ws, scale=SCALE, out=out_c))
        timed("hca_attn", lambda: S.hca_dense_attn(q, hca, ws, q_pos=pos, scale=SCALE, out=out_h))
        clk.keep_busy(step, min_samples=2)
    torch.cuda.synchronize()
    S.read_device_status()
    trace_info = traced_run(args.trace, step) if args.trace else None
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = job_throughput(B * T * args.steps, world, total_ms)
    # fp64 indexer: one exact 64-term fp64 dot product per visible (query, entry) pair
    pairs = sum(min(t // w.m_csa, T // w.m_csa) for t in range(T)) * B
    fma = pairs * 64
    sm_mhz = clk.summary().get("sm_mhz") or 1965.0
    fp64_peak = 148 * FP64_FMA_PER_CLK_PER_SM * 2 * sm_mhz * 1e6 / 1e12
    idx_tflops = 2 * fma / (stages["index_topk"] / 1e3) / 1e12
    # attention flops: QK^T and PV over the visible / selected entries, every head
    csa_rows = sum(min(k, t // w.m_csa) for t in range(T)) * B
    hca_rows = sum(t // w.m_hca for t in range(T)) * B
    csa_tf = 4 * csa_rows * H * 128 / (stages["csa_attn"] / 1e3) / 1e12
    hca_tf = 4 * hca_rows * H * 128 / (stages["hca_attn"] / 1e3) / 1e12
    result = {
        "metric": "hybrid-attn causal prefill tokens/s @128K",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B_per_gpu": B, "tokens": T, "heads": H, "head_dim": 128, "topk": k,
                   "l2": "inputs larger than L2 (q alone is %.1f GB)" % (q.numel() * 2 / 1e9),
                   "launch": "eager (one call per step)", "prefill_select": args.prefill_select,
                   "hca_prefill": args.hca_prefill},
        "stages_ms": stages,
        "roofline": {"kernel": "csa_index_topk prefill stage: score_prefill_kernel + the selection kernel",
                     "bound": "alu", "achieved": idx_tflops, "peak": fp64_peak, "unit": "TFLOP/s (fp64)",
                     "frac": idx_tflops / fp64_peak, "traffic": None,
                     "peak_kind": "derived: 148 SMs x 64 fp64 FMA/clk x 2 x sampled SM clock",
                     "note": "the scoring's fp64 FMAs over the whole stage's time, selection included: "
                             "a lower bound on the scoring kernel's own rate"},
        "attn_tflops": {"csa": csa_tf, "hca": hca_tf},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "setup_s": round(time.time() - t_gen, 1),
    }
    if trace_info:
        result["trace"] = trace_info
    return result


# ----------------------------------------------------------- oracle (CPU) ---

def oracle_query(w, cs, q, qI, t, indexer="bf16", kv="workload"):
    """One decode query on the fp64 oracle: bf16 indexer scores, or FP4 ones
    (the MXFP4 keys are built once per sequence, outside any timing); the
    workload's KV storage, or mixed storage (built once the same way)."""
    from oracle import oracle as O
    if kv == "mixed":
        if indexer != "bf16" and not hasattr(cs, "mx"):
            cs.mx = O.mxfp4_quantize(cs.cidx)
        if not hasattr(cs, "mixed"):
            cs.mixed = {}
            for name, (kb, vb) in (("c", (cs.ck_bf16, cs.cv_bf16)), ("h", (cs.hk_bf16, cs.hv_bf16))):
                codes, ks, rope = O.mixed_quantize(kb, 64)
                vc, vs = O.fp8_quantize(vb)
                cs.mixed[name] = ({"mode": "mixed", "data": codes, "scales": ks, "rope": rope},
                                  {"mode": "fp8", "data": vc, "scales": vs})
        n_vis = min(int(t) // cs.m_csa, cs.n_csa)
        if indexer == "bf16":
            s = O.index_scores(qI, cs.cidx[:n_vis])
        else:
            qc, qs = O.mxfp4_quantize(np.asarray(qI, np.uint16).reshape(1, -1))
            s = O.mxfp4_index_scores(qc[0], qs[0], cs.mx[0][:n_vis], cs.mx[1][:n_vis])
        idx, cnt = O.topk(s, w.topk)
        oc = O.attention_kv(q, *cs.mixed["c"], idx[:cnt], SCALE)
        n_h = min(int(t) // cs.m_hca, cs.n_hca)
        oh = O.attention_kv(q, *cs.mixed["h"], np.arange(n_h, dtype=np.int32), SCALE)
        return {"idx": idx, "cnt": cnt, "out_csa": oc[0], "out_hca": oh[0]}
    if indexer == "bf16":
        return O.hybrid_query(cs, q, qI, t=t, k=w.topk, scale=SCALE)
    if not hasattr(cs, "mx"):
        cs.mx = O.mxfp4_quantize(cs.cidx)
    return O.hybrid_query_mxfp4(cs, q, qI, t=t, k=w.topk, scale=SCALE, idx_codes=cs.mx[0], idx_scales=cs.mx[1])


def oracle_decode_one(w, lengths, K, V, KI, q_h, qI_h, b, indexer="bf16", kv="workload"):
    """One decode token of sequence b on the fp64 oracle; returns (seconds, setup seconds)."""
    from oracle import oracle as O
    t0 = time.time()
    Lb = int(lengths[b])
    cs = O.CompressedSeq(K[b, :Lb], V[b, :Lb], KI[b, :Lb], m_csa=w.m_csa, m_hca=w.m_hca, fp8=w.fp8)
    if indexer != "bf16":
        cs.mx = O.mxfp4_quantize(cs.cidx)
    if kv == "mixed":  # the mixed copies are built here, untimed
        oracle_query(w, cs, q_h[b], qI_h[b], 0, indexer, kv)
    setup = time.time() - t0
    t1 = time.perf_counter()
    oracle_query(w, cs, q_h[b], qI_h[b], Lb, indexer, kv)
    return time.perf_counter() - t1, setup, cs


def cpu_baseline(w, lengths, K, V, KI, q_h, qI_h, budget_s=20.0, indexer="bf16", kv="workload"):
    el, setup, cs = oracle_decode_one(w, lengths, K, V, KI, q_h, qI_h, 0, indexer, kv)
    times = [el]
    t_end = time.time() + max(0.0, budget_s - el)
    while time.time() < t_end and len(times) < 8:
        t1 = time.perf_counter()
        oracle_query(w, cs, q_h[0], qI_h[0], int(lengths[0]), indexer, kv)
        times.append(time.perf_counter() - t1)
    return {"value": len(times) / sum(times), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(times)} decode token(s) of sequence 0 ({int(lengths[0])} tokens of context) on the "
                      f"single-threaded fp64 C oracle, caches pre-built by the oracle ({setup:.1f} s, untimed)"}, cs


def cpu_baseline_all_cores(w, lengths, K, V, KI, q_h, qI_h, cs=None, budget_s=10.0, indexer="bf16", kv="workload"):
    """The same oracle on every host core: independent decode tokens of
    sequence 0 in parallel threads (the C oracle releases the GIL and keeps no
    shared state), tokens over wall time."""
    import concurrent.futures as cf

    from oracle import oracle as O
    if cs is None:
        Lb = int(lengths[0])
        cs = O.CompressedSeq(K[0, :Lb], V[0, :Lb], KI[0, :Lb], m_csa=w.m_csa, m_hca=w.m_hca, fp8=w.fp8)
    cores = max(1, len(os.sched_getaffinity(0)))

    if indexer != "bf16" and not hasattr(cs, "mx"):
        cs.mx = O.mxfp4_quantize(cs.cidx)

    if kv == "mixed" and not hasattr(cs, "mixed"):
        oracle_query(w, cs, q_h[0], qI_h[0], 0, indexer, kv)

    def one(_):
        oracle_query(w, cs, q_h[0], qI_h[0], int(lengths[0]), indexer, kv)

    with cf.ThreadPoolExecutor(cores) as ex:
        list(ex.map(one, range(cores)))  # warm-up round
        done, t0 = 0, time.perf_counter()
        while True:
            list(ex.map(one, range(cores)))
            done += cores
            el = time.perf_counter() - t0
            if el >= budget_s or done >= 16 * cores:
                break
    return {"value": done / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} decode tokens of sequence 0 ({int(lengths[0])} tokens of context), {cores} at a "
                      f"time in parallel threads, on the fp64 C oracle"}


def run_reference_prefill(args, w):
    """Each step: one query row of the causal prefill, rows spread over the sequence."""
    from oracle import oracle as O
    seed = synth.BASE_SEED + w.index
    T, H = w.L, w.H
    K = synth.normal_bf16(seed, "k", (1, T, 128))[0]
    V = synth.normal_bf16(seed, "v", (1, T, 128))[0]
    KI = synth.normal_bf16(seed, "kidx", (1, T, 64))[0]
    cs = O.CompressedSeq(K, V, KI, m_csa=w.m_csa, m_hca=w.m_hca)
    n = args.warmup + args.steps
    rows = [int(T * (i + 0.5) / n) for i in range(n)]
    times = []
    for i, t in enumerate(rows):
        q = synth.normal_bf16_span(seed, "q", 0, t * H * 128, (t + 1) * H * 128).reshape(H, 128)
        qI = synth.normal_bf16_span(seed, "qidx", 0, t * 64, (t + 1) * 64)
        t1 = time.perf_counter()
        O.hybrid_query(cs, q, qI, t=t, k=w.topk, scale=SCALE)
        el = time.perf_counter() - t1
        if i >= args.warmup:
            times.append(el)
    value = len(times) / sum(times)
    sample = (f"each step: one query row of the causal prefill (rows spread evenly over 0..{T - 1}) on the "
              f"single-threaded fp64 C oracle; caches built by the oracle, untimed")
    return {"metric": "hybrid-attn causal prefill tokens/s @128K", "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(times) / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": w.name, "B_per_gpu": w.B, "tokens": T, "heads": H,
                                            "topk": w.topk},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, w, rank, world):
    if rank != 0:
        return None
    if w.mode == "prefill":
        res = run_reference_prefill(args, w)
        res["n_gpus"] = world
        return res
    lengths, K, V, KI, q_h, qI_h = make_inputs(w, 0)
    from oracle import oracle as O
    cs = {}
    times = []
    for i in range(args.warmup + args.steps):
        b = i % w.B
        if b not in cs:
            Lb = int(lengths[b])
            cs[b] = O.CompressedSeq(K[b, :Lb], V[b, :Lb], KI[b, :Lb], m_csa=w.m_csa, m_hca=w.m_hca, fp8=w.fp8)
            if args.indexer != "bf16":
                cs[b].mx = O.mxfp4_quantize(cs[b].cidx)
            if args.kv == "mixed":
                oracle_query(w, cs[b], q_h[b], qI_h[b], 0, args.indexer, args.kv)
        t1 = time.perf_counter()
        oracle_query(w, cs[b], q_h[b], qI_h[b], int(lengths[b]), args.indexer, args.kv)
        el = time.perf_counter() - t1
        if i >= args.warmup:
            times.append(el)
    total = sum(times)
    value = len(times) / total
    sample = (f"each step: one decode token of one sequence (sequences 0..{w.B - 1} in turn) on the "
              f"single-threaded fp64 C oracle; caches built by the oracle, untimed")
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B_per_gpu": w.B, "context": int(w.L), "heads": w.H, "topk": w.topk,
                       "indexer": args.indexer, "kv": args.kv},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


EXTRA_DECODE = ["decode_b1_t4k_h8_k64", "decode_b16_t64k_h64_k512", "ragged_fp8_b32_t64k-256k_h64_k1024"]
EXTRA_PREFILL = "prefill_b1_t128k_h64_k2048"


def run_extras(args, dev):
    """The other workloads, each briefly (10 timed steps, 3 warm-up; the
    prefill 3 and 3), on the same GPU after the headline: their own step
    times, throughputs and stage times for the same JSON line."""
    sub = argparse.Namespace(**vars(args))
    sub.steps, sub.warmup, sub.no_cpu_baseline, sub.trace = 10, 3, True, ""
    out = {}
    for name in EXTRA_DECODE:
        try:
            r = run_ours(sub, configs.BY_NAME[name], 0, 1, dev)
            out[name] = {"ms_per_step": r["ms_per_step"], "value": r["value"], "unit": r["unit"],
                         "steps": sub.steps, "warmup": sub.warmup, "dtype": r["dtype"],
                         "hbm_step_frac": r["hbm"]["step_frac"], "step_bytes": r["hbm"]["step_bytes"],
                         "score_frac": r["roofline"]["frac"], "stages_ms": r["stages_ms"],
                         "e2e": r["e2e"]["value"], "sm_mhz": r["clocks"].get("sm_mhz"),
                         "reasons": r["clocks"].get("reasons")}
        except Exception as ex:  # noqa: BLE001 -- recorded in the JSON line
            out[name] = {"error": str(ex)[:200]}
    sub.steps = 3
    try:
        r = run_prefill(sub, configs.BY_NAME[EXTRA_PREFILL], 0, 1, dev)
        peak, kind = measured_tensor_peak()
        pre = {"workload": EXTRA_PREFILL, "value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
               "steps": sub.steps, "warmup": sub.warmup, "stages_ms": r["stages_ms"],
               "attn_tflops": r["attn_tflops"],
               "tensor_frac": {n: v / peak for n, v in r["attn_tflops"].items()},
               "tensor_peak": peak, "tensor_peak_kind": kind,
               "indexer_fp64_frac": r["roofline"]["frac"], "sm_mhz": r["clocks"].get("sm_mhz"),
               "reasons": r["clocks"].get("reasons")}
    except Exception as ex:  # noqa: BLE001 -- recorded in the JSON line
        pre = {"workload": EXTRA_PREFILL, "error": str(ex)[:200]}
    return out, pre


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[x.name for x in configs.WORKLOADS])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload only: skip the brief runs of the other workloads (prefill and the "
                         "other decode configurations) that the JSON line carries under other_workloads / prefill")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--indexer", default="bf16", choices=["bf16", "mxfp4"],
                    help="decode only: the CSA indexer keys in bf16 (the workload) or FP4 (MXFP4)")
    ap.add_argument("--kv", default="workload", choices=["workload", "mixed"],
                    help="decode only: the workload's KV storage, or mixed storage (rotary dims bf16, the rest e4m3)")
    ap.add_argument("--cp", action="store_true",
                    help="decode only: context-parallel mode, one batch sharded by context over the ranks")
    ap.add_argument("--tokens", type=int, default=0,
                    help="prefill only: a shorter sequence than the workload's (small cases for profiling)")
    ap.add_argument("--e2e-io", type=int, default=None, choices=[0, 1, 2, 3],
                    help="decode only: the I/O mode of the e2e leg's captured step (sa_decode_graph_create flags: "
                         "1 a kernel copies the queries in, 2 the kernels write the outputs to host memory; "
                         "default: DecodeGraph.DEFAULT_FLAGS)")
    ap.add_argument("--decode-fast", type=int, default=0, choices=[0, 1],
                    help="decode only: the indexer + top-k kernels (SA_OPT_DECODE_FAST: 0 the general ones, "
                         "1 the sampled-bound fast path; same indices and outputs)")
    ap.add_argument("--hca-prefill", type=int, default=0, choices=[0, 1, 2],
                    help="prefill only: the HCA attention kernel (SA_OPT_HCA_PREFILL: 0 transposed tiles, two "
                         "query positions per tile with 64 heads; 1 the two-query kernel; 2 transposed tiles, one "
                         "query at a time)")
    ap.add_argument("--prefill-select", type=int, default=4, choices=[1, 2, 3, 4],
                    help="prefill only: the top-k selection kernel (SA_OPT_PREFILL_SELECT; same indices)")
    ap.add_argument("--trace", default="",
                    help="profiling: load the profiling build of the library and write the per-CTA timeline of "
                         "one extra untimed step to this file (one GPU, our arm; the timings of such a run "
                         "are not headline figures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = configs.BY_NAME[args.workload]
    if (args.indexer != "bf16" or args.kv != "workload" or args.cp) and w.mode != "decode":
        ap.error("--indexer, --kv and --cp apply to decode workloads")
    if args.cp and (args.indexer != "bf16" or args.kv != "workload" or args.impl != "ours"):
        ap.error("--cp runs the workload's own storage and indexer on our arm")
    if args.prefill_select != 4 and (w.mode != "prefill" or args.impl != "ours"):
        ap.error("--prefill-select applies to prefill workloads on our arm")
    if args.hca_prefill != 0 and (w.mode != "prefill" or args.impl != "ours"):
        ap.error("--hca-prefill applies to prefill workloads on our arm")
    if args.tokens:
        if w.mode != "prefill":
            ap.error("--tokens applies to prefill workloads")
        w = dataclasses.replace(w, L=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.trace:
        if args.impl != "ours" or args.cp or world > 1:
            ap.error("--trace runs our arm on one GPU, without --cp")
        os.environ["SA_TRACE_LIB"] = "1"  # before the first library call
    if args.impl == "reference":
        res = run_reference(args, w, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    try:
        if args.cp:
            res = run_cp(args, w, rank, world, dev)
        else:
            res = run_ours(args, w, rank, world, dev) if w.mode == "decode" else run_prefill(args, w, rank, world, dev)
            if (world == 1 and not args.no_extras and args.workload == DEFAULT_WORKLOAD and not args.trace
                    and args.indexer == "bf16" and args.kv == "workload"):
                res["other_workloads"], res["prefill"] = run_extras(args, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
