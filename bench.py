#!/usr/bin/env python3
"""Benchmark of the W8A16 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Headline metric: weight GB/s of the decode linear at M = 1 on the
ChatGLM2-6B h-to-4h shape (X fp16 [1, 4096] . W int8 [4096, 27392]).  One
step is one w8a16_linear call; each step reads a different copy of the
packed weight (6 copies, 673 MB > 126 MB L2), so no step is served from L2.
The timed region replays a CUDA graph of those calls; it is bracketed by a
barrier and a device synchronize and timed with CUDA events on the launching
stream, max over ranks.  The same JSON line also reports, measured in the
same run:
  - prefill: TFLOP/s of the M = 2048 linear on the same weight (two weight
    copies alternate; X 16 MB);
  - quantize / prepack: the one-time weight conversion (fp32 W 449 MB ->
    int8 q + fp16 scales; q -> packed tiles);
  - e2e: the decode metric with the per-step H2D copy of X from pinned host
    memory and the D2H copy of Y inside the timed region;
  - roofline of the dominant kernel, clocks sampled during the timed region,
    and the CPU oracle timed on a bounded sample (rank 0).

N > 1: every rank runs the same independent workload on its own GPU (the
problems are independent; there is no data-path collective), value = units
of all ranks / max-over-ranks time ("weak" scaling).

--impl reference times the CPU oracle (plain C, one thread) on the same
metric and workload, each step a bounded column slab of the weight.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A16 GEMM weight GB/s (M=1, 4096×27392) and TFLOP/s (M=2048) on 1 B200"
K_DIM, N_DIM, M_DECODE, M_PREFILL = 4096, 27392, 1, 2048
N_COPIES = 6                  # 6 x 112 MB rotating weight copies > 4 x L2
DECODE_REPS = 60              # timed repetitions behind each median per call
DECODE_GRAPH_STEPS = 600      # decode calls per captured graph (a multiple of 6)
E2E_GRAPH_STEPS = 48          # end-to-end steps per captured graph
WORKLOAD = ("chatglm2_h_to_4h_decode: X fp16 [1,4096] . W int8 [4096,27392] "
            "(per-channel int8, fp16 scales), W ~ N(0,0.02) with 0.1% N(0,0.2) outliers")
FALLBACK_HBM, FALLBACK_TF = 6650.0, 1590.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM, FALLBACK_TF, 1400.0, "fallback"


def kernel_source_hash(names):
    """Hash of the kernel sources with comments and layout removed: an edit
    of a comment leaves it (and the committed ncu traffic) valid, any change
    of code does not."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "int8_weight_only_b200", "csrc", n)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, sources):
    """DRAM bytes per launch from a committed ncu summary, only if the
    kernel sources are unchanged since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[kernel]
        if t["source_hash"] == kernel_source_hash(sources):
            return float(t["bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,power.draw")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        self.windows = []

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def window_mhz(self, window):
        """Median SM clock sampled inside one timed window (after stop())."""
        a, b = window
        vals = [r[1] for r in getattr(self, "rows", []) if a - 0.15 <= r[0] <= b + 0.15]
        return statistics.median(vals) if vals else None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = []
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts + frac, float(parts[1]), float(parts[2]), parts[3:7]))
            except Exception:
                continue
        os.unlink(self.f.name)
        self.rows = rows
        inside = [r for r in rows if any(a - 0.15 <= r[0] <= b + 0.15 for a, b in self.windows)]
        use = inside if len(inside) >= 2 else rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use),
                "window": "timed regions" if use is inside else "whole run"}


# ------------------------------------------------------------------ helpers
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl" if os.environ.get("W8_BENCH_BACKEND", "nccl") == "nccl" else "gloo",
                                timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, value: float, device) -> float:
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_sequence(seq, stream, ws, device, sampler):
    """Replay each (graph, n) of `seq` n times, in order, between a barrier
    and a synchronize on both sides; device time in s (CUDA events on the
    launching stream), max over ranks."""
    import torch
    barrier(ws)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        for graph, n in seq:
            for _ in range(n):
                graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    sampler.mark(t0, time.time())
    elapsed = start.elapsed_time(end) / 1e3
    barrier(ws)
    return max_over_ranks(ws, elapsed, device)


def timed_replays(graph, n_replays, stream, ws, device, sampler):
    """Replay `graph` n_replays times between synchronizes; device time in s."""
    return timed_sequence([(graph, n_replays)], stream, ws, device, sampler)


def replay_times(graph, reps, stream, ws, device, sampler):
    """Device time (s) of each of `reps` replays of `graph`, CUDA events
    around every replay on the launching stream; max over ranks per replay."""
    import torch
    barrier(ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    t0 = time.time()
    with torch.cuda.stream(stream):
        for a, b in evs:
            a.record(stream)
            graph.replay()
            b.record(stream)
    torch.cuda.synchronize()
    sampler.mark(t0, time.time())
    out = [max_over_ranks(ws, a.elapsed_time(b) / 1e3, device) for a, b in evs]
    barrier(ws)
    return out


# The measured bf16 peaks: a burst (best of 10 GEMMs) and a seconds-long
# loop under the power cap.  A timed region shorter than SUSTAINED_S is
# compared with the burst figure.
SUSTAINED_S = 2.0
# Idle time before the variants' prefill timings (see there).
IDLE_S = 2.0


def tensor_peak(region_s, tf_peak, tf_sustained):
    if region_s >= SUSTAINED_S and tf_sustained > 0:
        return tf_sustained, "bf16_tflops_sustained"
    return tf_peak, "bf16_tflops (burst)"


def capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


# ------------------------------------------------------------------ native arm
def run_native(args, ws, rank, local):
    import torch
    import synthetic
    import int8_weight_only_b200 as w8
    from int8_weight_only_b200 import build as w8build

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if rank == 0:
        w8build.build()
    barrier(ws)
    w8.load_library()
    hbm_peak, tf_peak, tf_sustained, peak_src = peaks()
    sampler = ClockSampler(local)
    stream = torch.cuda.Stream(device)

    # ---- inputs (host, seeded) -> device
    seed = synthetic.SEED + rank
    tid = synthetic.tensor_id(2, 0, 0, 0)
    W_host = synthetic.weights(K_DIM, N_DIM, seed, tid, outlier_frac=0.001)
    X1_host = synthetic.activations(M_DECODE, K_DIM, seed, tid + 1)
    Xp_host = synthetic.activations(M_PREFILL, K_DIM, seed, synthetic.tensor_id(4, M_PREFILL, 0, 1))
    W = torch.from_numpy(W_host).to(device)
    X1 = torch.from_numpy(X1_host).to(device)
    Xp = torch.from_numpy(Xp_host).to(device)
    del W_host

    with torch.cuda.stream(stream):
        q, scales = w8.quantize(W)
        packed0 = w8.prepack(q)
        copies = [packed0] + [packed0.clone() for _ in range(N_COPIES - 1)]
        Y1 = torch.empty((M_DECODE, N_DIM), dtype=torch.float16, device=device)
        Yp = torch.empty((M_PREFILL, N_DIM), dtype=torch.float16, device=device)
        ws_need = w8.workspace_bytes(M_DECODE, K_DIM, N_DIM, device)
        work = torch.zeros((max(ws_need, 1),), dtype=torch.uint8, device=device)
        # warm-up of every entry point outside capture (one-time device setup)
        w8.linear(X1, copies[0], scales, out=Y1, workspace=work)
        w8.linear(Xp, copies[0], scales, out=Yp)
    torch.cuda.synchronize()

    steps, warmup = args.steps, args.warmup

    # ---- decode (headline): a graph of N_COPIES calls, rotating the weight copy
    def decode_round():
        for c in copies:
            w8.linear(X1, c, scales, out=Y1, workspace=work)

    # exactly `steps` timed calls, cycling the 6 copies: one graph of
    # min(steps, DECODE_GRAPH_STEPS) calls (a multiple of 6 when it is
    # replayed), replayed steps // that many times, then a graph of the
    # remaining calls.  Graph launches are the only breaks in the calls'
    # programmatic overlap, so short runs take one graph.
    def decode_calls(n):
        for i in range(n):
            w8.linear(X1, copies[i % N_COPIES], scales, out=Y1, workspace=work)

    per_graph = steps if steps <= DECODE_GRAPH_STEPS else DECODE_GRAPH_STEPS
    g_dec = capture(decode_round, stream)       # the 6 copies once: warm-up and medians
    g_run = capture(lambda: decode_calls(per_graph), stream)
    rem = steps % per_graph
    g_rem = capture(lambda: decode_calls(rem), stream) if rem else None
    for _ in range(max(1, -(-warmup // N_COPIES))):
        with torch.cuda.stream(stream):
            g_dec.replay()
    with torch.cuda.stream(stream):   # each timed graph's first launch (its upload) outside the region
        g_run.replay()
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize()
    t_dec = timed_sequence([(g_run, steps // per_graph), (g_rem, 1 if rem else 0)], stream, ws, device, sampler)
    steps_done = steps
    dec_s = t_dec / steps_done
    weight_bytes = K_DIM * N_DIM
    alg_bytes = weight_bytes + 2 * N_DIM + 2 * M_DECODE * K_DIM + 2 * M_DECODE * N_DIM
    value = ws * weight_bytes * steps_done / t_dec / 1e9
    dec_achieved = alg_bytes / dec_s / 1e9
    # microseconds per call as the median of DECODE_REPS timed repetitions
    # (each a replay of the 6-copy graph, CUDA events around it)
    rep_t = replay_times(g_dec, DECODE_REPS, stream, ws, device, sampler)
    dec_med_s = statistics.median(rep_t) / N_COPIES

    # ---- quantize (fp32 W 449 MB > L2) and prepack (one-time weight path)
    q2 = torch.empty_like(q)
    s2 = torch.empty_like(scales)
    g_q = capture(lambda: w8.quantize(W, q=q2, scales=s2), stream)
    g_pk = capture(lambda: w8.prepack(q2, out=copies[1]), stream)
    for g in (g_q, g_pk):
        for _ in range(3):
            with torch.cuda.stream(stream):
                g.replay()
    torch.cuda.synchronize()
    n_q = max(5, args.prefill_reps)
    t_q = timed_replays(g_q, n_q, stream, ws, device, sampler) / n_q
    t_pk = timed_replays(g_pk, n_q, stream, ws, device, sampler) / n_q
    t_q_med = statistics.median(replay_times(g_q, 50, stream, ws, device, sampler))
    q_bytes = K_DIM * N_DIM * (4 + 1) + 2 * N_DIM
    pk_bytes = 2 * K_DIM * N_DIM
    same = bool(torch.equal(q, q2) and torch.equal(scales, s2))

    # ---- e2e: per step, the H2D copy of X from pinned host memory, the
    # public linear call and the D2H copy of Y to pinned host memory.  Two
    # X and two Y buffers on each side; the copies run on two copy streams
    # ordered against the compute stream by events, so step i+1's X comes in
    # and step i's Y goes out while step i or i+1 computes.
    h2d_stream = torch.cuda.Stream(device)
    d2h_stream = torch.cuda.Stream(device)
    Xh = [torch.from_numpy(X1_host).pin_memory() for _ in range(2)]
    Yh = [torch.empty((M_DECODE, N_DIM), dtype=torch.float16).pin_memory() for _ in range(2)]
    Xd = [torch.empty_like(X1) for _ in range(2)]
    Yd = [torch.empty_like(Y1) for _ in range(2)]

    def e2e_steps(n):
        cur = torch.cuda.current_stream(device)
        h2d_stream.wait_stream(cur)
        d2h_stream.wait_stream(cur)
        computed = [None, None]   # compute of the last step that used slot
        drained = [None, None]    # D2H of the last step that used slot
        for i in range(n):
            sl = i % 2
            if computed[sl] is not None:
                h2d_stream.wait_event(computed[sl])       # X[sl] no longer read
            with torch.cuda.stream(h2d_stream):
                Xd[sl].copy_(Xh[sl], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(h2d_stream)
            cur.wait_event(landed)
            if drained[sl] is not None:
                cur.wait_event(drained[sl])              # Y[sl] already copied out
            w8.linear(Xd[sl], copies[i % N_COPIES], scales, out=Yd[sl], workspace=work)
            computed[sl] = torch.cuda.Event()
            computed[sl].record(cur)
            d2h_stream.wait_event(computed[sl])
            with torch.cuda.stream(d2h_stream):
                Yh[sl].copy_(Yd[sl], non_blocking=True)
            drained[sl] = torch.cuda.Event()
            drained[sl].record(d2h_stream)
        cur.wait_stream(h2d_stream)
        cur.wait_stream(d2h_stream)

    e2e_full = min(steps, E2E_GRAPH_STEPS)
    g_e2e = capture(lambda: e2e_steps(e2e_full), stream)
    e2e_rem = steps % e2e_full
    g_e2e_rem = capture(lambda: e2e_steps(e2e_rem), stream) if e2e_rem else None
    for _ in range(2):
        with torch.cuda.stream(stream):
            g_e2e.replay()
    if g_e2e_rem is not None:
        with torch.cuda.stream(stream):
            g_e2e_rem.replay()
    torch.cuda.synchronize()
    t_e2e = timed_sequence([(g_e2e, steps // e2e_full), (g_e2e_rem, 1 if e2e_rem else 0)],
                           stream, ws, device, sampler)
    e2e_value = ws * weight_bytes * steps / t_e2e / 1e9
    e2e_ok = bool(torch.equal(Yh[0].to(device), Y1) or torch.equal(Yh[1].to(device), Y1))

    def graph_time(fn, reps):
        """Device seconds per call of fn: captured once, replayed; the median
        of max(reps, 50) timed replays, CUDA events around each."""
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        g = capture(fn, stream)
        for _ in range(3):
            with torch.cuda.stream(stream):
                g.replay()
        torch.cuda.synchronize()
        t = statistics.median(replay_times(g, max(reps, 50), stream, ws, device, sampler))
        del g
        return t

    # ---- the method's variants on the headline weight (4096 x 27392, 0.1 %
    # outliers): asymmetric codes, clipped scales, the outlier split.  Their
    # memory-bound calls (quantizers, decode) are timed here, before the
    # prefill loop; their prefill calls after it.
    variants = {}
    if not args.no_variants:
        qa, sa, za = w8.quantize_asym(W)
        pa = [w8.prepack(qa) for _ in range(N_COPIES)]
        t_qa = graph_time(lambda: w8.quantize_asym(W, qa, sa, za), 20)
        t_da = graph_time(lambda: [w8.linear_asym(X1, c, sa, za, out=Y1, workspace=work) for c in pa],
                          DECODE_REPS) / N_COPIES
        variants["asymmetric"] = {
            "quantize_us": round(t_qa * 1e6, 1), "quantize_GBps": round(q_bytes / t_qa / 1e9, 1),
            "quantize_frac_hbm": round(q_bytes / t_qa / 1e9 / hbm_peak, 4),
            "decode_m1_us": round(t_da * 1e6, 2), "decode_m1_weight_GBps": round(weight_bytes / t_da / 1e9, 1),
            "decode_m1_frac_hbm": round(alg_bytes / t_da / 1e9 / hbm_peak, 4)}
        del pa[2:]
        qc = torch.empty_like(q)
        sc_ = torch.empty_like(scales)
        t_cf = graph_time(lambda: w8.quantize_clip(W, "fixed", 0.05, qc, sc_), 20)
        t_cp = graph_time(lambda: w8.quantize_clip(W, "percentile", 0.999, qc, sc_), 5)
        variants["clip_fixed"] = {"clip": 0.05, "quantize_us": round(t_cf * 1e6, 1),
                                  "quantize_GBps": round(q_bytes / t_cf / 1e9, 1)}
        variants["clip_percentile"] = {"p": 0.999, "quantize_us": round(t_cp * 1e6, 1),
                                       "quantize_GBps": round(q_bytes / t_cp / 1e9, 1),
                                       "quantize_frac_hbm": round(q_bytes / t_cp / 1e9 / hbm_peak, 4)}
        qo, so, co, ro, vo = w8.quantize_outliers(W, 0.999)
        po = [w8.prepack(qo) for _ in range(N_COPIES)]
        t_qo = graph_time(lambda: w8.quantize_outliers(W, 0.999), 5)
        t_do = graph_time(lambda: [w8.linear_outliers(X1, c, so, co, ro, vo, out=Y1) for c in po],
                          DECODE_REPS) / N_COPIES
        variants["outlier_split"] = {
            "p": 0.999, "outliers_per_channel": int(ro.shape[1]), "quantize_us": round(t_qo * 1e6, 1),
            "decode_m1_us": round(t_do * 1e6, 2), "decode_m1_weight_GBps": round(weight_bytes / t_do / 1e9, 1),
            "decode_m1_frac_hbm": round(alg_bytes / t_do / 1e9 / hbm_peak, 4)}
        del po[2:], qo, qc
        torch.cuda.empty_cache()

    # ---- the variants' prefill calls (M = 2048), each timed as the plain
    # call is (a graph of two calls, back to back) and, like the plain call
    # timed for them, from an idle GPU: after seconds of power-capped tensor
    # work the outlier split's call measured up to 37 % slower (440 -> 602
    # us) and the plain call 17 % (298 -> 349 us), and two idle seconds
    # brought both back
    if not args.no_variants:
        fl_pf = 2.0 * M_PREFILL * K_DIM * N_DIM

        def from_idle(fn):
            torch.cuda.synchronize()
            time.sleep(IDLE_S)
            return graph_time(fn, 20) / 2

        t_plain = from_idle(lambda: [w8.linear(Xp, c, scales, out=Yp) for c in copies[:2]])
        t_pa = from_idle(lambda: [w8.linear_asym(Xp, c, sa, za, out=Yp) for c in pa])
        t_po = from_idle(lambda: [w8.linear_outliers(Xp, c, so, co, ro, vo, out=Yp) for c in po])
        variants["asymmetric"].update({
            "prefill_m2048_us": round(t_pa * 1e6, 1), "prefill_m2048_TFLOPs": round(fl_pf / t_pa / 1e12, 1),
            "prefill_m2048_frac_tensor_burst": round(fl_pf / t_pa / 1e12 / tf_peak, 4),
            "prefill_m2048_vs_plain": round(t_pa / t_plain, 3)})
        variants["outlier_split"].update({
            "prefill_m2048_us": round(t_po * 1e6, 1), "prefill_m2048_TFLOPs": round(fl_pf / t_po / 1e12, 1),
            "prefill_m2048_frac_tensor_burst": round(fl_pf / t_po / 1e12 / tf_peak, 4),
            "prefill_m2048_vs_plain": round(t_po / t_plain, 3)})
        variants["prefill_m2048_plain_us_alongside"] = round(t_plain * 1e6, 1)
        variants["prefill_m2048_timed_from"] = f"an idle GPU ({IDLE_S} s before each of the three)"
        del pa, po
        torch.cuda.empty_cache()

    # ---- prefill M = 2048 (two weight copies alternate: 224 MB > L2); after
    # the memory-bound sections, whose numbers a power-capped tensor-core
    # loop just before would skew
    def prefill_round():
        for c in copies[:2]:
            w8.linear(Xp, c, scales, out=Yp)

    g_pf = capture(prefill_round, stream)
    for _ in range(3):
        with torch.cuda.stream(stream):
            g_pf.replay()
    torch.cuda.synchronize()
    n_pf = max(5, args.prefill_reps)
    t_pf = timed_replays(g_pf, n_pf, stream, ws, device, sampler)
    pf_window = sampler.windows[-1]
    pf_s = t_pf / (2 * n_pf)
    pf_flops = 2.0 * M_PREFILL * K_DIM * N_DIM
    pf_tflops = pf_flops / pf_s / 1e12
    pf_peak, pf_peak_name = tensor_peak(t_pf, tf_peak, tf_sustained)
    pf_med_s = statistics.median(replay_times(g_pf, 50, stream, ws, device, sampler)) / 2

    # ---- the prefill sweep: M in {512, 1024, 2048} on 4096 x 27392 and
    # 13696 x 4096 (the latter's few tiles take the K split at M = 512)
    prefill_sweep = {}
    if not args.no_variants:
        sw = synthetic.WORKLOADS["chatglm2_prefill"]
        for i, (Ks, Ns) in enumerate(sw["matrices"]):
            Ws = torch.from_numpy(synthetic.weights(Ks, Ns, seed, synthetic.tensor_id(4, 0, i, 0),
                                                    outlier_frac=0.001)).to(device)
            qs, ss = w8.quantize(Ws)
            del Ws
            ncp = 2 if Ks * Ns > 64 << 20 else 4
            ps = [w8.prepack(qs) for _ in range(ncp)]
            row = {}
            for Ms in sw["M"]:
                Xs = torch.from_numpy(synthetic.activations(Ms, Ks, seed, synthetic.tensor_id(4, Ms, i, 1))).to(device)
                Ysw = torch.empty((Ms, Ns), dtype=torch.float16, device=device)
                t = graph_time(lambda: [w8.linear(Xs, c, ss, out=Ysw) for c in ps], 20) / ncp
                tf = 2.0 * Ms * Ks * Ns / t / 1e12
                row[f"M={Ms}"] = {"us": round(t * 1e6, 1), "TFLOPs": round(tf, 1),
                                  "frac_tensor_burst": round(tf / tf_peak, 4)}
                del Xs, Ysw
            prefill_sweep[f"{Ks}x{Ns}"] = row
            del ps, qs
        torch.cuda.empty_cache()

    # ---- BERT-base, 4096 tokens: quantize all 12 layers' 48 weights, then
    # the four linears of a layer at M = 4096 (distinct weights per layer)
    bert = {}
    if not args.no_variants:
        bw = synthetic.WORKLOADS["bert_base_4096_tokens"]
        Wb, qb, sb, pb = [], [], [], []
        for i, (Kb, Nb) in enumerate(bw["matrices"]):
            w0 = torch.from_numpy(synthetic.weights(Kb, Nb, seed, synthetic.tensor_id(5, 0, i, 0))).to(device)
            Wb.append([w0] + [w0.clone() for _ in range(bw["layers"] - 1)])
            qb.append([torch.empty((Kb, Nb), dtype=torch.int8, device=device) for _ in range(bw["layers"])])
            sb.append([torch.empty((Nb,), dtype=torch.float16, device=device) for _ in range(bw["layers"])])
        flat_w = [Wb[i][l] for i in range(len(Wb)) for l in range(bw["layers"])]
        flat_q = [qb[i][l] for i in range(len(Wb)) for l in range(bw["layers"])]
        flat_s = [sb[i][l] for i in range(len(Wb)) for l in range(bw["layers"])]

        def bert_quantize_each():
            for W_, q_, s_ in zip(flat_w, flat_q, flat_s):
                w8.quantize(W_, q_, s_)

        def bert_quantize_batched():
            w8.quantize_batched(flat_w, flat_q, flat_s)

        t_bq1 = graph_time(bert_quantize_each, 5)
        t_bq = graph_time(bert_quantize_batched, 5)
        bq_bytes = bw["layers"] * sum(Kb * Nb * 5 + 2 * Nb for Kb, Nb in bw["matrices"])
        for i in range(len(Wb)):
            pb.append([w8.prepack(qb[i][l]) for l in range(bw["layers"])])
        del Wb
        Mb = bw["M"][0]
        Xb = [torch.from_numpy(synthetic.activations(Mb, Kb, seed, synthetic.tensor_id(5, 0, i, 1))).to(device)
              for i, (Kb, Nb) in enumerate(bw["matrices"])]
        Yb = [torch.empty((Mb, Nb), dtype=torch.float16, device=device) for Kb, Nb in bw["matrices"]]
        def bert_layers():
            for l in range(bw["layers"]):
                for i in range(len(pb)):
                    w8.linear(Xb[i], pb[i][l], sb[i][l], out=Yb[i])
        t_bl = graph_time(bert_layers, 5)
        bl_flops = bw["layers"] * sum(2.0 * Mb * Kb * Nb for Kb, Nb in bw["matrices"])
        bert = {"workload": "BERT-base, 4096 tokens: QKV 768x2304, out 768x768, FFN 768x3072 and 3072x768, "
                            "x 12 layers (distinct weights)",
                "quantize_all_us": round(t_bq * 1e6, 1), "quantize_GBps": round(bq_bytes / t_bq / 1e9, 1),
                "quantize_launches": 1,
                "quantize_one_launch_per_weight_us": round(t_bq1 * 1e6, 1),
                "linears_us_per_layer": round(t_bl * 1e6 / bw["layers"], 1),
                "linears_TFLOPs": round(bl_flops / t_bl / 1e12, 1),
                "linears_frac_tensor_burst": round(bl_flops / t_bl / 1e12 / tf_peak, 4)}
        del pb, Xb, Yb, qb
        torch.cuda.empty_cache()

    # ---- the ChatGLM2-6B decode layer set: 28 layers x 4 linears (QKV,
    # dense, h-to-4h, 4h-to-h), each call on its own weight buffer (5.7 GB
    # in all, so nothing is served from L2), chained in one CUDA graph
    decode_set = {}
    if not args.no_decode_set:
        spec = synthetic.WORKLOADS["chatglm2_decode_set"]
        mats, layers = spec["matrices"], spec["layers"]
        packed_set, scale_set = [], []
        for i, (Kd, Nd) in enumerate(mats):
            Wd = torch.from_numpy(synthetic.weights(Kd, Nd, seed, synthetic.tensor_id(3, 0, i, 0),
                                                    outlier_frac=spec["outlier_frac"])).to(device)
            with torch.cuda.stream(stream):
                qd, sd = w8.quantize(Wd)
                pd = w8.prepack(qd)
            torch.cuda.synchronize()
            del Wd, qd
            # distinct buffers per layer (copies of one synthetic layer)
            packed_set.append([pd] + [pd.clone() for _ in range(layers - 1)])
            scale_set.append(sd)
        set_bytes = layers * sum(Kd * Nd for Kd, Nd in mats)
        names = ["qkv", "dense", "h_to_4h", "4h_to_h"]
        for Md in (1, 16):
            Xs = [torch.from_numpy(synthetic.activations(Md, Kd, seed, synthetic.tensor_id(3, Md, i, 1))).to(device)
                  for i, (Kd, Nd) in enumerate(mats)]
            Ys = [torch.empty((Md, Nd), dtype=torch.float16, device=device) for Kd, Nd in mats]
            wsd = torch.zeros((max(w8.workspace_bytes(Md, Kd, Nd, device) for Kd, Nd in mats),),
                              dtype=torch.uint8, device=device)

            def set_round():
                for layer in range(layers):
                    for i in range(len(mats)):
                        w8.linear(Xs[i], packed_set[i][layer], scale_set[i], out=Ys[i], workspace=wsd)

            with torch.cuda.stream(stream):
                set_round()   # first calls outside capture
            torch.cuda.synchronize()
            g_set = capture(set_round, stream)
            for _ in range(3):
                with torch.cuda.stream(stream):
                    g_set.replay()
            torch.cuda.synchronize()
            reps = max(10, args.set_reps)
            t_set = timed_replays(g_set, reps, stream, ws, device, sampler) / reps
            entry = {
                "us_per_layer_set": round(t_set * 1e6, 1),
                "us_per_layer": round(t_set * 1e6 / layers, 2),
                "weight_GBps": round(set_bytes / t_set / 1e9, 1),
                "frac_hbm": round(set_bytes / t_set / 1e9 / hbm_peak, 4),
                "linears": layers * len(mats), "weight_bytes": set_bytes,
            }
            del g_set
            # per shape: the 28 layers' calls of one matrix in one graph
            # (28 distinct weights, > L2), median of DECODE_REPS replays
            for i, (Kd, Nd) in enumerate(mats):
                def shape_round(i=i):
                    for layer in range(layers):
                        w8.linear(Xs[i], packed_set[i][layer], scale_set[i], out=Ys[i], workspace=wsd)
                g_sh = capture(shape_round, stream)
                for _ in range(2):
                    with torch.cuda.stream(stream):
                        g_sh.replay()
                torch.cuda.synchronize()
                t_call = statistics.median(replay_times(g_sh, DECODE_REPS, stream, ws, device, sampler)) / layers
                alg = Kd * Nd + 2 * Nd + 2 * Md * Kd + 2 * Md * Nd
                entry[f"{names[i]}_{Kd}x{Nd}"] = {
                    "us_per_call": round(t_call * 1e6, 2),
                    "weight_GBps": round(Kd * Nd / t_call / 1e9, 1),
                    "frac_hbm": round(alg / t_call / 1e9 / hbm_peak, 4),
                    "algorithmic_bytes": alg}
                del g_sh
            decode_set[f"M={Md}"] = entry
        del packed_set

    clocks = sampler.stop()
    pf_mhz = sampler.window_mhz(pf_window)

    pf_region_s = t_pf
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": steps_done,
        "warmup": warmup,
        "ms_per_step": round(dec_s * 1e3, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": WORKLOAD,
            "M": M_DECODE, "K": K_DIM, "N": N_DIM,
            "weights": "int8 per-output-channel, fp16 scales, prepacked tiles",
            "l2": f"inputs larger than L2: {N_COPIES} rotating weight copies "
                  f"({N_COPIES * weight_bytes / 1e6:.0f} MB), calls captured in CUDA graphs of "
                  f"{per_graph} calls",
            "parallelism": f"replicas x{ws} (independent problems, no collective)",
        },
        "roofline": {
            "bound": "hbm", "achieved": round(dec_achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(dec_achieved / hbm_peak, 4),
            "traffic": measured_traffic("decode_kernel", ["decode.cuh", "common.cuh"]),
            "kernel": "w8::decode::decode_kernel<1>",
            "algorithmic_bytes_per_launch": alg_bytes,
            "peak_source": f"{peak_src} hbm_gbs",
            "achieved_from": f"mean launch time over the {steps_done} timed calls",
        },
        "decode": {
            "us_per_call_median": round(dec_med_s * 1e6, 3),
            "us_per_call_mean_timed_region": round(dec_s * 1e6, 3),
            "median_of": f"{DECODE_REPS} timed repetitions of {N_COPIES} calls (one per weight copy)",
            "weight_GBps_at_median": round(weight_bytes / dec_med_s / 1e9, 1),
            "frac_hbm_at_median": round(alg_bytes / dec_med_s / 1e9 / hbm_peak, 4),
        },
        "prefill": {
            "metric": "TFLOP/s (M=2048, 4096x27392)", "value": round(pf_tflops, 1), "unit": "TFLOP/s",
            "us_per_call": round(pf_s * 1e6, 2),
            "us_per_call_median": round(pf_med_s * 1e6, 2),
            "calls_timed": 2 * n_pf,
            "timed_region_s": round(pf_region_s, 4),
            "sm_mhz_median_in_region": pf_mhz,
            "roofline": {"bound": "tensor", "achieved": round(pf_tflops, 1), "peak": pf_peak,
                         "unit": "TFLOP/s", "frac": round(pf_tflops / pf_peak, 4),
                         "frac_of_sustained": round(pf_tflops / tf_sustained, 4) if tf_sustained else None,
                         "traffic": measured_traffic("prefill2_kernel", ["prefill2.cuh", "common.cuh"]),
                         "kernel": "w8::prefill2::prefill2_kernel (CTA pairs)",
                         "peak_source": f"{peak_src} {pf_peak_name} x fp16/bf16 nominal ratio 1 "
                                        f"(timed region {pf_region_s:.3f} s; the sustained figure "
                                        f"{tf_sustained} applies to regions of {SUSTAINED_S:.0f} s or more)"},
        },
        "quantize": {
            "us_per_call": round(t_q * 1e6, 2), "us_per_call_median": round(t_q_med * 1e6, 2),
            "algorithmic_GBps": round(q_bytes / t_q / 1e9, 1),
            "frac_hbm": round(q_bytes / t_q / 1e9 / hbm_peak, 4), "bit_identical_rerun": same,
            "traffic": measured_traffic("quantize_kernel", ["quantize.cuh", "common.cuh"]),
        },
        "prepack": {"us_per_call": round(t_pk * 1e6, 2),
                    "algorithmic_GBps": round(pk_bytes / t_pk / 1e9, 1)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(Xh[0].numel() * Xh[0].element_size()),
                "d2h_bytes_per_step": int(Yh[0].numel() * Yh[0].element_size()),
                "steps": steps, "frac_of_device_value": round(e2e_value / value, 4),
                "result_read_back_matches": e2e_ok,
                "how": "per step: pinned-host X -> device copy, the public linear call, device -> pinned-host "
                       "Y copy; copies on two copy streams, double-buffered, ordered by events; "
                       f"graphs of {e2e_full} steps"},
        "decode_set": ({"workload": "ChatGLM2-6B decode linears, 28 layers x (QKV 4096x4608, dense 4096x4096, "
                                    "h-to-4h 4096x27392, 4h-to-h 13696x4096), distinct weight buffers, one CUDA graph",
                        **decode_set} if decode_set else None),
        "variants": variants or None,
        "prefill_sweep": prefill_sweep or None,
        "bert_base_4096": bert or None,
        "gpu_launches": steps_done,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    del g_dec, g_run, g_rem, g_pf, g_q, g_pk, g_e2e, g_e2e_rem
    return out


# ------------------------------------------------------------------ profiling driver
def run_profile(args):
    """A few plain launches of one kernel, for ncu captures (no graphs, no
    timing): the bench's workload, or the weight shape --profile-shape KxN
    (and --profile-m tokens).  Packed-weight copies alternate (at least 2, and enough for more than
    256 MB), so the weight is not served from L2."""
    import torch
    import synthetic
    import int8_weight_only_b200 as w8
    from int8_weight_only_b200 import build as w8build

    w8build.build()
    w8.load_library()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    K, N = (int(v) for v in args.profile_shape.lower().split("x")) if args.profile_shape else (K_DIM, N_DIM)
    tid = synthetic.tensor_id(2, 0, 0, 0)
    W = torch.from_numpy(synthetic.weights(K, N, synthetic.SEED, tid, outlier_frac=0.001)).to(device)
    q, scales = w8.quantize(W)
    ncp = max(2, -(-(256 << 20) // (K * N)))
    copies = [w8.prepack(q) for _ in range(ncp)]
    M = {"decode": M_DECODE, "decode16": 16, "prefill": M_PREFILL}.get(args.profile, M_DECODE)
    if args.profile_m:
        M = args.profile_m
    X = torch.from_numpy(synthetic.activations(M, K, synthetic.SEED, tid + 1)).to(device)
    Y = torch.empty((M, N), dtype=torch.float16, device=device)
    torch.cuda.synchronize()
    for i in range(args.steps):
        if args.profile in ("decode", "decode16", "prefill"):
            w8.linear(X, copies[i % ncp], scales, out=Y)
        elif args.profile == "quantize":
            w8.quantize(W, q=q, scales=scales)
        elif args.profile == "percentile":
            w8.quantize_clip(W, "percentile", 0.999, q=q, scales=scales)
        elif args.profile == "prepack":
            w8.prepack(q, out=copies[i % ncp])
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "launches": args.steps, "M": M, "K": K, "N": N}))
    return 0


# ------------------------------------------------------------------ oracle arm
def host_cpu():
    """(logical CPUs this process may use, CPU model name)."""
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return n, model


def column_slabs(q, chan, width):
    """q [K, N] and per-channel arrays cut into contiguous column slabs
    (done once, before any timing)."""
    N = q.shape[1]
    return [(np.ascontiguousarray(q[:, a:min(N, a + width)]),
             [np.ascontiguousarray(c[a:min(N, a + width)]) for c in chan]) for a in range(0, N, width)]


class SlabRunner:
    """Runs one of the oracle's functions over column slabs on a fixed pool
    of host threads.  Every output channel of the oracle is computed on its
    own, so the slabs give the oracle's whole-matrix result; only the wall
    time depends on the thread count."""

    def __init__(self, threads):
        from concurrent.futures import ThreadPoolExecutor
        self.threads = threads
        self.pool = ThreadPoolExecutor(max_workers=threads) if threads > 1 else None

    def map(self, fn, slabs):
        if self.pool is None:
            return [fn(*sl) for sl in slabs]
        return list(self.pool.map(lambda sl: fn(*sl), slabs))

    def close(self):
        if self.pool is not None:
            self.pool.shutdown()


def linear_width(K):
    """Columns per slab: about 1 MB of int8 codes."""
    return max(64, ((1 << 20) // K) // 64 * 64)


def time_repeated(fn, min_s):
    """Wall seconds per call of fn, repeated until min_s has passed (one
    untimed call first, unless min_s is 0: then a single timed call)."""
    if min_s > 0:
        fn()
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s:
            return el / reps, reps


def oracle_quantize_threads(W, runner):
    import oracle
    parts = runner.map(lambda w, _: oracle.quantize(w), column_slabs(W, [], 1024))
    return np.concatenate([p[0] for p in parts], axis=1), np.concatenate([p[1] for p in parts])


def oracle_linear_timer(X, q, s, runner):
    """A callable that runs the oracle's linear X . dequant(q, s) over column
    slabs prepared once here."""
    import oracle
    slabs = column_slabs(q, [s], linear_width(q.shape[0]))
    return lambda: runner.map(lambda qs, ch: oracle.linear(X, qs, ch[0]), slabs)


def cpu_baseline(min_s: float):
    """The CPU oracle as it stands, timed on this host's cores, on bounded
    samples of the workloads.  Headline: the decode call (M = 1, 4096 x
    27392) with the oracle driven over column slabs on every core; beside it
    one core, and the other workloads: the tiny one, one ChatGLM2 decode
    layer at M = 16 and the prefill shapes at M = 512."""
    import oracle
    import synthetic
    threads, model = host_cpu()
    runner, single = SlabRunner(threads), SlabRunner(1)
    seed = synthetic.SEED
    tid = synthetic.tensor_id(2, 0, 0, 0)
    W = synthetic.weights(K_DIM, N_DIM, seed, tid, outlier_frac=0.001)
    X1 = synthetic.activations(M_DECODE, K_DIM, seed, tid + 1)
    q, s = oracle_quantize_threads(W, runner)
    t_all, r_all = time_repeated(oracle_linear_timer(X1, q, s, runner), min_s)
    slab = 4096
    t_one, r_one = time_repeated(oracle_linear_timer(X1, q[:, :slab], s[:slab], single), min_s)
    Wslabs = column_slabs(W, [], 1024)
    t_q_all, _ = time_repeated(lambda: runner.map(lambda w, _: oracle.quantize(w), Wslabs), min_s / 2)
    Ws1 = np.ascontiguousarray(W[:, :slab])
    t_q_one, _ = time_repeated(lambda: oracle.quantize(Ws1), min_s / 2)
    del Wslabs, Ws1, W
    out = {"value": round(K_DIM * N_DIM / t_all / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
           "cpu_model": model,
           "sample": f"{r_all} x oracle linear, M=1, the whole 4096x27392 weight, on column slabs over "
                     f"{threads} host threads ({r_all * t_all:.1f} s)"}
    cfg = {
        "chatglm2_h_to_4h_decode": {
            "linear_M1_all_cores": {"threads": threads, "ms_per_call": round(t_all * 1e3, 2),
                                    "weight_GBps": round(K_DIM * N_DIM / t_all / 1e9, 4)},
            "linear_M1_one_core": {"threads": 1, "sample": f"4096x{slab} column slab",
                                   "weight_GBps": round(K_DIM * slab / t_one / 1e9, 4)},
            "quantize_all_cores": {"threads": threads, "ms_per_call": round(t_q_all * 1e3, 1),
                                   "algorithmic_GBps": round((K_DIM * N_DIM * 5 + 2 * N_DIM) / t_q_all / 1e9, 4)},
            "quantize_one_core": {"threads": 1, "sample": f"4096x{slab} column slab",
                                  "algorithmic_GBps": round((K_DIM * slab * 5 + 2 * slab) / t_q_one / 1e9, 4)},
        }}
    # tiny workload: quantize + linear, one core
    Wt = synthetic.weights(256, 512, seed, synthetic.tensor_id(1, 0, 0, 0))
    Xt = synthetic.activations(4, 256, seed, synthetic.tensor_id(1, 4, 0, 1))

    def tiny():
        qt, st = oracle.quantize(Wt)
        oracle.linear(Xt, qt, st)

    t_tiny, _ = time_repeated(tiny, min_s / 4)
    cfg["tiny"] = {"threads": 1, "us_per_quantize_and_linear": round(t_tiny * 1e6, 1)}
    # one ChatGLM2 decode layer (4 linears) at M = 16, every core; the h-to-4h
    # weight above stands in for the layer's (same shape and statistics)
    mats = synthetic.WORKLOADS["chatglm2_decode_set"]["matrices"]
    layer, layer_bytes = [], 0
    for i, (Kd, Nd) in enumerate(mats):
        if (Kd, Nd) == (K_DIM, N_DIM):
            qd, sd = q, s
        else:
            qd, sd = oracle_quantize_threads(
                synthetic.weights(Kd, Nd, seed, synthetic.tensor_id(3, 0, i, 0), outlier_frac=0.001), runner)
        layer.append((qd, sd, oracle_linear_timer(synthetic.activations(16, Kd, seed, synthetic.tensor_id(3, 16, i, 1)),
                                                  qd, sd, runner)))
        layer_bytes += Kd * Nd
    t_layer, _ = time_repeated(lambda: [f() for _, _, f in layer], min_s)
    cfg["chatglm2_decode_layer_M16"] = {"threads": threads, "ms_per_layer": round(t_layer * 1e3, 1),
                                        "weight_GBps": round(layer_bytes / t_layer / 1e9, 4)}
    # prefill at M = 512 on both prefill shapes, every core; the decode-set
    # weights of the same shapes stand in for the prefill workload's
    Xp = synthetic.activations(512, K_DIM, seed, synthetic.tensor_id(4, 512, 0, 1))
    t_p0, _ = time_repeated(oracle_linear_timer(Xp, q, s, runner), 0.0)
    K4, N4 = mats[3]
    Xp1 = synthetic.activations(512, K4, seed, synthetic.tensor_id(4, 512, 1, 1))
    t_p1, _ = time_repeated(oracle_linear_timer(Xp1, layer[3][0], layer[3][1], runner), 0.0)
    cfg["chatglm2_prefill_M512"] = {
        "threads": threads,
        f"{K_DIM}x{N_DIM}": {"s_per_call": round(t_p0, 2), "GFLOPs": round(2 * 512 * K_DIM * N_DIM / t_p0 / 1e9, 2)},
        f"{K4}x{N4}": {"s_per_call": round(t_p1, 2), "GFLOPs": round(2 * 512 * K4 * N4 / t_p1 / 1e9, 2)},
        "note": "M=2048 is not timed: it is 4x the M=512 work"}
    out["configs"] = cfg
    runner.close()
    return out


def run_reference(args):
    """The reference arm of this benchmark: the CPU oracle, as it stands, on
    the headline workload (M = 1, the whole 4096 x 27392 weight per step),
    driven over column slabs on every host core."""
    import synthetic
    threads, model = host_cpu()
    runner = SlabRunner(threads)
    tid = synthetic.tensor_id(2, 0, 0, 0)
    W = synthetic.weights(K_DIM, N_DIM, synthetic.SEED, tid, outlier_frac=0.001)
    X = synthetic.activations(M_DECODE, K_DIM, synthetic.SEED, tid + 1)
    q, s = oracle_quantize_threads(W, runner)
    del W
    step = oracle_linear_timer(X, q, s, runner)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    runner.close()
    value = K_DIM * N_DIM * args.steps / el / 1e9
    sample = (f"{args.steps} steps, each the oracle's linear over the whole 4096x{N_DIM} weight at M=1, "
              f"on column slabs over {threads} host threads ({model})")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_DECODE, "K": K_DIM, "N": N_DIM, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "cpu_model": model, "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30000)
    ap.add_argument("--warmup", type=int, default=60)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--prefill-reps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=3.0,
                    help="minimum seconds per CPU-oracle measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-set", action="store_true",
                    help="skip the 28-layer decode set measurement")
    ap.add_argument("--set-reps", type=int, default=100)
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the variant, prefill-sweep and BERT sections")
    ap.add_argument("--profile", choices=["decode", "decode16", "prefill", "quantize", "percentile", "prepack"],
                    help="run --steps plain launches of one kernel (for ncu) and exit")
    ap.add_argument("--profile-shape", default="",
                    help="weight shape KxN for --profile (default: the bench's 4096x27392)")
    ap.add_argument("--profile-m", type=int, default=0,
                    help="tokens M for a linear --profile (default: the profile's own)")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args)
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    ws, rank, local = dist_setup()
    out = run_native(args, ws, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
