"""Benchmark of the partition-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the 720p attention step: partition attention of the fresh
(query group, KV group) pairs on the tensor cores, then the LSE merge with the cached
states and the fused partition importance.  Inputs are resident in HBM and larger than L2
(2.3 GB of Q/K/V, 25 GB of states per set).  Reported value: algorithmic TFLOP/s of the
step (fresh-pair flops / step time), whole job over N GPUs (replicas: each rank runs the
same workload on its own GPU, no data-path collective).  Extra keys: per-kernel times,
the merge and relayout HBM GB/s, the chunked relayout overlapped with attention on a
second stream, the end-to-end figure through host buffers, clocks, and the oracle timed on
the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "partition-attn TFLOP/s & 720p attn step ms on 1 B200; merge/relayout HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def workload_desc(wl):
    return (f"720p video DiT attention step: B{wl.B} H{wl.H} N{wl.N} (grid {wl.grid[0]}x"
            f"{wl.grid[1]}x{wl.grid[2]}) D{wl.D} {wl.dtype}, P={wl.P} (S={wl.S}, tail "
            f"{wl.N - (wl.P - 1) * wl.S}) G={wl.G}, nearest {wl.mask_keep} of {wl.KG} KV groups "
            f"fresh per query group, cached states from K,V + {wl.cache_sigma}*N(0,1); "
            "partition attention + merge with fused importance")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        self.proc = None
        self.lines = []
        try:
            pr = torch.cuda.get_device_properties(device_index)
            self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    """Max of a host scalar over the ranks (NCCL on the GPUs; gloo groups reduce on the host)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(ws, units_per_step, steps, elapsed_ms_max):
    """Whole-job throughput of `ws` replicas that each processed `units_per_step` per step
    for `steps` steps, timed by the slowest rank: units per second over all ranks."""
    return ws * units_per_step * steps / (elapsed_ms_max / 1e3)


# ------------------------------------------------------------------ traffic from the ncu summary
def traffic_per_launch():
    """dram read+write bytes per launch of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    src = os.path.join(ROOT, "sequence_partition_attn_b200", "csrc", "attn_tc.cu")
    summ = os.path.join(ROOT, "profiles", "partition_attn_720p.md")
    if not os.path.exists(summ):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    text = open(summ).read()
    m_src = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    if not m_src or not m_b or m_src.group(1) != h:
        return None
    return float(m_b.group(1))


# ------------------------------------------------------------------ oracle sample (CPU)
def oracle_sample(wl, heads, rows_per_group, seed=5, host=None):
    """Time the fp64 oracle on a bounded sample of the 720p step: `rows_per_group` random
    query rows per query group, `heads` heads; fresh states for the mask plus the merge
    with (seeded random) cached states and the importance.  Returns (seconds, flops,
    threads, description)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count()
    if host is not None:
        oracle_sample._cache = host
    t = oracle_sample._cache if hasattr(oracle_sample, "_cache") else W.make_qkv(wl)
    oracle_sample._cache = t
    off = W.part_offsets(wl.N, wl.P)
    fresh = W.reuse_mask(wl)
    gb = O.group_bounds(off, wl.G)
    rng = np.random.default_rng(seed)
    rows = np.sort(np.concatenate([rng.choice(np.arange(gb[g], gb[g + 1]), rows_per_group, replace=False)
                                   for g in range(wl.QG)]))
    R = len(rows)
    qg_of_row = np.searchsorted(gb, rows, side="right") - 1
    fresh_keys = sum(int(gb[kg + 1] - gb[kg]) for g in qg_of_row for kg in range(wl.KG) if fresh[g, kg])
    flops = 4.0 * wl.D * fresh_keys * heads
    inputs = []
    for h in range(heads):
        q, k, v = (W.to_f64(t[n][0:1, h:h + 1]) for n in ("q", "k", "v"))
        oc = rng.standard_normal((wl.P, 1, 1, R, wl.D))
        lc = rng.normal(5.0, 1.0, size=(wl.P, 1, 1, R))
        inputs.append((q, k, v, oc, lc))
    t0 = time.perf_counter()
    for q, k, v, oc, lc in inputs:
        of, lf, _ = O.partition_states(q, k, v, off, wl.G, fresh, wl.scale, rows=rows)
        o, lse, chosen = O.merge_with_reuse(of, lf, oc, lc, off, wl.G, fresh, rows=rows)
        O.importance(chosen, lse, off, wl.G, rows=rows)
    dt = time.perf_counter() - t0
    desc = (f"{heads} of {wl.H} heads x {R} query rows ({rows_per_group} random per query group): "
            "fresh states + merge + importance, fp64 NumPy")
    return dt, flops, threads, desc


def cpu_baseline_entry(wl, full_flops, host=None):
    dt, flops, threads, desc = oracle_sample(wl, heads=wl.H, rows_per_group=128, host=host)
    tflops = flops / dt / 1e12
    entry = {"value": tflops, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
             "sample": desc, "seconds": dt,
             "extrapolated_full_step_s": full_flops / (flops / dt)}
    try:                                   # the same oracle on one core, smaller sample
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt1, flops1, _, desc1 = oracle_sample(wl, heads=4, rows_per_group=32, seed=6)
        entry["one_core"] = {"value": flops1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                             "sample": desc1, "seconds": dt1}
    except ImportError:
        pass
    return entry


# ------------------------------------------------------------------ reference arm
def bench_workload(name):
    """The 720p workload, or the same recipe on 6 frames and 8 heads (profiling case: inputs
    still larger than L2, a few GB on the device)."""
    wl = W.workload(2)
    if name == "720p-small":
        wl = W.small_variant(wl, grid=(6, 45, 80), H=8)
    return wl


def run_reference(args, ws, rank):
    if rank != 0:
        return 0
    wl = bench_workload(args.workload)
    times, flops_l = [], []
    for i in range(args.warmup + args.steps):
        dt, flops, threads, desc = oracle_sample(wl, heads=8, rows_per_group=64, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops_l.append(flops)
    total = sum(times)
    value = sum(flops_l) / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl), "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ the other configurations
def config_extras(ctx, dev, stream, pk, reps=20):
    """Kernel times of the tiny fp32 workload and the image DiT workload with reuse (one
    attention launch for the fresh pairs, one merge with fused importance), each timed
    alone with L2 flushed before every repetition, and of the Ulysses-layout workload's
    attention alone (all pairs fresh, one launch)."""
    from sequence_partition_attn_b200.step import AttentionStep
    import sequence_partition_attn_b200 as pa
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    for i in (0, 1):
        wl = W.workload(i)
        off = W.part_offsets(wl.N, wl.P)
        fresh = W.reuse_mask(wl)
        host = W.make_qkv(wl)
        st = AttentionStep(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, fresh, dtype=wl.torch_dtype, device=dev)
        st.q.copy_(host["q"])
        st.k.copy_(host["k"])
        st.v.copy_(host["v"])
        if st.o_cached is not None:
            kc, vc = W.make_cached_kv(wl, host["k"], host["v"])
            st.fill_cache(kc.to(dev), vc.to(dev))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps + 3)]
        for e in ev:
            flush.zero_()
            e[0].record(stream)
            st.attention()
            e[1].record(stream)
            st.merge()
            e[2].record(stream)
        torch.cuda.synchronize()
        ctx.sync_status()
        a_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev[3:])
        m_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev[3:])
        entry = {"workload": f"{wl.name}: B{wl.B} H{wl.H} N{wl.N} D{wl.D} {wl.dtype}, P={wl.P}, "
                             f"{int(fresh.sum())} of {fresh.size} pairs fresh",
                 "attention_ms": a_ms, "attention_tflops": st.flops / (a_ms / 1e3) / 1e12,
                 "attention_flops": st.flops,
                 "merge_ms": m_ms, "merge_gbs": st.merge_bytes / (m_ms / 1e3) / 1e9,
                 "merge_bytes": st.merge_bytes, "l2": "flushed before every repetition"}
        if wl.dtype == "bf16":
            entry["attention_frac_of_burst"] = entry["attention_tflops"] / pk["bf16_tflops"]
            entry["merge_frac_of_hbm"] = entry["merge_gbs"] / pk["hbm_gbs"]
        out[f"config{i}"] = entry
        del st
    # Ulysses-layout workload: the attention of every pair in one launch on head-major inputs
    wl = W.workload(4)
    off = W.part_offsets(wl.N, wl.P)
    q, k, v = (torch.empty(1, wl.H, wl.N, wl.D, dtype=torch.bfloat16, device=dev).normal_()
               for _ in range(3))
    o = torch.empty(wl.P, 1, wl.H, wl.N, wl.D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.P, 1, wl.H, wl.N, dtype=torch.float32, device=dev)
    pa.pa_partition_attn(ctx, q, k, v, off, 1, None, o, lse)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    pa.pa_partition_attn(ctx, q, k, v, off, 1, None, o, lse)
    b.record(stream)
    torch.cuda.synchronize()
    ctx.sync_status()
    ms = a.elapsed_time(b)
    fl = 4.0 * wl.D * wl.H * float(wl.N) * wl.N
    out["config4"] = {"workload": f"{wl.name}: B1 H{wl.H} N{wl.N} D{wl.D} bf16, P={wl.P}, all fresh, "
                                  "head-major inputs (attention only)",
                      "attention_ms": ms, "attention_tflops": fl / (ms / 1e3) / 1e12,
                      "attention_frac_of_burst": fl / (ms / 1e3) / 1e12 / pk["bf16_tflops"]}
    del q, k, v, o, lse, flush
    out["config3"] = trajectory_extras(ctx, dev, stream, pk)
    return out


def trajectory_extras(ctx, dev, stream, pk):
    """The denoising trajectory (image-DiT shape, 10 steps, K and V drifting, anchors 0 and 5)
    under each reuse policy: the threshold as specified (0.05), a threshold that reuses
    (0.12) and the online prediction.  Per step, wall time on the host around the step
    (device work, the host's mask selection, and at anchors the copy of w to the host) with
    the stream synchronized on both sides; inputs of every step are generated and moved to
    the device before timing."""
    from sequence_partition_attn_b200.step import Trajectory
    wl = W.workload(3)
    off = W.part_offsets(wl.N, wl.P)
    host = W.make_qkv(wl)
    q = host["q"].to(dev)
    kv, k, v = [], host["k"], host["v"]
    for s_ in range(wl.steps):
        if s_ > 0:
            k, v = W.drift_kv(wl, k, v, s_)
        kv.append((k.to(dev), v.to(dev)))
    per_pair = 4.0 * wl.D * wl.B * wl.H * float(wl.N // wl.P) ** 2     # flops of one (query, KV) partition pair
    out = {"workload": f"{wl.name}: B{wl.B} H{wl.H} N{wl.N} D{wl.D} bf16, P={wl.P}, {wl.steps} steps, "
                       f"anchors {list(wl.anchors)}, drift {wl.drift}"}
    for name, thr, policy in (("threshold_0.05", wl.threshold, "threshold"), ("threshold_0.12", 0.12, "threshold"),
                              ("online_prediction", 1e-3, "predict")):
        tr = Trajectory(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, wl.anchors, thr, device=dev, policy=policy)
        times, fresh = [], []
        for s_ in range(wl.steps):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            mask = tr.step(s_, q, kv[s_][0], kv[s_][1], stream=stream)
            torch.cuda.synchronize()
            times.append((time.perf_counter() - t0) * 1e3)
            fresh.append(int(mask.sum()))
        ctx.sync_status()
        reuse_steps = [i for i in range(wl.steps) if i not in wl.anchors]
        out[name] = {"ms_per_step": times, "fresh_pairs_per_step": fresh, "pairs": int(wl.P * wl.P),
                     "mean_ms_anchor": statistics.mean(times[i] for i in wl.anchors),
                     "mean_ms_between_anchors": statistics.mean(times[i] for i in reuse_steps),
                     "attention_flops_per_step": [f * per_pair for f in fresh]}
        del tr
    del kv, q
    return out


# ------------------------------------------------------------------ our arm
def run_ours(args, ws, rank, local):
    import sequence_partition_attn_b200 as pa
    from sequence_partition_attn_b200.step import AttentionStep, StreamedSteps, relayout_overlapped
    pa.lib()
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    ctx = pa.Context(local)
    wl = bench_workload(args.workload)
    fresh = W.reuse_mask(wl)
    off = W.part_offsets(wl.N, wl.P)
    host = W.make_qkv(wl)
    kc, vc = W.make_cached_kv(wl, host["k"], host["v"])
    step = AttentionStep(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, fresh, device=dev)
    step.q.copy_(host["q"])
    step.k.copy_(host["k"])
    step.v.copy_(host["v"])
    kcd, vcd = kc.to(dev), vc.to(dev)
    step.fill_cache(kcd, vcd)
    del kcd, vcd, kc, vc
    ctx.sync_status()
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        step.run()
    ctx.sync_status()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(K):
        ev[i][0].record(stream)
        step.attention()
        ev[i][1].record(stream)
        step.merge()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ctx.sync_status()
    elapsed_ms = ev[0][0].elapsed_time(ev[-1][2])
    attn_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    merge_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    elapsed_ms = max_over_ranks(elapsed_ms, ws)
    ms_per_step = elapsed_ms / K
    value = replica_throughput(ws, step.flops, K, elapsed_ms) / 1e12
    pk, pk_kind = peaks()
    attn_tflops = step.flops / (attn_ms / 1e3) / 1e12
    merge_gbs = step.merge_bytes / (merge_ms / 1e3) / 1e9
    step_flops = step.flops
    traffic = traffic_per_launch()

    # ---- end to end through the public API with host buffers (pinned), every step
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (host[n].pin_memory() for n in ("q", "k", "v"))
        ho = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()
        hl = torch.empty(step.lse.shape, dtype=torch.float32).pin_memory()
        hw = torch.empty(step.w.shape, dtype=torch.float32).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
        d2h = sum(x.numel() * x.element_size() for x in (ho, hl, hw))
        def e2e_step():
            step.q.copy_(hq, non_blocking=True)
            step.k.copy_(hk, non_blocking=True)
            step.v.copy_(hv, non_blocking=True)
            step.run()
            ho.copy_(step.o, non_blocking=True)
            hl.copy_(step.lse, non_blocking=True)
            hw.copy_(step.w, non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        serial_ms = max_over_ranks(e0.elapsed_time(e1), ws)
        # the same steps with the copies of neighbouring steps overlapped (StreamedSteps)
        streamed = StreamedSteps(step)
        h_in = [(hq, hk, hv)] * K
        h_out = [(ho, hl, hw)] * K
        done = streamed.run(h_in[:2], h_out[:2], after=stream)
        stream.wait_event(done)
        torch.cuda.synchronize()
        barrier(ws)
        e0.record(stream)
        done = streamed.run(h_in, h_out, after=stream)
        stream.wait_event(done)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        ctx.sync_status()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws)
        e2e = {"value": replica_throughput(ws, step.flops, K, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
               "api": "StreamedSteps.run: host inputs and outputs of every step, copies of "
                      "neighbouring steps overlapped with compute",
               "serial_ms_per_step": serial_ms / K}
        del streamed
        del hq, hk, hv, ho, hl, hw
    # ---- dynamic group compose: the cache composed per KV group, merged without importance
    if not args.no_extras and step.o_cached is not None:
        B, H, N, D, G, KG = wl.B, wl.H, wl.N, wl.D, wl.G, wl.KG
        ocg = torch.empty(KG, B, H, N, D, dtype=torch.bfloat16, device=dev)
        lcg = torch.empty(KG, B, H, N, dtype=torch.float32, device=dev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pa.pa_compose_states(ctx, step.o_cached, step.lse_cached, G, ocg, lcg)
        c0.record(stream)
        pa.pa_compose_states(ctx, step.o_cached, step.lse_cached, G, ocg, lcg)
        c1.record(stream)
        for _ in range(3):
            pa.pa_merge_states(ctx, off, G, fresh, step.o_fresh, step.lse_fresh, ocg, lcg, step.o,
                               step.lse, cached_per_group=True)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        m0.record(stream)
        for _ in range(reps):
            pa.pa_merge_states(ctx, off, G, fresh, step.o_fresh, step.lse_fresh, ocg, lcg, step.o,
                               step.lse, cached_per_group=True)
        m1.record(stream)
        torch.cuda.synchronize()
        ctx.sync_status()
        gb = W.group_row_bounds(off, G)
        row_b = D * 2 + 4
        states = sum(int(gb[qg + 1] - gb[qg]) * sum(G if fresh[qg, kg] else 1 for kg in range(KG))
                     for qg in range(wl.QG))
        cm_bytes = float(B * H) * (states * row_b + N * row_b)
        cm_ms = m0.elapsed_time(m1) / reps
        cp_ms = c0.elapsed_time(c1)
        compose_bytes = float(B * H * N) * row_b * (wl.P + KG)
        composed_extra = {"merge_composed_cache": {"ms": cm_ms, "gbs": cm_bytes / (cm_ms / 1e3) / 1e9,
                                                   "bytes": cm_bytes},
                          "compose_cache": {"ms": cp_ms, "gbs": compose_bytes / (cp_ms / 1e3) / 1e9,
                                            "cache_bytes_before": float(B * H * N) * row_b * wl.P,
                                            "cache_bytes_after": float(B * H * N) * row_b * KG}}
        del ocg, lcg
        # ---- online prediction: drift of the own groups' states from the cached states
        own = np.eye(wl.QG, dtype=np.uint8)
        d2 = torch.empty(wl.QG, wl.P, dtype=torch.float32, device=dev)
        r2 = torch.empty_like(d2)
        for _ in range(3):
            pa.pa_state_drift(ctx, off, G, own, step.o_fresh, step.o_cached, d2, r2)
        m0.record(stream)
        for _ in range(reps):
            pa.pa_state_drift(ctx, off, G, own, step.o_fresh, step.o_cached, d2, r2)
        m1.record(stream)
        torch.cuda.synchronize()
        ctx.sync_status()
        dr_ms = m0.elapsed_time(m1) / reps
        own_rows = sum(int(gb[qg + 1] - gb[qg]) * min(G, wl.P - qg * G) for qg in range(wl.QG))
        dr_bytes = 2.0 * B * H * own_rows * D * 2
        composed_extra["state_drift"] = {"ms": dr_ms, "gbs": dr_bytes / (dr_ms / 1e3) / 1e9,
                                         "bytes": dr_bytes, "selection": "own groups"}
        del d2, r2
    else:
        composed_extra = {}
    del step
    torch.cuda.empty_cache()

    # ---- relayout HBM GB/s and the chunked relayout overlapped with attention (Ulysses layout)
    extras = {}
    if not args.no_extras:
        wl4 = W.workload(4)
        if args.workload == "720p-small":          # 2 of 16 chunks' worth: 4 chunks, 16 partitions
            wl4 = W.small_variant(wl4, grid=(2, 90, 160), H=wl4.H, P=16, chunks=4)
        N4, H4, D4 = wl4.N, wl4.H, wl4.D
        srcs = [torch.empty(N4, H4, D4, dtype=torch.bfloat16, device=dev).normal_() for _ in range(3)]
        dsts = [torch.empty(1, H4, N4, D4, dtype=torch.bfloat16, device=dev) for _ in range(3)]
        for _ in range(3):
            pa.pa_relayout_seq2head(ctx, srcs[0], dsts[0][0], n_chunks=1, chunk=-1)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        r0.record(stream)
        for i in range(reps):
            pa.pa_relayout_seq2head(ctx, srcs[i % 3], dsts[i % 3][0], n_chunks=1, chunk=-1)
        r1.record(stream)
        torch.cuda.synchronize()
        rel_ms = r0.elapsed_time(r1) / reps
        rel_bytes = 2.0 * N4 * H4 * D4 * 2
        extras["relayout"] = {"ms": rel_ms, "gbs": rel_bytes / (rel_ms / 1e3) / 1e9,
                              "bytes": rel_bytes, "shape": f"[{N4}][{H4}][{D4}] bf16 -> head-major"}
        off4 = W.part_offsets(N4, wl4.P)
        o4 = torch.empty(wl4.P, 1, H4, N4, D4, dtype=torch.bfloat16, device=dev)
        l4 = torch.empty(wl4.P, 1, H4, N4, dtype=torch.float32, device=dev)
        s_copy, s_attn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        def overlapped():
            s_copy.wait_stream(stream)
            s_attn.wait_stream(stream)
            relayout_overlapped(ctx, srcs, dsts, wl4.chunks, off4, 1, o4, l4, s_copy, s_attn)
            stream.wait_stream(s_attn)
            stream.wait_stream(s_copy)
        def sequential():
            for s, d in zip(srcs, dsts):
                pa.pa_relayout_seq2head(ctx, s, d[0], n_chunks=1, chunk=-1)
            pa.pa_partition_attn(ctx, dsts[0], dsts[1], dsts[2], off4, 1, None, o4, l4)
        res = {}
        for name, fn in (("overlapped_16_chunks", overlapped), ("sequential", sequential)):
            fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            res[name] = a.elapsed_time(b)
        ctx.sync_status()
        fl4 = 4.0 * D4 * H4 * float(N4) * N4
        extras["ulysses_layout_step"] = {
            "workload": f"B1 H{H4} N{N4} D{D4} bf16, P={wl4.P}, all fresh, relayout of Q,K,V in "
                        f"{wl4.chunks} chunks on a second stream",
            "overlapped_ms": res["overlapped_16_chunks"], "sequential_ms": res["sequential"],
            "overlapped_tflops": fl4 / (res["overlapped_16_chunks"] / 1e3) / 1e12}
        del srcs, dsts, o4, l4
        torch.cuda.empty_cache()

    if not args.no_extras:
        extras["configs"] = config_extras(ctx, dev, stream, pk)
        torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) + 3-D sinusoidal PE)",
        "config": {"workload": workload_desc(wl), "parallelism": f"replicas x{ws}",
                   "l2": "no flush: inputs larger than L2 (2.3 GB Q/K/V, 24.8 GB states per set)"},
        "step_ms": ms_per_step,
        "kernels": {"partition_attn": {"ms": attn_ms, "tflops": attn_tflops, "flops": step_flops},
                    "merge_importance": {"ms": merge_ms, "gbs": merge_gbs,
                                         "frac_of_hbm": merge_gbs / pk["hbm_gbs"]},
                    **composed_extra, **extras},
        # denominator: the burst GEMM figure (a cuBLAS bf16 GEMM timed alone, clocks free);
        # the ratio to the sustained figure (seconds of back-to-back GEMMs at the power cap)
        # and the SM clock seen during the timed region are reported beside it
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": attn_tflops / pk["bf16_tflops"],
                     "traffic": traffic,
                     "peak_kind": f"{pk_kind} burst bf16 (cuBLAS GEMM timed alone)",
                     "frac_of_sustained": attn_tflops / pk["bf16_tflops_sustained"],
                     "sm_mhz_median": clk.get("sm_mhz")},
        "gpu_launches": 3 * K,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = e2e
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_entry(wl, step_flops, host)
    ctx.close()
    if rank == 0:
        print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("720p", "720p-small"), default="720p")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)          # at least 3 untimed warm-up steps
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, ws, rank)
        return run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
