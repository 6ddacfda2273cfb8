#!/usr/bin/env python
"""CSA2 decode-step benchmark: prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload hier1m|full128k|verify|tiny]
                    [--impl ours|reference]

A step is one whole decode step of the workload: pack the step's new tokens into the FP4
cache, the Full layer's indexer scan (hierarchical: best 2048 blocks of 8, then its own
Top-512 inside them), every Reindex layer's rescoring, and the sparse attention of every
layer (Reuse layers with the inherited Top-K).  Inputs are seeded synthetic tensors
resident in HBM; the cache (1.5 GB for hier1m) is larger than L2 and L2 is also flushed
between timed steps.  The step is captured once in a CUDA graph and replayed.

N > 1 (torchrun): every rank runs the same workload on its own GPU (replicas, weak
scaling, no data-path collective); time is the max over ranks.  `--impl reference` times
the CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

METRIC = "CSA2 decode step µs/token and HBM GB/s at 128K/1M ctx; FP4 KV pack GB/s"
UNIT = "µs/token"

WORKLOAD_TEXT = {
    "hier1m": "hierarchical decoder at 1M context: B=4 x 1,048,576 FP4 entries, Full layer keeps 2048 "
              "blocks of 8, then 10 Reindex + 9 Reuse layers, H=64 x 512, HI=8 x 128, Top-512, W=128",
    "full128k": "Full-mode decode at 128K: B=32, entries U[64K,128K], flat scan + Top-512, Full + Reuse "
                "layer, H=64 x 512, HI=8 x 128, W=128",
    "verify": "multi-query verify: B=8 x 128K entries (2:1 of 256K tokens), Q=64 drafts, Full + Reuse layer",
    "tiny": "tiny decode: 1 sequence, 4096 entries, H=16, HI=4, Top-512, W=128",
    "hier256k": "hierarchical decoder at 256K context: B=4 x 262,144 FP4 entries, as hier1m (profiling size)",
    "prefill": "chunked prefill: 1 sequence of 256K tokens at 2:1 (128K entries), a chunk of 1024 new "
               "tokens as queries (own causal limits), Full + Reuse layer, H=64 x 512, HI=8 x 128, Top-512",
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="hier1m", choices=list(WORKLOAD_TEXT))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-seqs", type=int, default=1, help="sequences in the oracle's timed sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-pack-throughput", action="store_true",
                   help="skip the separate FP4 pack throughput measurement (2^20 tokens)")
    p.add_argument("--no-call-timing", action="store_true",
                   help="time the step without the per-call events (no breakdown or roofline)")
    p.add_argument("--no-configs", action="store_true",
                   help="measure only --workload (by default hier1m also brings full128k, verify and prefill)")
    p.add_argument("--cp-ranks", type=int, default=8,
                   help="at N=1, also time hier1m split over this many context-parallel ranks (0: skip)")
    return p.parse_args()


# ---- distributed plumbing ------------------------------------------------------------------
def dist_setup():
    """One process per GPU (torchrun sets RANK / LOCAL_RANK / WORLD_SIZE); NCCL on GPUs,
    gloo when the host has no GPU (the CPU tests of the multi-rank path)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        timeout = datetime.timedelta(seconds=300)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Max of a host float over all ranks (the timing reduction: the slowest rank counts)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---- clocks during the timed region ---------------------------------------------------------
def l2_note(cache_bytes, flush_bytes=256 << 20, l2_bytes=126 << 20):
    """How the timed steps see L2: the cache's size against L2, and the flush between steps."""
    rel = ">" if cache_bytes > l2_bytes else "<="
    size = f"{cache_bytes / 1e9:.2f} GB" if cache_bytes >= 1e9 else f"{cache_bytes / 1e6:.1f} MB"
    return f"cache {size} {rel} L2 ({l2_bytes >> 20} MB) and a {flush_bytes >> 20} MB L2 flush between timed steps"


def step_stats(ms_list):
    """Median, 10th and 90th percentile (nearest rank) of per-step device times in ms."""
    if not ms_list:
        return None
    s = sorted(ms_list)

    def pct(p):
        return s[min(len(s) - 1, max(0, math.ceil(p / 100.0 * len(s)) - 1))]

    return {"median": round(statistics.median(s), 4), "p10": round(pct(10), 4), "p90": round(pct(90), 4),
            "n": len(s)}


def cpu_model():
    """The host CPU's model name (first 'model name' of /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# Separate process (no share of this process's interpreter lock): read-only NVML queries of
# one GPU every 2 ms, one "time,sm_mhz,reasons_bitmask" line each, until terminated.
_NVML_POLL = """
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByPciBusId(sys.argv[1])
with open(sys.argv[2], "w", buffering=1) as f:
    f.write("max,%f\\n" % pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
    while True:
        f.write("%.6f,%d,%d\\n" % (time.time(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                   pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
        time.sleep(0.002)
"""


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this rank's GPU during the timed steps.
    A separate process polls NVML every 2 ms from construction on (so it is running before
    the timed region starts) and the samples time-stamped inside [start, stop] are kept; with
    no NVML, `nvidia-smi -lms 200` runs over the same window."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device):
        p = torch.cuda.get_device_properties(device)
        self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        self.proc = None
        self.path = None
        self.poller = None
        try:
            import pynvml  # noqa: F401  (the poller needs it)
            fd, self.poll_path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.poller = subprocess.Popen([sys.executable, "-c", _NVML_POLL, self.bus, self.poll_path],
                                           stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.poller = None

    def start(self):
        if self.poller is not None:
            # wait (at most 10 s) for the poller's first sample so the window is covered
            for _ in range(1000):
                with open(self.poll_path) as f:
                    if f.read().count("\n") >= 2:
                        break
                if self.poller.poll() is not None:
                    break
                time.sleep(0.01)
            self.t0 = time.time()
            return
        self.t0 = time.time()
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        t1 = time.time()
        if self.poller is not None:
            time.sleep(0.005)
            self.poller.terminate()
            try:
                self.poller.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.poller.kill()
            mx, rows = None, []
            with open(self.poll_path) as f:
                for line in f:
                    parts = line.strip().split(",")
                    if parts[0] == "max" and len(parts) == 2:
                        mx = float(parts[1])
                    elif len(parts) == 3:
                        rows.append((float(parts[0]), float(parts[1]), int(parts[2])))
            os.unlink(self.poll_path)
            inside = [r for r in rows if self.t0 <= r[0] <= t1]
            if not inside and rows:  # a window shorter than the poll interval: nearest samples
                inside = sorted(rows, key=lambda r: abs(r[0] - (self.t0 + t1) / 2))[:2]
            if not inside:
                return None
            reasons = sorted(n for n, bit in self.REASONS.items() if any(r[2] & bit for r in inside))
            return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": mx, "reasons": reasons,
                    "samples": len(inside), "source": "nvml every 2 ms, samples inside the timed steps"}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi every 200 ms"}


# ---- roofline bookkeeping -------------------------------------------------------------------
def load_peaks():
    """Roofline denominators.  Every call here is timed inside a step of well under a second,
    so tensor-bound calls take the burst GEMM figure (the sustained one is for seconds-long
    loops under the power cap)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_mhz": p.get("sm_max_mhz", 1965.0), "src": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "sm_mhz": 1965.0, "src": "fallback"}


def algorithmic(wl, name, count):
    """Algorithmic bytes and flops of `count` launches of call `name` in one step."""
    Kent, W, H = wl.K, wl.window, wl.H
    BQ = wl.B * wl.Q
    if name in ("index_full", "index_hier"):
        _, n_vis = query_positions(wl)
        # a query reads each visible 68 B key once; Q queries of a sequence share its keys
        nbytes = sum(int(n_vis[b].max()) for b in range(wl.B)) * 68
        flops = 2 * wl.HI * 128 * int(n_vis.sum())
        return count * nbytes, count * flops
    if name == "reindex":
        return count * BQ * wl.n_blocks * wl.block * 68, count * 2 * wl.HI * 128 * BQ * wl.n_blocks * wl.block
    if name == "attn":
        return count * BQ * (Kent * 288 + W * 512), count * BQ * 4 * H * (Kent + W) * 512
    if name == "pack":
        t = wl.B * wl.new_tokens
        return count * (t * 1280 + (t // wl.ratio) * 356), 0
    return 0, 0


def query_positions(wl):
    import synth
    return synth.query_positions(wl)


# the kernels behind each library call, and what bounds the call
CALL_KERNELS = {
    "index_hier": ("stream_scan_kernel<hier> + select_kernel", "hbm"),
    "index_full": ("stream_scan_kernel<flat> + select_kernel", "hbm"),
    "reindex": ("reindex_scan_kernel + select_kernel", "hbm"),
    "attn": ("attn_kernel", "tensor"),
    "pack": ("pack_kv_kernel", "hbm"),
}

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the call's
# dominant kernel, from an ncu capture of that kernel as it is now, per workload; a kernel
# that changes drops out of this table until it is captured again.  The attention launch
# of hier1m was captured on hier256k, whose attention launch is the same (4 queries, 512
# entries + 128 window tokens each, the same grid): its traffic does not depend on the
# context length.
NCU_DRAM_BYTES_PER_LAUNCH = {("hier1m", "attn"): 1656320}


def call_rooflines(wl, per_call, counts, steps, peaks):
    """Per library call of the step: its device time and its algorithmic HBM bandwidth as a
    fraction of the measured copy peak; attention also as algorithmic tensor flops against
    the burst bf16 peak (f16 has the same nominal rate)."""
    out = {}
    for name, ms in per_call.items():
        n = counts[name]
        step_ms = ms / steps
        avg_ms = step_ms / n
        nbytes, flops = algorithmic(wl, name, 1)
        gbs = nbytes / (avg_ms * 1e-3) / 1e9
        kernel, bound = CALL_KERNELS[name]
        d = {"kernel": kernel, "bound": bound, "launches": n, "ms_per_step": round(step_ms, 4),
             "avg_launch_ms": round(avg_ms, 4), "algorithmic_bytes": nbytes,
             "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm"], 4)}
        if flops and name != "pack":
            tf = flops / (avg_ms * 1e-3) / 1e12
            d.update({"algorithmic_flops": flops, "tflops": round(tf, 2)})
            if bound == "tensor":
                d["tensor_frac"] = round(tf / peaks["bf16"], 4)
        out[name] = d
    return out


def dominant_roofline(wl, calls, peaks):
    """The roofline object of the call with the largest share of the step."""
    dom = max(calls, key=lambda k: calls[k]["ms_per_step"])
    c = calls[dom]
    if c["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": c["hbm_gbs"], "peak": peaks["hbm"], "unit": "GB/s",
                "frac": c["hbm_frac"]}
    else:
        roof = {"bound": "tensor", "achieved": c["tflops"], "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": c["tensor_frac"]}
    roof["traffic"] = NCU_DRAM_BYTES_PER_LAUNCH.get((wl.name, dom))
    roof.update({"kernel": c["kernel"], "call": dom, "avg_launch_ms": c["avg_launch_ms"],
                 "algorithmic_bytes": c["algorithmic_bytes"], "algorithmic_flops": c.get("algorithmic_flops"),
                 "peak_src": peaks["src"] + (" (bf16 burst; f16 has the same nominal rate)"
                                             if c["bound"] == "tensor" else " (copy bandwidth)")})
    return roof


# arithmetic of the path: f16 x f16 -> fp32 Full / hierarchical indexer dots and attention
# (tcgen05 kind::f16), int8 x int8 -> int32 Reindex dots (kind::i8), fp32 epilogues; FP4/FP8
# storage
DTYPE = "f16+i8"


# ---- our implementation ---------------------------------------------------------------------
def measure(name, steps, warmup, world, dev, call_timing=True, e2e=True):
    """One workload's decode step: device time of a CUDA-graph replay (inputs resident, L2
    flushed between steps), the per-call breakdown from a second graph with timing events,
    and the end-to-end time through the public API with host buffers."""
    import synth
    from sparse_attention_fp4_pack_b200.decode import CallTimer, DecodeStep
    from sparse_attention_fp4_pack_b200.workload import build_state

    wl = synth.workload(name)
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device=dev), qd, device=dev)

    def new_step():
        return DecodeStep(B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                          schedule=sched, hier=wl.hier, max_n_vis=max(wl.lengths), n_blocks=wl.n_blocks,
                          block=wl.block, device=dev)

    step = new_step()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # 256 MB > 126 MB L2

    def one(graph_step):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph_step.replay()
        e1.record()
        flush.fill_(1)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1), (graph_step.timer.collect() if graph_step.timer else {})

    # Per-call breakdown from a separate graph that brackets every library call with timing
    # events (each event node adds about 2 us, so the headline step is timed without them).
    per_call, counts = {}, {}
    if call_timing:
        probe = new_step()
        probe.timer = CallTimer()
        probe.capture(x)
        for i in range(warmup + steps):
            _, calls = one(probe)
            if i >= warmup:
                for k, v in calls.items():
                    per_call[k] = per_call.get(k, 0.0) + v
        counts = probe.timer.counts()
        probe.check_status()
        del probe
    step.capture(x)

    clocks = ClockSampler(dev)  # its poller starts now and is running by the timed steps
    for _ in range(warmup):
        one(step)
    step.check_status()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    total_ms = 0.0
    step_ms = []
    for _ in range(steps):
        ms, _ = one(step)
        total_ms += ms
        step_ms.append(ms)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    step.check_status()
    t_max = max_over_ranks(total_ms, world)
    tokens = wl.B * wl.Q * world
    res = {"wl": wl, "sched": sched, "us_per_token": t_max * 1000.0 / (steps * tokens),
           "ms_per_step": t_max / steps, "stats": step_stats(step_ms), "clocks": clk,
           "launches": step.launches_per_step() * steps, "per_call": per_call, "counts": counts,
           "cache_bytes": x.kv_pool.numel() + x.ik_pool.numel()}

    if e2e:
        # the step as a user runs it with host data: DecodeStep.run_io captured in a graph,
        # which overlaps each layer's input copies and output read-back with the other
        # layers' work; pinned host inputs in, results out, every step
        h_in = {k: getattr(x, k).cpu().pin_memory() for k in ("new_kv", "new_ik", "q", "qi", "w", "swa")}
        h_out = {"out": torch.empty_like(step.out, device="cpu").pin_memory(),
                 "lse": torch.empty_like(step.lse, device="cpu").pin_memory(),
                 "topk": torch.empty_like(step.topk, device="cpu").pin_memory()}
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = sum(t.numel() * t.element_size() for t in h_out.values())
        step.capture_io(x, h_in, h_out)
        e2e_ms = 0.0
        for i in range(warmup + steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            step.replay_io()
            e1.record()
            torch.cuda.synchronize()
            if i >= warmup:
                e2e_ms += e0.elapsed_time(e1)
            flush.fill_(1)
        step.check_status()
        e2e_max = max_over_ranks(e2e_ms, world)
        res["e2e"] = {"value": round(e2e_max * 1000.0 / (steps * tokens), 3), "unit": UNIT,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del step, x, flush
    torch.cuda.empty_cache()
    return res


def measure_cp(name, ranks, steps, warmup, dev):
    """Context parallelism over `ranks` ranks, emulated on this one GPU.  Every rank's step runs
    once in lockstep (the ranks reading their shards in place from one shared pool) to record
    what each exchange delivers.  Then each rank's step runs on its own in a CUDA graph, the
    recorded buffers taking the place of the all-gathers, timed like the main step (L2 flushed
    between steps).  The slowest rank's time is the step's compute critical path on `ranks`
    GPUs; the all-gathers themselves (NCCL over NVLink) are not in it, so their count and
    sizes are reported beside it."""
    import synth
    from sparse_attention_fp4_pack_b200.cp import CPDecodeStep, ShardLayout, run_lockstep, run_replay
    from sparse_attention_fp4_pack_b200.workload import build_state

    wl = synth.workload(name)
    sched = synth.layer_schedule(wl)
    qd = synth.step_queries(wl)
    x = build_state(wl, lambda b: synth.seq_tokens(wl, b, device=dev), qd, device=dev)
    lengths = [int(n) for n in wl.lengths]
    cps = []
    for c in range(ranks):
        lay = ShardLayout.in_shared_pool(c, ranks, lengths, x.seq_base, dev, block=wl.block)
        cps.append(CPDecodeStep(lay, B=wl.B, Q=wl.Q, H=wl.H, HI=wl.HI, K=wl.K, window=wl.window, ratio=wl.ratio,
                                schedule=sched, hier=wl.hier, max_shard_len=int(lay.length.max()),
                                n_blocks=wl.n_blocks, block=wl.block, device=dev))
    rec = []
    run_lockstep(cps, [x] * ranks, record=rec)
    torch.cuda.synchronize()
    for s_ in cps:
        s_.check_status()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    per_rank = []
    for c, st in enumerate(cps):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            run_replay(st, x, rec)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_replay(st, x, rec)
        total = 0.0
        for i in range(warmup + steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            flush.fill_(1)
            torch.cuda.synchronize()
            if i >= warmup:
                total += e0.elapsed_time(e1)
        st.check_status()
        per_rank.append(total / steps)
        del g
    sizes = [int(r[0].numel() * r[0].element_size()) for r in rec]
    worst = max(per_rank)
    out = {"workload": f"{name} split over {ranks} ranks (contiguous shards of every sequence), emulated on one GPU",
           "ranks": ranks, "ms_per_step_per_rank": [round(v, 4) for v in per_rank],
           "ms_per_step_slowest_rank": round(worst, 4),
           "us_per_token_compute": round(worst * 1000.0 / (wl.B * wl.Q), 3), "unit": UNIT,
           "exchanges_per_step": len(rec), "exchange_bytes_per_rank_per_step": sum(sizes),
           "largest_exchange_bytes_per_rank": max(sizes),
           "note": "device time of one rank's kernels, its exchanges' gathered buffers replayed from a recorded "
                   "lockstep run; the all-gathers are not timed (one GPU)"}
    del cps, x, rec, flush
    torch.cuda.empty_cache()
    return out


def config_of(name, wl, sched, world, cache_bytes):
    return {"workload": f"{name}: {WORKLOAD_TEXT[name]}", "B": wl.B, "Q": wl.Q, "H": wl.H, "HI": wl.HI,
            "K": wl.K, "window": wl.window, "layers": len(sched), "entries_per_seq": max(wl.lengths),
            "parallelism": f"replicas x{world}", "l2": l2_note(cache_bytes), "graph": "CUDA graph replay"}


def run_ours(args, world, rank, local):
    from sparse_attention_fp4_pack_b200 import csa2

    csa2.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    r = measure(args.workload, args.steps, args.warmup, world, dev, call_timing=not args.no_call_timing)
    wl = r["wl"]
    calls = call_rooflines(wl, r["per_call"], r["counts"], args.steps, peaks) if r["per_call"] else {}
    line = {
        "metric": METRIC, "value": round(r["us_per_token"], 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 4),
        "ms_per_step_rank0": r["stats"],
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic (seeded)",
        "config": config_of(args.workload, wl, r["sched"], world, r["cache_bytes"]),
        "e2e": r["e2e"],
        "gpu_launches": r["launches"],
        "roofline": dominant_roofline(wl, calls, peaks) if calls else None,
        "calls": calls,
        "clocks": r["clocks"],
        "peaks": peaks,
    }
    # the metric's other decode configurations, each measured the same way
    configs = {}
    if not args.no_configs and args.workload == "hier1m":
        for name in ("full128k", "verify", "prefill"):
            c = measure(name, args.steps, args.warmup, world, dev, call_timing=not args.no_call_timing)
            cc = call_rooflines(c["wl"], c["per_call"], c["counts"], args.steps, peaks) if c["per_call"] else {}
            configs[name] = {"value": round(c["us_per_token"], 3), "unit": UNIT,
                             "ms_per_step": round(c["ms_per_step"], 4), "ms_per_step_rank0": c["stats"],
                             "config": config_of(name, c["wl"], c["sched"], world, c["cache_bytes"]),
                             "e2e": c["e2e"], "gpu_launches": c["launches"], "calls": cc,
                             "roofline": dominant_roofline(c["wl"], cc, peaks) if cc else None,
                             "clocks": c["clocks"]}
    if configs:
        line["configs"] = configs
    if not args.no_configs and args.workload == "hier1m" and args.cp_ranks > 1 and world == 1:
        line["context_parallel"] = measure_cp(args.workload, args.cp_ranks, args.steps, args.warmup, dev)
    return line, wl


# ---- the oracle, timed on the host cores ------------------------------------------------------
def oracle_sample_state(wl, nseq, device, nq=None):
    """The oracle's own pool for the first `nseq` sequences (packed from the same seeded
    tokens) plus the step inputs of those sequences (of their first `nq` queries only,
    when given: the new tokens are still all packed)."""
    import oracle
    import synth
    lengths = [int(n) for n in wl.lengths[:nseq]]
    bases = np.cumsum([0] + lengths[:-1]).astype(np.int64)
    kv_pools, ik_pools, new_kv, new_ik = [], [], [], []
    for b in range(nseq):
        kv, ik = synth.seq_tokens(wl, b, device=device)
        old = kv.shape[0] - wl.new_tokens
        kvb = kv.cpu().view(torch.int16).numpy().astype(np.uint16)
        ikb = ik.cpu().view(torch.int16).numpy().astype(np.uint16)
        del kv, ik
        a, c = oracle.pack_kv(kvb[:old], ikb[:old], wl.ratio)
        kv_pools.append(np.concatenate([a, np.zeros((wl.new_tokens // wl.ratio, 288), np.uint8)]))
        ik_pools.append(np.concatenate([c, np.zeros((wl.new_tokens // wl.ratio, 68), np.uint8)]))
        new_kv.append(kvb[old:])
        new_ik.append(ikb[old:])
    qd = synth.step_queries(wl)
    sl, ql = slice(0, nseq), slice(0, nq if nq else wl.Q)
    return dict(kv_pool=np.concatenate(kv_pools), ik_pool=np.concatenate(ik_pools), base=bases,
                lengths=lengths, new_kv=new_kv, new_ik=new_ik,
                q=qd["q"][:, sl, ql].numpy(), qi=qd["qi"][:, sl, ql].numpy(), w=qd["w"][:, sl, ql].numpy(),
                swa=qd["swa"][:, sl].numpy(), swa_start=qd["swa_start"][sl].numpy(),
                q_pos=qd["q_pos"][sl, ql].numpy(), n_vis=qd["n_vis"][sl, ql].numpy())


def oracle_step(wl, st):
    """One decode step of the sample, entirely in the oracle."""
    import oracle
    import synth
    sched = synth.layer_schedule(wl)
    sm = 1.0 / math.sqrt(512)
    for b in range(len(st["lengths"])):  # pack the step's new tokens into their slots
        a, c = oracle.pack_kv(st["new_kv"][b], st["new_ik"][b], wl.ratio)
        e0 = st["base"][b] + st["lengths"][b] - a.shape[0]
        st["kv_pool"][e0:e0 + a.shape[0]] = a
        st["ik_pool"][e0:e0 + a.shape[0]] = c
    cur = blocks = None
    for l, mode in enumerate(sched):
        if mode == "full":
            if wl.hier:
                blocks, _ = oracle.index_hier(st["qi"][l], st["w"][l], st["ik_pool"], st["base"], st["n_vis"],
                                              wl.n_blocks, wl.block)
                cur, _ = oracle.reindex(st["qi"][l], st["w"][l], st["ik_pool"], st["base"], st["n_vis"], blocks,
                                        wl.K, block=wl.block)
            else:
                cur, _ = oracle.index_full(st["qi"][l], st["w"][l], st["ik_pool"], st["base"], st["n_vis"], wl.K)
        elif mode == "reindex":
            cur, _ = oracle.reindex(st["qi"][l], st["w"][l], st["ik_pool"], st["base"], st["n_vis"], blocks, wl.K,
                                    block=wl.block)
        oracle.sparse_attn(st["q"][l], st["kv_pool"], st["base"], cur, st["swa"][l], st["swa_start"], st["q_pos"],
                           sm, window=wl.window)


def time_pack(steps, warmup, device):
    """FP4 pack throughput on 2^20 new tokens (512-channel main KV + 128-dim indexer key,
    bf16, resident in HBM) at 1:1 and 2:1: (bytes read + bytes written) / device time, L2
    flushed between launches.  Inputs follow the pack workload's value recipe.  The same
    for the producer that normalises and rotates raw tokens before packing them."""
    import synth
    from sparse_attention_fp4_pack_b200 import csa2
    T = 1 << 20
    kv, ik = synth.kv_tokens(1, T, device=device, recipe="rmsnorm")
    kvp = torch.empty(T, 288, dtype=torch.uint8, device=device)
    ikp = torch.empty(T, 68, dtype=torch.uint8, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    res = {}
    for ratio in (1, 2):
        ms = 0.0
        for i in range(warmup + steps):
            flush.fill_(i)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            csa2.csa2_pack_kv(kv, ik, ratio, kvp, ikp)
            e1.record()
            torch.cuda.synchronize()
            if i >= warmup:
                ms += e0.elapsed_time(e1)
        ms /= steps
        nbytes = T * 1280 + (T // ratio) * 356
        res[f"{ratio}:1"] = {"GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1), "us": round(ms * 1e3, 1),
                             "bytes": nbytes}
    # the producer (RMSNorm + rotation + pack) on raw tokens at positions 0..T-1: it also
    # reads the token's position and its cos/sin table rows (8 + 2048 B per token)
    del kv, ik
    raw, rik = synth.raw_kv_tokens(1, T, device=device)
    cos, sin = synth.rope_tables(T, device=device)
    pos = torch.arange(T, dtype=torch.int64, device=device)
    for ratio in (1, 2):
        ms = 0.0
        for i in range(warmup + steps):
            flush.fill_(i)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            csa2.csa2_pack_kv_normed(raw, rik, ratio, pos, cos, sin, kvp, ikp)
            e1.record()
            torch.cuda.synchronize()
            if i >= warmup:
                ms += e0.elapsed_time(e1)
        ms /= steps
        nbytes = T * (1280 + 8 + 2048) + (T // ratio) * 356
        res[f"normed {ratio}:1"] = {"GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1), "us": round(ms * 1e3, 1),
                                    "bytes": nbytes}
    del raw, rik, cos, sin, pos, kvp, ikp, flush
    torch.cuda.empty_cache()
    return res


def time_oracle(wl, nseq, steps, warmup, device, nq=None):
    import oracle
    st = oracle_sample_state(wl, nseq, device, nq)
    for _ in range(warmup):
        oracle_step(wl, st)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_step(wl, st)
    dt = time.perf_counter() - t0
    nq = nq if nq else wl.Q
    tokens = nseq * nq
    # the oracle spreads queries over its threads, or the work inside a query when there
    # are fewer queries than threads, so every thread takes part either way
    cores = oracle.num_threads()
    sample = (f"{nseq} of {wl.B} sequences of the {wl.name} workload (full context, all "
              f"{wl.n_layers} layers, {nq} of {wl.Q} quer{'y' if wl.Q == 1 else 'ies'} each), {steps} step(s)")
    return dt * 1e6 / (steps * tokens), cores, sample


def cpu_baseline(wl, nseq, nq=None):
    v, cores, sample = time_oracle(wl, nseq, 1, 0, "cuda", nq)
    return {"value": round(v, 1), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model()}


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        if rank == 0:
            import synth
            wl = synth.workload(args.workload)
            dev = "cuda" if torch.cuda.is_available() else "cpu"
            v, cores, sample = time_oracle(wl, args.cpu_seqs, args.steps, args.warmup, dev)
            line = {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "higher_is_better": False, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
                    "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]}"},
                    "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
                                     "sample": sample, "cpu_model": cpu_model()},
                    "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            print(json.dumps(line, ensure_ascii=False), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    line, wl = run_ours(args, world, rank, local)
    if not args.no_pack_throughput:
        pk = time_pack(5, 3, "cuda")
        peak = load_peaks()["hbm"]
        line["pack_throughput"] = {"tokens": 1 << 20, "unit": "GB/s", "peak": peak,
                                   **{k: dict(v, frac=round(v["GB/s"] / peak, 3)) for k, v in pk.items()}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import synth
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seqs)
        for name, c in line.get("configs", {}).items():
            # the prefill chunk's oracle sample: 64 of its 1024 queries (about 10 s of CPU)
            c["cpu_baseline"] = cpu_baseline(synth.workload(name), 1, 64 if name == "prefill" else None)
    if rank == 0:
        print(json.dumps(line, ensure_ascii=False), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
