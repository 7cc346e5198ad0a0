"""Benchmark: hybrid prefill + decode attention, microseconds per call.

One "step" is one ``pod_attn_hybrid`` call (FUSED) on a synthetic hybrid batch
whose inputs are already resident in HBM; L2 is flushed (a write larger than
L2) before every timed call and each call is timed with CUDA events on the
launching stream. The headline workload is the long-context mix (64 q / 8 kv
heads, d 128, a 1024-token chunk after 16384 cached tokens plus 16 decodes of
16K-32K keys). The same run times the library's SERIAL and TWO_STREAM modes
and the prefill-only / decode-only launches, reports the fused max(FLOP, HBM)
roofline fraction with the measured peaks, times FUSED / SERIAL / TWO_STREAM
on the other full-size configurations, times one full fp64 oracle call on the
host cores, samples the clocks during the timed region, and measures the same
call end to end through the C ABI with host buffers.

Launch: ``python bench.py --gpus N --steps K --warmup W`` (N > 1 under
torch.distributed.run: N independent replicas, one per GPU, max over ranks).
``--impl reference`` times the fp64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hybrid_prefill_decode_pod_b200 import workloads as W  # noqa: E402

METRIC = "hybrid attention µs/call & % of max(FLOP,HBM) roofline vs serial P+D, 1 B200"
UNIT = "us/call"
DEFAULT_WORKLOAD = "long_context"
# the other full-size configurations, timed in the same run as extra keys
EXTRA_WORKLOADS = ("tiny", "llama3_8b", "decode_heavy", "paged",
                   # shape variants: multi-head, group of 8, head_dim 64, many small chunks
                   "llama2_7b_mha", "yi6b_g8", "d64_mix", "many_chunks")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "hybrid_prefill_decode_pod_b200", "csrc")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes per fused launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except Exception:
        return None
    e = d.get(workload)
    if not e or e.get("kernel_sha") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        time.sleep(0.25)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, lo=0, hi=None):
        """Median SM clock (and power) over samples lo..hi, with every throttle reason seen."""
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[lo:hi]:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[2]))
            except ValueError:
                pass
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
               "reasons": sorted(reasons)}
        if pw:
            out["power_w"] = statistics.median(pw)
        return out


def dist_setup(n_gpus):
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_max(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- CPU oracle leg
def oracle_full_call(batch):
    """One full, unsampled fp64 oracle call on every host core (wall clock).
    Returns (us, threads)."""
    import oracle
    n_threads = oracle.max_threads()
    t0 = time.perf_counter()
    oracle.hybrid(batch)
    return (time.perf_counter() - t0) * 1e6, n_threads


def run_reference(args, rank, world):
    """The base contract's reference arm: the fp64 oracle (rank 0 only), one
    full, unsampled call of the workload per step. Steps stop once the time
    budget is spent (at least one runs), and the line reports the steps that
    ran; there is no warm-up, the oracle keeps no state between calls."""
    if rank != 0:
        return 0
    batch = W.make_batch(W.get_config(args.workload))
    vals, threads = [], 0
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        us, threads = oracle_full_call(batch)
        vals.append(us)
        if time.perf_counter() - t0 >= args.ref_budget_seconds:
            break
    v = statistics.median(vals)
    desc = ("each step: one full, unsampled call of this workload (every (row, head) item), "
            "wall clock, fp64, %d OpenMP threads; %d of the %d requested steps ran within the "
            "%.0f s budget, median reported; no warm-up (the oracle keeps no state)"
            % (threads, len(vals), args.steps, args.ref_budget_seconds))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(vals), "warmup": 0, "ms_per_step": v / 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": W.CONFIG_DESCRIPTIONS[args.workload]},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU leg
def time_calls(fn, n, flush_buf, stream):
    """Time n calls of fn() with CUDA events on `stream`; L2 flushed before each."""
    times = []
    for _ in range(n):
        flush_buf.add_(1)   # write > L2 between calls
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        times.append((s, e))
    torch.cuda.synchronize()
    return [s.elapsed_time(e) * 1000.0 for s, e in times]  # us


def sustained(fn, seconds, stream, local):
    """Back-to-back calls (no L2 flush) for `seconds` after one second of the same
    load, so the board's power limit has settled: mean us per call and the SM
    clock and power sampled over the timed part."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 1.0:  # settle: same load, not timed
            for _ in range(10):
                fn()
            torch.cuda.synchronize()
        lo = len(clk.lines)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        n = 0
        s.record(stream)
        t1 = time.perf_counter()
        while time.perf_counter() - t1 < seconds:
            for _ in range(20):
                fn()
            n += 20
            torch.cuda.synchronize()
        e.record(stream)
        torch.cuda.synchronize()
        hi = len(clk.lines)
    out = {"us_per_call": s.elapsed_time(e) * 1000.0 / n, "calls": n}
    out.update(clk.summary(lo, hi))
    return out


def mean(xs):
    return sum(xs) / len(xs)


def roofline_bound(batch, peaks):
    """Algorithmic FLOPs and bytes of one call and the fused bound
    T* = max(F / tensor peak, B / HBM peak) in us."""
    cfg = batch.cfg
    f_p, f_d, b_p, b_d = W.algorithmic_work(cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim,
                                            batch.priors, batch.chunks, batch.ctx,
                                            paged=cfg.paged)
    F, B = f_p + f_d, b_p + b_d
    t_tc = F / (peaks["bf16_tflops"] * 1e12) * 1e6
    t_bw = B / (peaks["hbm_gbs"] * 1e9) * 1e6
    return F, B, max(t_tc, t_bw), ("tensor" if t_tc > t_bw else "hbm"), f_p


def time_modes(pa, pod, pre, dec, stream, flush, steps, warmup):
    """Mean us of FUSED, SERIAL and TWO_STREAM calls (warm-up first)."""
    out = {}
    for name, mode in (("fused", pa.MODE_FUSED), ("serial", pa.MODE_SERIAL),
                       ("two_stream", pa.MODE_TWO_STREAM)):
        fn = (lambda m: (lambda: pod.hybrid(pre, dec, m, stream)))(mode)
        for _ in range(warmup):
            fn()
        out[name] = mean(time_calls(fn, steps, flush, stream))
    return out


def run_extra_workload(pa, name, dev, local, stream, flush, peaks, steps):
    """FUSED / SERIAL / TWO_STREAM on another full-size configuration."""
    batch = W.make_batch(W.get_config(name))
    pod = pa.context_for(batch, device=local)
    db = pa.DeviceBatch(batch, device=dev)
    pre, dec = db.args(pod)
    t = time_modes(pa, pod, pre, dec, stream, flush, steps, 3)
    st = pod.status(stream)
    plan = pod.last_plan()
    pod.close()
    if st != pa.POD_OK:
        raise RuntimeError("device status %d on %s" % (st, name))
    F, B, t_star, bound, _ = roofline_bound(batch, peaks)
    del db
    torch.cuda.empty_cache()
    return {"fused_us": t["fused"], "serial_us": t["serial"], "two_stream_us": t["two_stream"],
            "t_star_us": t_star, "bound": bound, "fused_roofline_frac": t_star / t["fused"],
            "speedup_vs_serial": t["serial"] / t["fused"],
            "speedup_vs_two_stream": t["two_stream"] / t["fused"], "steps": steps,
            "decode_split_len": plan["decode_split_len"], "prefill_units": plan["prefill_units"]}


def run_gpu(args, rank, world, local):
    from hybrid_prefill_decode_pod_b200 import pod_attn as pa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    cfg = W.get_config(args.workload)
    batch = W.make_batch(cfg)
    pod = pa.context_for(batch, device=local, flags=pa.FLAG_STATS if args.stats else 0)
    db = pa.DeviceBatch(batch, device=dev)
    pre, dec = db.args(pod)
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    F, B, t_star, bound, f_prefill = roofline_bound(batch, peaks)

    def call(mode):
        return lambda: pod.hybrid(pre, dec, mode, stream)

    if args.only:
        # one mode alone (for profiler captures): warm-up, then `steps` calls
        fn = {"fused": call(pa.MODE_FUSED), "serial": call(pa.MODE_SERIAL),
              "two_stream": call(pa.MODE_TWO_STREAM),
              "prefill_only": lambda: pod.prefill_only(pre, stream),
              "decode_only": lambda: pod.decode_only(dec, stream)}[args.only]
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = time_calls(fn, args.steps, flush, stream)
        st = pod.status(stream)
        pod.close()
        if rank == 0:
            print(json.dumps({"only": args.only, "workload": args.workload,
                              "us_mean": mean(ts), "us_median": statistics.median(ts),
                              "status": st}), flush=True)
        return 0 if st == pa.POD_OK else 1

    # warm-up (>= 3)
    for m in (pa.MODE_FUSED, pa.MODE_SERIAL, pa.MODE_TWO_STREAM):
        for _ in range(max(3, args.warmup)):
            call(m)()
    torch.cuda.synchronize()
    st = pod.status(stream)
    if st != pa.POD_OK:
        raise RuntimeError("device status %d after warm-up" % st)

    # ---- the timed region: K fused calls
    dist_barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        fused = time_calls(call(pa.MODE_FUSED), args.steps, flush, stream)
        wall = time.perf_counter() - wall0
    torch.cuda.synchronize()
    dist_barrier(world)
    clocks = clk.summary()
    fused_mean = mean(fused)
    value = dist_max(fused_mean, world)

    # ---- the library's own baselines and the standalone phases (same run)
    extra_steps = max(5, args.steps // 2)
    serial = time_calls(call(pa.MODE_SERIAL), extra_steps, flush, stream)
    two = time_calls(call(pa.MODE_TWO_STREAM), extra_steps, flush, stream)
    p_only = time_calls(lambda: pod.prefill_only(pre, stream), extra_steps, flush, stream) if pre else [0.0]
    d_only = time_calls(lambda: pod.decode_only(dec, stream), extra_steps, flush, stream) if dec else [0.0]
    # ---- sustained: each mode back to back under the board's power limit
    sus = None
    if world == 1 and args.sustained_seconds > 0:
        sus = {"note": "calls back to back without L2 flush, after 1 s of the same load; "
                       "clock and power are nvidia-smi medians over the timed part"}
        modes = [("fused", call(pa.MODE_FUSED)), ("serial", call(pa.MODE_SERIAL)),
                 ("two_stream", call(pa.MODE_TWO_STREAM))]
        if pre:
            modes.append(("prefill_only", lambda: pod.prefill_only(pre, stream)))
        if dec:
            modes.append(("decode_only", lambda: pod.decode_only(dec, stream)))
        for name, fn in modes:
            sus[name] = sustained(fn, args.sustained_seconds, stream, local)
        # a step timed inside a long loop takes the sustained tensor peak
        sus_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        t_sus = max(F / (sus_peak * 1e12), B / (peaks["hbm_gbs"] * 1e9)) * 1e6
        sus["fused"]["roofline_frac_sustained_peak"] = t_sus / sus["fused"]["us_per_call"]
        sus["sustained_tensor_peak_tflops"] = sus_peak
    pod.hybrid(pre, dec, pa.MODE_FUSED, stream)
    plan = pod.last_plan()
    stats = pod.stats(stream) if args.stats else None
    st = pod.status(stream)
    if st != pa.POD_OK:
        raise RuntimeError("device status %d after timing" % st)

    # ---- end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(pa, pod, batch, db, dev, stream, min(args.steps, args.e2e_steps), flush)
    pod.close()
    del db
    torch.cuda.empty_cache()

    # ---- the other full-size configurations (single GPU only)
    extras = {}
    if world == 1 and not args.no_extras:
        for name in EXTRA_WORKLOADS:
            if name != args.workload:
                extras[name] = run_extra_workload(pa, name, dev, local, stream, flush, peaks,
                                                  args.extra_steps)

    # ---- CPU oracle baseline: one full call (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        us, cores = oracle_full_call(batch)
        cpu = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": "one full, unsampled call of this workload (every (row, head) item), "
                         "wall clock, fp64, %d OpenMP threads" % cores}

    achieved_tflops = F / (value * 1e-6) / 1e12
    achieved_gbs = B / (value * 1e-6) / 1e9
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved_tflops / peaks["bf16_tflops"]}
    roof["peak_kind"] = ("of measured" if peak_kind == "measured" else "of fallback") + " (burst)"
    roof["kernel"] = "pod_fused_kernel"
    roof["traffic"] = committed_traffic(args.workload)
    roof["algorithmic_bytes"] = B
    roof["algorithmic_flops"] = F
    roof["statistic"] = "mean of the timed calls (the same as value)"

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value / 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": W.CONFIG_DESCRIPTIONS[args.workload],
                   "l2": "flushed before every timed call (write of %d MB)" % (flush.numel() * 4 >> 20),
                   "mode": "fused", "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roof,
        "fused_roofline_frac": t_star / value,
        "t_star_us": t_star,
        "fused_us": {"mean": fused_mean, "median": statistics.median(fused),
                     "p10": float(np.percentile(fused, 10)), "p90": float(np.percentile(fused, 90))},
        "serial_us": mean(serial), "two_stream_us": mean(two),
        "prefill_only_us": mean(p_only), "decode_only_us": mean(d_only),
        "prefill_only_tflops": f_prefill / (mean(p_only) * 1e-6) / 1e12 if pre else None,
        "speedup_vs_serial": mean(serial) / fused_mean,
        "speedup_vs_two_stream": mean(two) / fused_mean,
        "tflops": achieved_tflops, "gbs": achieved_gbs,
        "plan": plan,
        "other_workloads": extras,
        "clocks": clocks,
        "sustained": sus,
        "gpu_launches": args.steps,
        "wall_s_timed_region": wall,
        "cpu_baseline": cpu,
        "e2e": e2e,
    }
    if stats:
        line["virtual_cta_mix"] = stats
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# Variants of the chunked-prompt study (the POD-Attention summary, §4.2.3 and
# §5.4.3 / Table 8: limiting the prefill's KV splits to two waves; §4.2.2 /
# §5.4.1: the prefill tile's size). Each is a set of planner levers read when
# a context is created.
SWEEP_VARIANTS = {
    "pair_model": {"POD_ATTN_PREFILL_TILE": "pair"},         # CTA-pair tile, split model
    "pair_nosplit": {"POD_ATTN_PREFILL_TILE": "pair", "POD_ATTN_PREFILL_SPLIT": "1"},
    "pair_uncapped8": {"POD_ATTN_PREFILL_TILE": "pair",      # 8 splits, two-wave cap off
                       "POD_ATTN_PREFILL_SPLIT": "-8"},
    "1sm_model": {"POD_ATTN_PREFILL_TILE": "1sm"},           # one-SM pair tile, split model
    "1sm_uncapped8": {"POD_ATTN_PREFILL_TILE": "1sm", "POD_ATTN_PREFILL_SPLIT": "-8"},
}
SWEEP_POLICIES = {  # the fused kernel's role policy (§4.1, §5.4.2 / Figure 14)
    "prefill_first": {"POD_ATTN_POLICY": "prefill_first"},
    "front": {"POD_ATTN_POLICY": "front"},
    "even": {"POD_ATTN_POLICY": "even"},
    "proportional": {"POD_ATTN_POLICY": "proportional"},
    "balanced": {"POD_ATTN_POLICY": "balanced"},
    "decode_first": {"POD_ATTN_POLICY": "decode_first"},
    "proportional_global_ticket": {"POD_ATTN_POLICY": "proportional", "POD_ATTN_SMID_AWARE": "0"},
}


def run_sweep(args, rank, world, local):
    """One JSON line per (workload, variant): FUSED, SERIAL and TWO_STREAM
    mean us (L2 flushed before every call, CUDA events), the plan, and the
    fused roofline fraction."""
    from hybrid_prefill_decode_pod_b200 import pod_attn as pa
    if rank != 0:
        return 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, _ = load_peaks()
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    if args.sweep == "chunked16k":
        points = [int(x) for x in args.sweep_points.split(",")] if args.sweep_points else \
            [0, 4, 8, 12, 16, 20, 24, 28, 29, 30, 31]
        workloads = ["chunked16k_%d" % i for i in points]
        variants = SWEEP_VARIANTS
    else:  # policies on the full-size configurations, with either prefill tile
        workloads = args.sweep_points.split(",") if args.sweep_points else \
            ["llama3_8b", "decode_heavy", "long_context", "paged"]
        variants = {}
        for tile, tenv in (("1sm", {"POD_ATTN_PREFILL_TILE": "1sm"}),
                           ("pair", {"POD_ATTN_PREFILL_TILE": "pair"})):
            for pname, penv in SWEEP_POLICIES.items():
                variants["%s_%s" % (tile, pname)] = dict(tenv, **penv)
    for name in workloads:
        batch = W.make_batch(W.get_config(name))
        db = pa.DeviceBatch(batch, device=dev)
        F, B, t_star, bound, _ = roofline_bound(batch, peaks)
        for vname, env in variants.items():
            old = {k: os.environ.get(k) for k in env}
            os.environ.update(env)
            try:
                pod = pa.context_for(batch, device=local)
            finally:
                for k, v in old.items():
                    if v is None:
                        os.environ.pop(k, None)
                    else:
                        os.environ[k] = v
            pre, dec = db.args(pod)
            t = time_modes(pa, pod, pre, dec, stream, flush, args.steps, max(3, args.warmup))
            pod.hybrid(pre, dec, pa.MODE_FUSED, stream)
            plan = pod.last_plan()
            st = pod.status(stream)
            pod.close()
            line = {"sweep": args.sweep, "workload": name, "variant": vname, "env": env,
                    "fused_us": t["fused"], "serial_us": t["serial"],
                    "two_stream_us": t["two_stream"],
                    "speedup_vs_serial": t["serial"] / t["fused"],
                    "speedup_vs_two_stream": t["two_stream"] / t["fused"],
                    "t_star_us": t_star, "bound": bound,
                    "fused_roofline_frac": t_star / t["fused"], "plan": plan, "status": st,
                    "steps": args.steps}
            print(json.dumps(line), flush=True)
            if st != pa.POD_OK:
                return 1
        del db
        torch.cuda.empty_cache()
    return 0


def run_e2e(pa, pod, batch, db, dev, stream, steps, flush):
    """Same metric through the C ABI with inputs in pinned host memory: every
    step copies Q and all K/V (or the pool and block tables) host -> device,
    runs the fused call, and copies O and LSE back."""
    host_in = [batch.q_prefill, batch.q_decode]
    dev_in = [db.q_p, db.q_d]
    if db.paged:
        host_in += [batch.k_pool, batch.v_pool, batch.block_table_prefill, batch.block_table_decode]
        dev_in += [db.k_pool, db.v_pool, db.bt_p, db.bt_d]
    else:
        host_in += list(batch.k_prefill) + list(batch.v_prefill) + list(batch.k_decode) + list(batch.v_decode)
        dev_in += list(db.k_p) + list(db.v_p) + list(db.k_d) + list(db.v_d)
    pinned = [t.pin_memory() for t in host_in]
    outs_dev = [db.o_p, db.lse_p, db.o_d, db.lse_d]
    outs_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs_dev]
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    d2h = sum(t.numel() * t.element_size() for t in outs_host)
    pre, dec = db.args(pod)
    times = []
    for _ in range(steps):
        flush.add_(1)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for dst, src in zip(dev_in, pinned):
            dst.copy_(src, non_blocking=True)
        pod.hybrid(pre, dec, pa.MODE_FUSED, stream)
        for dst, src in zip(outs_host, outs_dev):
            dst.copy_(src, non_blocking=True)
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e) * 1000.0)
    return {"value": mean(times), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "inputs (Q and every K/V byte the call reads) copied from pinned host memory each step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.CONFIGS) + sorted(W.PROBE_CONFIGS))
    ap.add_argument("--ref-budget-seconds", type=float, default=120.0,
                    help="reference arm: stop taking full oracle calls once this much time is spent")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other full-size configurations")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--sustained-seconds", type=float, default=2.0,
                    help="per mode, back-to-back timing under the power limit (0: skip)")
    ap.add_argument("--stats", action="store_true")
    ap.add_argument("--sweep", default=None, choices=["chunked16k", "policies"],
                    help="ablation sweeps: the chunked 16K prompt (split limit, prefill tile) "
                         "or the fused kernel's role policies; one JSON line per point")
    ap.add_argument("--sweep-points", default=None,
                    help="chunk indices (chunked16k) or workload names (policies), comma-separated")
    ap.add_argument("--only", default=None,
                    choices=["fused", "serial", "two_stream", "prefill_only", "decode_only"],
                    help="time one mode alone (profiler captures); prints a short JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        if args.sweep:
            return run_sweep(args, rank, world, local)
        return run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
