"""Benchmark: hybrid prefill + decode attention, microseconds per call.

One "step" is one ``pod_attn_hybrid`` call (FUSED) on a synthetic hybrid batch
whose inputs are already resident in HBM; L2 is flushed (a write larger than
L2) before every timed call and each call is timed with CUDA events on the
launching stream. The same run also times the library's SERIAL and TWO_STREAM
modes and the prefill-only / decode-only launches, reports the fused
max(FLOP, HBM) roofline fraction with the measured peaks, the fp64 oracle on
the host cores (bounded sample), the clocks seen during the timed region, and
an end-to-end number through the C ABI with host buffers.

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
DEFAULT_WORKLOAD = "llama3_8b"
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

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


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
def oracle_sample_time(batch, budget_s: float, seed: int = 0):
    """Time the fp64 oracle on a random sample of (row, head) items and scale to
    one full call by FLOPs. Returns (us_per_call, cores, description)."""
    import oracle
    cfg = batch.cfg
    H, d = cfg.num_qo_heads, cfg.head_dim
    rng = np.random.default_rng(seed)
    # per-item key counts
    pk = []
    for p, c in zip(batch.priors, batch.chunks):
        pk.append(p + 1 + np.arange(c))
    pk = np.concatenate(pk) if pk else np.zeros(0, np.int64)
    dk = np.asarray(batch.ctx, np.int64)
    total_keys = pk.sum() * H + dk.sum() * H
    # calibrate: a small sample first
    n_threads = oracle.max_threads()
    frac = 1e-4
    spent = 0.0
    for _ in range(6):
        np_items = max(1, int(len(pk) * H * frac))
        nd_items = max(1, int(len(dk) * H * frac)) if len(dk) else 0
        np_items = min(np_items, len(pk) * H)
        nd_items = min(nd_items, len(dk) * H)
        ps = np.sort(rng.choice(len(pk) * H, size=np_items, replace=False)) if len(pk) else None
        ds = np.sort(rng.choice(len(dk) * H, size=nd_items, replace=False)) if len(dk) else None
        t0 = time.perf_counter()
        oracle.hybrid(batch, prefill_sample=ps, decode_sample=ds)
        dt = time.perf_counter() - t0
        keys = (pk[ps // H].sum() if ps is not None else 0) + (dk[ds // H].sum() if ds is not None else 0)
        spent += dt
        if dt > budget_s * 0.3 or spent > budget_s:
            break
        if frac >= 0.25:
            break
        frac = min(0.25, frac * max(2.0, min(8.0, budget_s * 0.4 / max(dt, 1e-3))))
    us = dt / max(keys, 1) * total_keys * 1e6
    desc = ("%d prefill + %d decode (row, head) items drawn at random (%.3g%% of the keys), "
            "scaled to one call by key count; fp64, %d OpenMP threads"
            % (0 if ps is None else len(ps), 0 if ds is None else len(ds),
               100.0 * keys / total_keys, n_threads))
    return us, n_threads, desc, dt


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    batch = W.make_batch(W.get_config(args.workload))
    vals = []
    for i in range(args.warmup + args.steps):
        budget = 0.5 if i < args.warmup else args.ref_step_seconds
        us, cores, desc, _ = oracle_sample_time(batch, budget, seed=i)
        if i >= args.warmup:
            vals.append(us)
    v = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": W.CONFIG_DESCRIPTIONS[args.workload]},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU leg
def time_calls(fn, n, flush_buf, stream, per_call=True):
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


def run_gpu(args, rank, world, local):
    from hybrid_prefill_decode_pod_b200 import pod_attn as pa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    cfg = W.get_config(args.workload)
    batch = W.make_batch(cfg)
    paged = cfg.paged
    pod = pa.context_for(batch, device=local, flags=pa.FLAG_STATS if args.stats else 0)
    db = pa.DeviceBatch(batch, device=dev)
    pre, dec = db.args(pod)
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)

    H, Hk, d = cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim
    f_p, f_d, b_p, b_d = W.algorithmic_work(H, Hk, d, batch.priors, batch.chunks, batch.ctx,
                                            paged=paged)
    F, B = f_p + f_d, b_p + b_d
    tc_peak = peaks["bf16_tflops"] * 1e12
    bw_peak = peaks["hbm_gbs"] * 1e9
    t_star = max(F / tc_peak, B / bw_peak) * 1e6  # us
    bound = "tensor" if F / tc_peak > B / bw_peak else "hbm"

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
                              "us_median": statistics.median(ts), "status": st}), flush=True)
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
    fused_mean = sum(fused) / len(fused)
    fused_med = statistics.median(fused)
    fused_max_ranks = dist_max(fused_mean, world)

    # ---- the library's own baselines and the standalone phases (same run)
    extra_steps = max(5, args.steps // 2)
    serial = time_calls(call(pa.MODE_SERIAL), extra_steps, flush, stream)
    two = time_calls(call(pa.MODE_TWO_STREAM), extra_steps, flush, stream)
    p_only = time_calls(lambda: pod.prefill_only(pre, stream), extra_steps, flush, stream) if pre else [0.0]
    d_only = time_calls(lambda: pod.decode_only(dec, stream), extra_steps, flush, stream) if dec else [0.0]
    plan = None
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

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        us, cores, desc, _ = oracle_sample_time(batch, args.cpu_seconds)
        cpu = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    achieved_tflops = F / (fused_med * 1e-6) / 1e12
    achieved_gbs = B / (fused_med * 1e-6) / 1e9
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved_tflops / peaks["bf16_tflops"]}
    roof["peak_kind"] = peak_kind + " (burst)"
    roof["kernel"] = "pod_fused_kernel"
    roof["traffic"] = committed_traffic(args.workload)
    roof["algorithmic_bytes"] = B
    roof["algorithmic_flops"] = F

    med = statistics.median
    line = {
        "metric": METRIC, "value": fused_max_ranks, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": fused_max_ranks / 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": W.CONFIG_DESCRIPTIONS[args.workload],
                   "l2": "flushed before every timed call (write of %d MB)" % (flush.numel() * 4 >> 20),
                   "mode": "fused", "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roof,
        "fused_roofline_frac": t_star / fused_med,
        "t_star_us": t_star,
        "fused_us": {"mean": fused_mean, "median": fused_med, "p10": float(np.percentile(fused, 10)),
                     "p90": float(np.percentile(fused, 90))},
        "serial_us": med(serial), "two_stream_us": med(two),
        "prefill_only_us": med(p_only), "decode_only_us": med(d_only),
        "speedup_vs_serial": med(serial) / fused_med,
        "speedup_vs_two_stream": med(two) / fused_med,
        "tflops": achieved_tflops, "gbs": achieved_gbs,
        "plan": plan,
        "clocks": clocks,
        "gpu_launches": args.steps,
        "wall_s_timed_region": wall,
        "cpu_baseline": cpu,
        "e2e": e2e,
    }
    if stats:
        line["virtual_cta_mix"] = stats
    pod.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
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
    return {"value": statistics.median(times), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "inputs (Q and every K/V byte the call reads) copied from pinned host memory each step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.CONFIGS) + sorted(W.PROBE_CONFIGS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=2.0)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--stats", action="store_true")
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
        return run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
